/*
 * fftconv_oracle.c -- plain, slow, fp64 reference for the exact causal long
 * convolution.  TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and
 * the benchmark's CPU-baseline leg call it; the product path never does.
 *
 * What it computes (page "FlashFFTConv: Efficient Convolutions for Long
 * Sequences with Tensor Cores", summary paragraph and "Approach"): the exact
 * FFT convolution of a length-N input with a filter as long as the sequence,
 *
 *     y[t] = v[t] * sum_{s=0}^{min(t, L-1)} k[s] * (u*w)[t-s],   0 <= t < N,
 *
 * evaluated by the plain definition y = irfft(rfft(x, 2N) * rfft(k, 2N))[:N]
 * with x = u*w.  The gates w and v are the "gated convolution" of "Key
 * results"; a filter shorter than N (L < N) is the "partial convolution"; a
 * block mask that zeroes rfft bins of the filter is the "frequency-sparse
 * convolution" ("Approach", measured-effects table rows on 75% / 79%
 * frequency-domain sparsity).
 *
 * Everything here is written from the definition of the DFT:
 *   X[f] = sum_t x[t] * exp(-2*pi*i*f*t/M)
 * computed by an own recursive radix-2 decimation-in-time FFT whose twiddles
 * come from cos/sin of 2*pi*(j mod M)/M in double precision.  A second,
 * independent route (the direct O(N*L) causal sum, and a direct O(M^2) DFT)
 * is provided so the tests can pin the FFT route against it.
 *
 * Frequency mask reading (the pages do not define it): rfft bins [0, N) are
 * split into N/32 blocks of 32 consecutive bins; the Nyquist bin N belongs to
 * the last block.  mask[m] == 0 zeroes every bin of block m, and zeroing bin f
 * also zeroes its Hermitian mirror M-f of the full spectrum, so the filter
 * stays real.  mask_h is 1 (one mask for all channels) or H (one per channel).
 *
 * Parity status: every function below is pinned by the CPU tests (brute-force
 * DFT and direct sums, closed forms, Parseval, shift/linearity invariants,
 * hand-computed fixtures).  Nothing here is "parity unpinned".
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct { double re, im; } cplx;

#define ORACLE_BLOCK 32

/* ---------------------------------------------------------------- FFT --- */

/* Twiddle table w[j] = exp(sign * 2*pi*i * j / M) for j < M/2. */
static cplx* make_twiddles(int64_t M, int sign) {
    int64_t half = M / 2 > 0 ? M / 2 : 1;
    cplx* w = (cplx*)malloc(sizeof(cplx) * (size_t)half);
    if (!w) return NULL;
    const double two_pi = 6.283185307179586476925286766559;
    for (int64_t j = 0; j < half; ++j) {
        double a = two_pi * (double)(j % M) / (double)M;
        w[j].re = cos(a);
        w[j].im = (double)sign * sin(a);
    }
    return w;
}

/* Radix-2 decimation in time, out of place.  Transforms the m values
 * in[0], in[stride], ..., in[(m-1)*stride] into out[0..m).  tw[] holds
 * exp(sign*2*pi*i*j/M) for the top-level length M; a sub-transform of length
 * m uses every (M/m)-th entry, passed as twstride. */
static void fft_rec(const cplx* in, cplx* out, int64_t m, int64_t stride,
                    const cplx* tw, int64_t twstride) {
    if (m == 1) { out[0] = in[0]; return; }
    int64_t h = m / 2;
    fft_rec(in, out, h, 2 * stride, tw, 2 * twstride);            /* even t */
    fft_rec(in + stride, out + h, h, 2 * stride, tw, 2 * twstride); /* odd t  */
    for (int64_t k = 0; k < h; ++k) {
        cplx w = tw[k * twstride];
        cplx o = out[k + h];
        cplx t = { w.re * o.re - w.im * o.im, w.re * o.im + w.im * o.re };
        cplx e = out[k];
        out[k].re = e.re + t.re;      out[k].im = e.im + t.im;
        out[k + h].re = e.re - t.re;  out[k + h].im = e.im - t.im;
    }
}

/* In-place length-M DFT of (re, im), M a power of two.  inverse != 0 uses
 * exp(+2*pi*i*f*t/M) and does NOT divide by M.  Returns 0 on success. */
int oracle_fft(double* re, double* im, int64_t M, int inverse) {
    if (M <= 0 || (M & (M - 1))) return -1;
    cplx* a = (cplx*)malloc(sizeof(cplx) * (size_t)M);
    cplx* b = (cplx*)malloc(sizeof(cplx) * (size_t)M);
    cplx* tw = make_twiddles(M, inverse ? +1 : -1);
    if (!a || !b || !tw) { free(a); free(b); free(tw); return -2; }
    for (int64_t i = 0; i < M; ++i) { a[i].re = re[i]; a[i].im = im[i]; }
    fft_rec(a, b, M, 1, tw, 1);
    for (int64_t i = 0; i < M; ++i) { re[i] = b[i].re; im[i] = b[i].im; }
    free(a); free(b); free(tw);
    return 0;
}

/* Direct O(M^2) DFT, the textbook sum, used only to pin oracle_fft. */
int oracle_dft_direct(const double* re, const double* im, double* ore,
                      double* oim, int64_t M, int inverse) {
    const double two_pi = 6.283185307179586476925286766559;
    double sign = inverse ? 1.0 : -1.0;
    for (int64_t f = 0; f < M; ++f) {
        double sr = 0.0, si = 0.0;
        for (int64_t t = 0; t < M; ++t) {
            double a = two_pi * (double)((f * t) % M) / (double)M;
            double c = cos(a), s = sign * sin(a);
            sr += re[t] * c - im[t] * s;
            si += re[t] * s + im[t] * c;
        }
        ore[f] = sr; oim[f] = si;
    }
    return 0;
}

/* ------------------------------------------------------- mask helpers --- */

/* 1 if rfft bin g (0 <= g <= N) survives the block mask row `mrow`. */
static int bin_kept(const uint8_t* mrow, int64_t N, int64_t g) {
    if (!mrow) return 1;
    int64_t nblk = N / ORACLE_BLOCK;
    int64_t blk = g / ORACLE_BLOCK;
    if (blk >= nblk) blk = nblk - 1;           /* Nyquist joins the last block */
    return mrow[blk] != 0;
}

/* ---------------------------------------------------------- FFT route --- */

typedef struct {
    /* problem */
    const double *u, *k, *w, *v;
    const uint8_t* mask;
    const uint8_t* binmask;   /* [binmask_h, 2N] per-bin mask of the full spectrum, or NULL */
    int64_t B, H, N, L, mask_h, binmask_h;
    double* y;
    double* max_imag_ratio;   /* per-thread self-check output */
    /* work split */
    int64_t first, last;      /* sequence index range [first, last) over B*H */
    int status;
} conv_job;

static void* conv_worker(void* arg) {
    conv_job* J = (conv_job*)arg;
    int64_t N = J->N, M = 2 * N, L = J->L;
    cplx* x = (cplx*)malloc(sizeof(cplx) * (size_t)M);
    cplx* X = (cplx*)malloc(sizeof(cplx) * (size_t)M);
    cplx* kap = (cplx*)malloc(sizeof(cplx) * (size_t)M);
    cplx* K = (cplx*)malloc(sizeof(cplx) * (size_t)M);
    cplx* twf = make_twiddles(M, -1);
    cplx* twi = make_twiddles(M, +1);
    int64_t cached_h = -1;
    double worst = 0.0;
    if (!x || !X || !kap || !K || !twf || !twi) { J->status = -2; goto done; }
    for (int64_t s = J->first; s < J->last; ++s) {
        int64_t h = s % J->H;
        const double* us = J->u + s * N;
        const double* ws = J->w ? J->w + s * N : NULL;
        const double* vs = J->v ? J->v + s * N : NULL;
        if (h != cached_h) {
            /* K = FFT_M(k zero-padded to M); masked bins and mirrors zeroed. */
            for (int64_t t = 0; t < M; ++t) {
                kap[t].re = (t < L) ? J->k[h * L + t] : 0.0;
                kap[t].im = 0.0;
            }
            fft_rec(kap, K, M, 1, twf, 1);
            if (J->mask) {
                const uint8_t* mrow = J->mask + (J->mask_h == 1 ? 0 : h) * (N / ORACLE_BLOCK);
                for (int64_t g = 0; g <= N; ++g) {
                    if (!bin_kept(mrow, N, g)) {
                        K[g].re = K[g].im = 0.0;
                        K[(M - g) % M].re = K[(M - g) % M].im = 0.0;
                    }
                }
            }
            if (J->binmask) {
                /* a zero byte zeroes bin f of the full M-point spectrum */
                const uint8_t* brow = J->binmask + (J->binmask_h == 1 ? 0 : h) * M;
                for (int64_t f = 0; f < M; ++f)
                    if (!brow[f]) K[f].re = K[f].im = 0.0;
            }
            cached_h = h;
        }
        /* x = u*w, zero-padded to M */
        for (int64_t t = 0; t < M; ++t) {
            x[t].re = (t < N) ? us[t] * (ws ? ws[t] : 1.0) : 0.0;
            x[t].im = 0.0;
        }
        fft_rec(x, X, M, 1, twf, 1);
        for (int64_t f = 0; f < M; ++f) {
            cplx a = X[f], b = K[f];
            x[f].re = a.re * b.re - a.im * b.im;
            x[f].im = a.re * b.im + a.im * b.re;
        }
        fft_rec(x, X, M, 1, twi, 1);          /* unnormalised inverse */
        double zmax = 0.0, imax = 0.0;
        for (int64_t t = 0; t < M; ++t) {
            double ar = fabs(X[t].re), ai = fabs(X[t].im);
            if (ar > zmax) zmax = ar;
            if (ai > zmax) zmax = ai;
            if (ai > imax) imax = ai;
        }
        if (zmax > 0.0 && imax / zmax > worst) worst = imax / zmax;
        for (int64_t t = 0; t < N; ++t) {
            double z = X[t].re / (double)M;
            J->y[s * N + t] = vs ? vs[t] * z : z;
        }
    }
    J->status = 0;
done:
    if (J->max_imag_ratio) *J->max_imag_ratio = worst;
    free(x); free(X); free(kap); free(K); free(twf); free(twi);
    return NULL;
}

/* The FFT route over all B*H sequences, split across nthreads POSIX threads.
 *   u, y      : [B, H, N] row-major
 *   k         : [H, L]
 *   w, v      : [B, H, N] or NULL (gate absent == all ones)
 *   mask      : [mask_h, N/32] bytes (1 = keep) or NULL
 *   imag_ratio: out, max over sequences of max|Im z| / max|z| (self-check)
 * Returns 0, or a negative code for bad arguments / allocation failure. */
static int run_conv(const double* u, const double* k, double* y, int64_t B,
                    int64_t H, int64_t N, int64_t L, const double* w,
                    const double* v, const uint8_t* mask, int64_t mask_h,
                    const uint8_t* binmask, int64_t binmask_h,
                    int nthreads, double* imag_ratio);

int oracle_fftconv(const double* u, const double* k, double* y, int64_t B,
                   int64_t H, int64_t N, int64_t L, const double* w,
                   const double* v, const uint8_t* mask, int64_t mask_h,
                   int nthreads, double* imag_ratio) {
    if (mask && (mask_h != 1 && mask_h != H)) return -1;
    if (mask && N < ORACLE_BLOCK) return -1;
    return run_conv(u, k, y, B, H, N, L, w, v, mask, mask_h, NULL, 0, nthreads, imag_ratio);
}

/* As oracle_fftconv with a per-bin mask of the full 2N-point filter spectrum:
 * binmask is [binmask_h, 2N] bytes (binmask_h 1 or H), a zero byte zeroes
 * that bin.  The caller keeps each row Hermitian-symmetric (binmask[f] ==
 * binmask[(2N - f) mod 2N]) so that y stays real; imag_ratio reports it. */
int oracle_fftconv_bins(const double* u, const double* k, double* y, int64_t B,
                        int64_t H, int64_t N, int64_t L, const double* w,
                        const double* v, const uint8_t* binmask, int64_t binmask_h,
                        int nthreads, double* imag_ratio) {
    if (!binmask || (binmask_h != 1 && binmask_h != H)) return -1;
    return run_conv(u, k, y, B, H, N, L, w, v, NULL, 0, binmask, binmask_h, nthreads, imag_ratio);
}

static int run_conv(const double* u, const double* k, double* y, int64_t B,
                    int64_t H, int64_t N, int64_t L, const double* w,
                    const double* v, const uint8_t* mask, int64_t mask_h,
                    const uint8_t* binmask, int64_t binmask_h,
                    int nthreads, double* imag_ratio) {
    if (B < 0 || H <= 0 || N <= 0 || (N & (N - 1)) || L <= 0 || L > N) return -1;
    int64_t S = B * H;
    if (S == 0) { if (imag_ratio) *imag_ratio = 0.0; return 0; }
    if (nthreads < 1) nthreads = 1;
    if (nthreads > S) nthreads = (int)S;
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
    conv_job* jobs = (conv_job*)calloc((size_t)nthreads, sizeof(conv_job));
    double* ratios = (double*)calloc((size_t)nthreads, sizeof(double));
    if (!th || !jobs || !ratios) { free(th); free(jobs); free(ratios); return -2; }
    for (int i = 0; i < nthreads; ++i) {
        conv_job* J = &jobs[i];
        J->u = u; J->k = k; J->w = w; J->v = v; J->mask = mask;
        J->binmask = binmask; J->binmask_h = binmask_h;
        J->B = B; J->H = H; J->N = N; J->L = L; J->mask_h = mask_h; J->y = y;
        J->max_imag_ratio = &ratios[i];
        J->first = S * i / nthreads;
        J->last = S * (i + 1) / nthreads;
        J->status = -3;
        if (nthreads == 1) conv_worker(J);
        else pthread_create(&th[i], NULL, conv_worker, J);
    }
    int rc = 0;
    double worst = 0.0;
    for (int i = 0; i < nthreads; ++i) {
        if (nthreads > 1) pthread_join(th[i], NULL);
        if (jobs[i].status != 0) rc = jobs[i].status;
        if (ratios[i] > worst) worst = ratios[i];
    }
    if (imag_ratio) *imag_ratio = worst;
    free(th); free(jobs); free(ratios);
    return rc;
}

/* rfft of each zero-padded filter: out[h, f, 0..1] = K[h, f] for f in [0, N],
 * masked bins zeroed as in oracle_fftconv. */
int oracle_filter_rfft(const double* k, double* out, int64_t H, int64_t N,
                       int64_t L, const uint8_t* mask, int64_t mask_h) {
    if (H <= 0 || N <= 0 || (N & (N - 1)) || L <= 0 || L > N) return -1;
    int64_t M = 2 * N;
    cplx* a = (cplx*)malloc(sizeof(cplx) * (size_t)M);
    cplx* b = (cplx*)malloc(sizeof(cplx) * (size_t)M);
    cplx* tw = make_twiddles(M, -1);
    if (!a || !b || !tw) { free(a); free(b); free(tw); return -2; }
    for (int64_t h = 0; h < H; ++h) {
        for (int64_t t = 0; t < M; ++t) { a[t].re = (t < L) ? k[h * L + t] : 0.0; a[t].im = 0.0; }
        fft_rec(a, b, M, 1, tw, 1);
        const uint8_t* mrow = mask ? mask + (mask_h == 1 ? 0 : h) * (N / ORACLE_BLOCK) : NULL;
        for (int64_t f = 0; f <= N; ++f) {
            int keep = bin_kept(mrow, N, f);
            out[(h * (N + 1) + f) * 2 + 0] = keep ? b[f].re : 0.0;
            out[(h * (N + 1) + f) * 2 + 1] = keep ? b[f].im : 0.0;
        }
    }
    free(a); free(b); free(tw);
    return 0;
}

/* ------------------------------------------------------- direct route --- */

/* Direct causal sum at the listed (sequence, t) samples:
 *   y = v[t] * sum_{s=0}^{min(t,L-1)} k[h,s] * u[t-s] * w[t-s]
 * seq[i] indexes the flattened [B*H] sequences (h = seq % H).  With ns < 0 the
 * routine evaluates every t of every sequence (y is then [B,H,N]). */
int oracle_direct_conv(const double* u, const double* k, double* y, int64_t B,
                       int64_t H, int64_t N, int64_t L, const double* w,
                       const double* v, const int64_t* seq, const int64_t* ts,
                       int64_t ns) {
    if (H <= 0 || N <= 0 || L <= 0 || L > N) return -1;
    if (ns < 0) {
        for (int64_t s = 0; s < B * H; ++s) {
            int64_t h = s % H;
            for (int64_t t = 0; t < N; ++t) {
                double acc = 0.0;
                int64_t smax = t < L - 1 ? t : L - 1;
                for (int64_t q = 0; q <= smax; ++q) {
                    double x = u[s * N + t - q] * (w ? w[s * N + t - q] : 1.0);
                    acc += k[h * L + q] * x;
                }
                y[s * N + t] = (v ? v[s * N + t] : 1.0) * acc;
            }
        }
        return 0;
    }
    for (int64_t i = 0; i < ns; ++i) {
        int64_t s = seq[i], t = ts[i], h = s % H;
        if (s < 0 || s >= B * H || t < 0 || t >= N) return -1;
        double acc = 0.0;
        int64_t smax = t < L - 1 ? t : L - 1;
        for (int64_t q = 0; q <= smax; ++q) {
            double x = u[s * N + t - q] * (w ? w[s * N + t - q] : 1.0);
            acc += k[h * L + q] * x;
        }
        y[i] = (v ? v[s * N + t] : 1.0) * acc;
    }
    return 0;
}

/* Effective time-domain filter of a masked spectrum, by the direct inverse
 * DFT (no FFT involved): keff[h, t] = (1/M) sum_f Kmasked[f] e^{+2 pi i f t/M},
 * t in [0, M).  Kmasked is built from the direct DFT of the padded filter.
 * O(M^2) per channel: tiny sizes only. */
int oracle_masked_filter_direct(const double* k, double* keff, int64_t H,
                                int64_t N, int64_t L, const uint8_t* mask,
                                int64_t mask_h) {
    if (H <= 0 || N <= 0 || L <= 0 || L > N) return -1;
    int64_t M = 2 * N;
    double* kr = (double*)calloc((size_t)M, sizeof(double));
    double* ki = (double*)calloc((size_t)M, sizeof(double));
    double* Kr = (double*)malloc(sizeof(double) * (size_t)M);
    double* Ki = (double*)malloc(sizeof(double) * (size_t)M);
    double* zr = (double*)malloc(sizeof(double) * (size_t)M);
    double* zi = (double*)malloc(sizeof(double) * (size_t)M);
    if (!kr || !ki || !Kr || !Ki || !zr || !zi) {
        free(kr); free(ki); free(Kr); free(Ki); free(zr); free(zi); return -2;
    }
    for (int64_t h = 0; h < H; ++h) {
        for (int64_t t = 0; t < M; ++t) { kr[t] = (t < L) ? k[h * L + t] : 0.0; ki[t] = 0.0; }
        oracle_dft_direct(kr, ki, Kr, Ki, M, 0);
        const uint8_t* mrow = mask ? mask + (mask_h == 1 ? 0 : h) * (N / ORACLE_BLOCK) : NULL;
        for (int64_t f = 0; f < M; ++f) {
            int64_t g = f <= N ? f : M - f;             /* rfft bin of f */
            if (!bin_kept(mrow, N, g)) { Kr[f] = 0.0; Ki[f] = 0.0; }
        }
        oracle_dft_direct(Kr, Ki, zr, zi, M, 1);
        for (int64_t t = 0; t < M; ++t) keff[h * M + t] = zr[t] / (double)M;
    }
    free(kr); free(ki); free(Kr); free(Ki); free(zr); free(zi);
    return 0;
}

/* Same effective filter as oracle_masked_filter_direct, but by the FFT route
 * (forward and inverse through fft_rec); usable at full sizes. */
int oracle_masked_filter_fft(const double* k, double* keff, int64_t H,
                             int64_t N, int64_t L, const uint8_t* mask,
                             int64_t mask_h) {
    if (H <= 0 || N <= 0 || (N & (N - 1)) || L <= 0 || L > N) return -1;
    int64_t M = 2 * N;
    cplx* a = (cplx*)malloc(sizeof(cplx) * (size_t)M);
    cplx* b = (cplx*)malloc(sizeof(cplx) * (size_t)M);
    cplx* twf = make_twiddles(M, -1);
    cplx* twi = make_twiddles(M, +1);
    if (!a || !b || !twf || !twi) { free(a); free(b); free(twf); free(twi); return -2; }
    for (int64_t h = 0; h < H; ++h) {
        for (int64_t t = 0; t < M; ++t) { a[t].re = (t < L) ? k[h * L + t] : 0.0; a[t].im = 0.0; }
        fft_rec(a, b, M, 1, twf, 1);
        const uint8_t* mrow = mask ? mask + (mask_h == 1 ? 0 : h) * (N / ORACLE_BLOCK) : NULL;
        for (int64_t f = 0; f < M; ++f) {
            int64_t g = f <= N ? f : M - f;
            if (!bin_kept(mrow, N, g)) { b[f].re = 0.0; b[f].im = 0.0; }
        }
        fft_rec(b, a, M, 1, twi, 1);
        for (int64_t t = 0; t < M; ++t) keff[h * M + t] = a[t].re / (double)M;
    }
    free(a); free(b); free(twf); free(twi);
    return 0;
}

/* Circular sum with a full-length effective filter at sampled points:
 *   y = v[t] * sum_{s=0}^{M-1} keff[h, s] * x[(t - s) mod M],  x = u*w padded.
 * keff is [H, M].  Used for the frequency-sparse path. */
int oracle_circular_conv_samples(const double* u, const double* keff, double* y,
                                 int64_t B, int64_t H, int64_t N,
                                 const double* w, const double* v,
                                 const int64_t* seq, const int64_t* ts,
                                 int64_t ns) {
    int64_t M = 2 * N;
    for (int64_t i = 0; i < ns; ++i) {
        int64_t s = seq[i], t = ts[i], h = s % H;
        if (s < 0 || s >= B * H || t < 0 || t >= N) return -1;
        double acc = 0.0;
        for (int64_t q = 0; q < M; ++q) {
            int64_t src = ((t - q) % M + M) % M;
            if (src >= N) continue;                      /* zero padding */
            double x = u[s * N + src] * (w ? w[s * N + src] : 1.0);
            acc += keff[h * M + q] * x;
        }
        y[i] = (v ? v[s * N + t] : 1.0) * acc;
    }
    return 0;
}

/* ------------------------------------------------------- backward pass --- */

/* Gradients of the gated causal convolution, for training (page
 * "FlashFFTConv: Efficient Convolutions for Long Sequences with Tensor Cores",
 * "Key results": models trained with the convolution; the page states no
 * backward, so these are the plain adjoints of the forward definition).
 * With x = u*w, z[t] = sum_{s<=min(t,L-1)} k[s] x[t-s], y = v*z and the
 * incoming gradient dy, and g = dy*v:
 *     dv[t]  = dy[t] * z[t]
 *     dx[t]  = sum_{s=0}^{min(L-1, N-1-t)} g[t+s] * k[s]      (correlation)
 *     du[t]  = dx[t] * w[t],   dw[t] = dx[t] * u[t]
 *     dk[h,s] = sum_b sum_{t=s}^{N-1} g_b[t] * x_b[t-s],   s < L
 * Direct sums, O(N*L) per sequence.  Outputs may be NULL (not computed); dw
 * needs w, dv needs v.  du, dw, dv: [B, H, N]; dk: [H, L].  Gates absent
 * (NULL) are all ones. */
int oracle_conv_backward_direct(const double* u, const double* k, const double* w,
                                const double* v, const double* dy, int64_t B, int64_t H,
                                int64_t N, int64_t L, double* du, double* dw, double* dv,
                                double* dk) {
    if (B < 0 || H <= 0 || N <= 0 || L <= 0 || L > N) return -1;
    if ((dw && !w) || (dv && !v)) return -1;
    double* g = (double*)malloc(sizeof(double) * (size_t)N);
    double* x = (double*)malloc(sizeof(double) * (size_t)N);
    if (!g || !x) { free(g); free(x); return -2; }
    if (dk) memset(dk, 0, sizeof(double) * (size_t)(H * L));
    for (int64_t s = 0; s < B * H; ++s) {
        int64_t h = s % H;
        const double* kh = k + h * L;
        for (int64_t t = 0; t < N; ++t) {
            x[t] = u[s * N + t] * (w ? w[s * N + t] : 1.0);
            g[t] = dy[s * N + t] * (v ? v[s * N + t] : 1.0);
        }
        if (dv) {
            for (int64_t t = 0; t < N; ++t) {
                double z = 0.0;
                int64_t smax = t < L - 1 ? t : L - 1;
                for (int64_t q = 0; q <= smax; ++q) z += kh[q] * x[t - q];
                dv[s * N + t] = dy[s * N + t] * z;
            }
        }
        if (du || dw) {
            for (int64_t t = 0; t < N; ++t) {
                double acc = 0.0;
                int64_t smax = (N - 1 - t) < (L - 1) ? (N - 1 - t) : (L - 1);
                for (int64_t q = 0; q <= smax; ++q) acc += g[t + q] * kh[q];
                if (du) du[s * N + t] = acc * (w ? w[s * N + t] : 1.0);
                if (dw) dw[s * N + t] = acc * u[s * N + t];
            }
        }
        if (dk) {
            for (int64_t q = 0; q < L; ++q) {
                double acc = 0.0;
                for (int64_t t = q; t < N; ++t) acc += g[t] * x[t - q];
                dk[h * L + q] += acc;
            }
        }
    }
    free(g); free(x);
    return 0;
}

/* The same gradients by the FFT route (own radix-2 FFT, length M = 2N):
 * dx = IFFT(FFT(g) * conj(FFT(k)))[:N] / M -- the circular correlation of the
 * zero-padded g with the zero-padded k, which equals the linear correlation
 * for t < N because the wrapped terms meet the padding -- and
 * dk = IFFT(sum_b FFT(g_b) * conj(FFT(x_b)))[:L] / M; dv through the forward
 * FFT route.  Usable at full sizes; pinned against the direct sums. */
int oracle_conv_backward_fft(const double* u, const double* k, const double* w,
                             const double* v, const double* dy, int64_t B, int64_t H,
                             int64_t N, int64_t L, double* du, double* dw, double* dv,
                             double* dk) {
    if (B < 0 || H <= 0 || N <= 0 || (N & (N - 1)) || L <= 0 || L > N) return -1;
    if ((dw && !w) || (dv && !v)) return -1;
    int64_t M = 2 * N;
    cplx* a = (cplx*)malloc(sizeof(cplx) * (size_t)M);
    cplx* G = (cplx*)malloc(sizeof(cplx) * (size_t)M);
    cplx* X = (cplx*)malloc(sizeof(cplx) * (size_t)M);
    cplx* K = (cplx*)malloc(sizeof(cplx) * (size_t)M);
    cplx* DK = (cplx*)malloc(sizeof(cplx) * (size_t)M);
    cplx* twf = make_twiddles(M, -1);
    cplx* twi = make_twiddles(M, +1);
    int rc = 0;
    if (!a || !G || !X || !K || !DK || !twf || !twi) { rc = -2; goto out; }
    for (int64_t h = 0; h < H; ++h) {
        for (int64_t t = 0; t < M; ++t) { a[t].re = (t < L) ? k[h * L + t] : 0.0; a[t].im = 0.0; }
        fft_rec(a, K, M, 1, twf, 1);
        for (int64_t f = 0; f < M; ++f) DK[f].re = DK[f].im = 0.0;
        for (int64_t b = 0; b < B; ++b) {
            int64_t s = b * H + h;
            for (int64_t t = 0; t < M; ++t) {
                a[t].re = (t < N) ? dy[s * N + t] * (v ? v[s * N + t] : 1.0) : 0.0;
                a[t].im = 0.0;
            }
            fft_rec(a, G, M, 1, twf, 1);
            for (int64_t t = 0; t < M; ++t) {
                a[t].re = (t < N) ? u[s * N + t] * (w ? w[s * N + t] : 1.0) : 0.0;
                a[t].im = 0.0;
            }
            fft_rec(a, X, M, 1, twf, 1);
            /* dk: accumulate G * conj(X) */
            for (int64_t f = 0; f < M; ++f) {
                DK[f].re += G[f].re * X[f].re + G[f].im * X[f].im;
                DK[f].im += G[f].im * X[f].re - G[f].re * X[f].im;
            }
            if (dv) {   /* z = IFFT(X * K) */
                for (int64_t f = 0; f < M; ++f) {
                    a[f].re = X[f].re * K[f].re - X[f].im * K[f].im;
                    a[f].im = X[f].re * K[f].im + X[f].im * K[f].re;
                }
                fft_rec(a, X, M, 1, twi, 1);
                for (int64_t t = 0; t < N; ++t) dv[s * N + t] = dy[s * N + t] * X[t].re / (double)M;
            }
            if (du || dw) {   /* dx = IFFT(G * conj(K)) */
                for (int64_t f = 0; f < M; ++f) {
                    a[f].re = G[f].re * K[f].re + G[f].im * K[f].im;
                    a[f].im = G[f].im * K[f].re - G[f].re * K[f].im;
                }
                fft_rec(a, G, M, 1, twi, 1);
                for (int64_t t = 0; t < N; ++t) {
                    double dx = G[t].re / (double)M;
                    if (du) du[s * N + t] = dx * (w ? w[s * N + t] : 1.0);
                    if (dw) dw[s * N + t] = dx * u[s * N + t];
                }
            }
        }
        if (dk) {
            fft_rec(DK, a, M, 1, twi, 1);
            for (int64_t q = 0; q < L; ++q) dk[h * L + q] = a[q].re / (double)M;
        }
    }
out:
    free(a); free(G); free(X); free(K); free(DK); free(twf); free(twi);
    return rc;
}
