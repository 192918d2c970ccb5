// simt_kernels.cu -- fp32 FFT-convolution kernels on the FP32 lanes.
//
// Fused path (one launch): one CTA per pair of batch rows of one channel.  The
// two real sequences ride in the real and imaginary parts of one complex
// sequence ("two for one": the filter is real, so its spectrum is Hermitian
// and the real/imaginary parts of the result are the two convolutions).  The
// whole length-M (= 2N) transform stays in shared memory: the first stage
// reads u*w straight from global memory (only the nonzero half), the last
// forward stage, the product with K_f and the first inverse stage are fused
// in registers, and the last inverse stage writes y*v for t < N only.
//
// Staged path (three launches per chunk of pairs, any N): M = R*C with a
// column pass (length-R DFTs at stride C plus the exp(-2 pi i c r/M)
// twiddle), a row pass (length-C forward DFT, product with K_f, inverse) and
// an inverse column pass, through a plan-owned workspace.  This is the
// "I/O between memory levels" regime of the FlashFFTConv page (Limitations).
#include <cmath>

#include "internal.h"
#include "simt_fft.cuh"

namespace fftconv {

namespace {

constexpr int kMaskBlock = 32;

// ------------------------------------------------------------ pair I/O ---

template <typename T>
struct PairRows {
    const T* u0 = nullptr; const T* u1 = nullptr;
    const T* w0 = nullptr; const T* w1 = nullptr;
    const T* v0 = nullptr; const T* v1 = nullptr;
    T* y0 = nullptr; T* y1 = nullptr;
    int nvalid = 0;   // inputs at t >= nvalid read as zero (filter length)
    bool vec4 = false;  // rows aligned for 4-element vector accesses (load4 / store4)

    __device__ __forceinline__ float2 load(int t) const {
        if (t >= nvalid) return make_float2(0.f, 0.f);
        float a = to_f32(u0[t]);
        if (w0) a *= to_f32(w0[t]);
        float b = 0.f;
        if (u1) {
            b = to_f32(u1[t]);
            if (w1) b *= to_f32(w1[t]);
        }
        return make_float2(a, b);
    }
    // Four consecutive positions t .. t+3 (t a multiple of 4) with one vector
    // access per row where the rows allow it; positions at or past nvalid
    // read as zero.
    __device__ __forceinline__ void load4(int t, float2 (&x)[4]) const {
        if (vec4 && t + 4 <= nvalid) {
            float a[4], b[4] = {0.f, 0.f, 0.f, 0.f}, g[4];
            ld4(u0 + t, a);
            if (w0) { ld4(w0 + t, g); for (int e = 0; e < 4; ++e) a[e] *= g[e]; }
            if (u1) {
                ld4(u1 + t, b);
                if (w1) { ld4(w1 + t, g); for (int e = 0; e < 4; ++e) b[e] *= g[e]; }
            }
            for (int e = 0; e < 4; ++e) x[e] = make_float2(a[e], b[e]);
        } else {
            for (int e = 0; e < 4; ++e) x[e] = load(t + e);
        }
    }
    __device__ __forceinline__ void store4(int t, const float2 (&z)[4]) const {
        if (!vec4) {
            for (int e = 0; e < 4; ++e) store(t + e, z[e]);
            return;
        }
        float a[4], b[4], g[4];
        for (int e = 0; e < 4; ++e) { a[e] = z[e].x; b[e] = z[e].y; }
        if (v0) { ld4(v0 + t, g); for (int e = 0; e < 4; ++e) a[e] *= g[e]; }
        st4(y0 + t, a);
        if (y1) {
            if (v1) { ld4(v1 + t, g); for (int e = 0; e < 4; ++e) b[e] *= g[e]; }
            st4(y1 + t, b);
        }
    }
    static __device__ __forceinline__ void ld4(const T* p, float (&o)[4]) {
        if constexpr (sizeof(T) == 4) {
            const float4 q = __ldg(reinterpret_cast<const float4*>(p));
            o[0] = q.x; o[1] = q.y; o[2] = q.z; o[3] = q.w;
        } else {
            const uint2 q = __ldg(reinterpret_cast<const uint2*>(p));
            const T* h = reinterpret_cast<const T*>(&q);
            for (int e = 0; e < 4; ++e) o[e] = to_f32(h[e]);
        }
    }
    static __device__ __forceinline__ void st4(T* p, const float (&v)[4]) {
        if constexpr (sizeof(T) == 4) {
            *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
        } else {
            T h[4];
            for (int e = 0; e < 4; ++e) h[e] = from_f32<T>(v[e]);
            *reinterpret_cast<uint2*>(p) = *reinterpret_cast<const uint2*>(h);
        }
    }
    __device__ __forceinline__ void store(int t, float2 z) const {
        float a = z.x, b = z.y;
        if (v0) a *= to_f32(v0[t]);
        y0[t] = from_f32<T>(a);
        if (y1) {
            if (v1) b *= to_f32(v1[t]);
            y1[t] = from_f32<T>(b);
        }
    }
};

// Rows of pair `pair` (pairs are channel-major: all batch pairs of channel 0
// first, so consecutive CTAs share the channel's K_f in L2).
template <typename T>
__device__ __forceinline__ PairRows<T> pair_rows(const ForwardArgs& a, int64_t H, int64_t N,
                                                 int64_t pair, int* h_out) {
    const int64_t PB = (a.B + 1) / 2;
    const int64_t h = pair / PB;
    const int64_t b0 = 2 * (pair % PB), b1 = b0 + 1;
    const int64_t o0 = (b0 * H + h) * N, o1 = (b1 * H + h) * N;
    const bool has1 = b1 < a.B;
    PairRows<T> r;
    r.u0 = (const T*)a.u + o0;
    r.u1 = has1 ? (const T*)a.u + o1 : nullptr;
    if (a.w) { r.w0 = (const T*)a.w + o0; r.w1 = has1 ? (const T*)a.w + o1 : nullptr; }
    if (a.v) { r.v0 = (const T*)a.v + o0; r.v1 = has1 ? (const T*)a.v + o1 : nullptr; }
    r.y0 = (T*)a.y + o0;
    r.y1 = has1 ? (T*)a.y + o1 : nullptr;
    r.nvalid = (int)N;
    r.vec4 = (N % 4) == 0;      // rows start at multiples of N; buffers are 16-byte aligned
    *h_out = (int)h;
    return r;
}

// 1 if rfft bin of full-spectrum frequency f survives the mask row.
__device__ __forceinline__ bool bin_kept(const uint8_t* __restrict__ mrow, int64_t f, int64_t N) {
    const int64_t M = 2 * N;
    const int64_t g = f <= N ? f : M - f;
    int64_t blk = g / kMaskBlock;
    const int64_t nblk = N / kMaskBlock;
    if (blk >= nblk) blk = nblk - 1;
    return __ldg(&mrow[blk]) != 0;
}

__device__ __forceinline__ float2 tw_M(const float2* __restrict__ lo, const float2* __restrict__ hi,
                                       int split, int64_t e) {
    return cmul(__ldg(&hi[e >> split]), __ldg(&lo[e & ((1LL << split) - 1)]));
}

// ------------------------------------------------------- fused kernel ---

template <int LOGM>
constexpr int fused_threads() {
    return (1 << LOGM) / 32 < 128 ? 128 : ((1 << LOGM) / 32 > 512 ? 512 : (1 << LOGM) / 32);
}

// Stage 0 of the fused transform, reading the zero-padded input from global
// memory: position j*S + r, j < R/2 (t < N); the upper half is zero.
template <int LOGM, int NT, typename T, typename IOT = PairRows<T>>
__device__ __forceinline__ void first_stage_global(float2* s, const float2* __restrict__ tw,
                                                   const IOT& io, int tid) {
    constexpr int LB = Sched<LOGM>::bits(0);
    constexpr int R = 1 << LB;
    constexpr int S = 1 << (LOGM - LB);
    for (int r = tid; r < S; r += NT) {
        float2 x[R];
#pragma unroll
        for (int j = 0; j < R / 2; ++j) x[j] = io.load(j * S + r);
        Dft<R, -1>::run_half_input(x);
        twiddle_powers<R, false>(x, tw, r);
#pragma unroll
        for (int c = 0; c < R; ++c) s[sidx<1>(c * S + r, 0)] = x[c];
    }
}

// Inverse of stage 0, writing y = v * z for t < N only.
template <int LOGM, int NT, typename T>
__device__ __forceinline__ void last_stage_global(const float2* s, const float2* __restrict__ tw,
                                                  const PairRows<T>& io, int tid) {
    constexpr int LB = Sched<LOGM>::bits(0);
    constexpr int R = 1 << LB;
    constexpr int S = 1 << (LOGM - LB);
    for (int r = tid; r < S; r += NT) {
        float2 x[R];
#pragma unroll
        for (int c = 0; c < R; ++c) x[c] = s[sidx<1>(c * S + r, 0)];
        twiddle_powers<R, true>(x, tw, r);
        Dft<R, +1>::run(x);
#pragma unroll
        for (int j = 0; j < R / 2; ++j) io.store(j * S + r, x[j]);
    }
}

// Last forward stage (unit stride), product with the filter spectrum and
// first inverse stage, fused in registers.  freq(p) maps a permuted position
// to its full-spectrum frequency for the mask; Krow is indexed by position.
template <int LOGL, int NT, typename FreqFn>
__device__ __forceinline__ void middle_stage(float2* s, const float2* __restrict__ Krow,
                                             const uint8_t* __restrict__ mrow, int64_t N,
                                             FreqFn freq, int tid) {
    constexpr int I = Sched<LOGL>::K - 1;
    constexpr int LB = Sched<LOGL>::bits(I);
    constexpr int R = 1 << LB;
    static_assert(Sched<LOGL>::stride_bits(I) == 0, "middle stage must have unit stride");
    constexpr int G = (1 << LOGL) / R;
    for (int g = tid; g < G; g += NT) {
        const int base = g * R;
        float2 x[R];
#pragma unroll
        for (int c = 0; c < R; ++c) x[c] = s[sidx<1>(base + c, 0)];
        Dft<R, -1>::run(x);
        const float4* K4 = reinterpret_cast<const float4*>(Krow + base);
#pragma unroll
        for (int c = 0; c < R; c += 2) {
            float4 kk = __ldg(&K4[c / 2]);
            float2 k0 = make_float2(kk.x, kk.y), k1 = make_float2(kk.z, kk.w);
            if (mrow) {
                if (!bin_kept(mrow, freq(base + c), N)) k0 = make_float2(0.f, 0.f);
                if (!bin_kept(mrow, freq(base + c + 1), N)) k1 = make_float2(0.f, 0.f);
            }
            x[c] = cmul(x[c], k0);
            x[c + 1] = cmul(x[c + 1], k1);
        }
        Dft<R, +1>::run(x);
#pragma unroll
        for (int j = 0; j < R; ++j) s[sidx<1>(base + j, 0)] = x[j];
    }
}

template <int LOGM, typename T>
__global__ void __launch_bounds__(fused_threads<LOGM>())
simt_fused_kernel(ForwardArgs a, int64_t H, const float2* __restrict__ tw) {
    constexpr int NT = fused_threads<LOGM>();
    constexpr int K = Sched<LOGM>::K;
    static_assert(K >= 2, "fused path needs at least two stages");
    extern __shared__ float2 s[];
    const int tid = threadIdx.x;
    const int64_t N = (int64_t)1 << (LOGM - 1);
    int h;
    const PairRows<T> io = pair_rows<T>(a, H, N, blockIdx.x, &h);
    const float2* Krow = (const float2*)a.Kf + (int64_t)h * (1 << LOGM);
    const uint8_t* mrow = a.mask ? a.mask + (a.mask_h == 1 ? 0 : h) * (N / kMaskBlock) : nullptr;

    first_stage_global<LOGM, NT, T>(s, tw, io, tid);
    __syncthreads();
    fwd_stages<LOGM, 1, K - 1, 1, NT>(s, tw, 0, tid);
    middle_stage<LOGM, NT>(s, Krow, mrow, N, [](int p) { return perm_to_freq(p, LOGM); }, tid);
    __syncthreads();
    inv_stages<LOGM, 1, K - 1, 1, NT>(s, tw, 0, tid);
    last_stage_global<LOGM, NT, T>(s, tw, io, tid);
}

// K_f[h, p] = FFT_M(k_h zero-padded)[freq(p)] / M, one channel per CTA.
template <int LOGM, typename T>
__global__ void __launch_bounds__(fused_threads<LOGM>())
simt_fused_precompute_kernel(const T* __restrict__ k, int64_t L, float2* __restrict__ Kf,
                             const float2* __restrict__ tw) {
    constexpr int NT = fused_threads<LOGM>();
    constexpr int K = Sched<LOGM>::K;
    extern __shared__ float2 s[];
    const int tid = threadIdx.x;
    const int h = blockIdx.x;
    PairRows<T> io;
    io.u0 = k + (int64_t)h * L;
    io.nvalid = (int)L;
    first_stage_global<LOGM, NT, T>(s, tw, io, tid);
    __syncthreads();
    fwd_stages<LOGM, 1, K, 1, NT>(s, tw, 0, tid);
    const float inv = 1.0f / (float)(1 << LOGM);
    float2* out = Kf + (int64_t)h * (1 << LOGM);
    for (int p = tid; p < (1 << LOGM); p += NT) out[p] = cscale(s[sidx<1>(p, 0)], inv);
}

// Same transform written in the tensor-core kernel's filter format for
// M = 8192: per channel, 8192 complex fp16 values K[f] / s_h at position
// ((c2*2 + c3/4)*32 + c1)*4 + c3%4 (f = c1 + 32 c2 + 1024 c3), with
// s_h = max |Re|, |Im| over the channel stored after the H rows.
template <typename T>
__global__ void __launch_bounds__(fused_threads<13>())
simt_precompute_tc8192_kernel(const T* __restrict__ k, int64_t L, __half2* __restrict__ Kh,
                              float* __restrict__ scales, const float2* __restrict__ tw) {
    constexpr int LOGM = 13;
    constexpr int NT = fused_threads<LOGM>();
    constexpr int K = Sched<LOGM>::K;
    extern __shared__ float2 s[];
    __shared__ float red[NT / 32];
    const int tid = threadIdx.x;
    const int h = blockIdx.x;
    PairRows<T> io;
    io.u0 = k + (int64_t)h * L;
    io.nvalid = (int)L;
    first_stage_global<LOGM, NT, T>(s, tw, io, tid);
    __syncthreads();
    fwd_stages<LOGM, 1, K, 1, NT>(s, tw, 0, tid);
    float m = 0.f;
    for (int p = tid; p < (1 << LOGM); p += NT) {
        const float2 z = s[sidx<1>(p, 0)];
        m = fmaxf(m, fmaxf(fabsf(z.x), fabsf(z.y)));
    }
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((tid & 31) == 0) red[tid >> 5] = m;
    __syncthreads();
    m = 0.f;
    for (int i = 0; i < NT / 32; ++i) m = fmaxf(m, red[i]);
    const float sc = m > 0.f ? m : 1.f;
    const float inv = 1.f / sc;
    __half2* out = Kh + (int64_t)h * (1 << LOGM);
    for (int p = tid; p < (1 << LOGM); p += NT) {
        const int f = (int)perm_to_freq(p, LOGM);
        const int c1 = f & 31, c2 = (f >> 5) & 31, c3 = f >> 10;
        const float2 z = s[sidx<1>(p, 0)];
        out[((c2 * 2 + (c3 >> 2)) * 32 + c1) * 4 + (c3 & 3)] = __floats2half2_rn(z.x * inv, z.y * inv);
    }
    if (tid == 0) scales[h] = sc;
}

// The same 8192-point spectrum in the planar tensor-core format
// (tc_planar.cu): per channel 8192 complex fp16 values K[f] / s_h, f = c1 +
// 32 c2 + 1024 c3, the real part in half (c3 & 1) of 32-bit word
// ((c2*2 + c3/4)*32 + c1)*4 + 2*((c3 & 3)/2) and the imaginary part in the
// same half of the next word; s_h = max |Re|, |Im| over the channel, stored
// after the H rows.
template <typename T>
__global__ void __launch_bounds__(fused_threads<13>())
simt_precompute_tc_pp_kernel(const T* __restrict__ k, int64_t L, __half* __restrict__ Kh,
                             float* __restrict__ scales, const float2* __restrict__ tw) {
    constexpr int LOGM = 13;
    constexpr int NT = fused_threads<LOGM>();
    constexpr int K = Sched<LOGM>::K;
    extern __shared__ float2 s[];
    __shared__ float red[NT / 32];
    const int tid = threadIdx.x;
    const int h = blockIdx.x;
    PairRows<T> io;
    io.u0 = k + (int64_t)h * L;
    io.nvalid = (int)L;
    first_stage_global<LOGM, NT, T>(s, tw, io, tid);
    __syncthreads();
    fwd_stages<LOGM, 1, K, 1, NT>(s, tw, 0, tid);
    float m = 0.f;
    for (int p = tid; p < (1 << LOGM); p += NT) {
        const float2 z = s[sidx<1>(p, 0)];
        m = fmaxf(m, fmaxf(fabsf(z.x), fabsf(z.y)));
    }
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((tid & 31) == 0) red[tid >> 5] = m;
    __syncthreads();
    m = 0.f;
    for (int i = 0; i < NT / 32; ++i) m = fmaxf(m, red[i]);
    const float sc = m > 0.f ? m : 1.f;
    const float inv = 1.f / sc;
    __half* out = Kh + (int64_t)h * (2 << LOGM);
    for (int p = tid; p < (1 << LOGM); p += NT) {
        const int f = (int)perm_to_freq(p, LOGM);
        const int c1 = f & 31, c2 = (f >> 5) & 31, c3 = f >> 10;
        const int word = ((c2 * 2 + (c3 >> 2)) * 32 + c1) * 4 + 2 * ((c3 & 3) >> 1);
        const float2 z = s[sidx<1>(p, 0)];
        out[2 * word + (c3 & 1)] = __float2half_rn(z.x * inv);
        out[2 * word + 2 + (c3 & 1)] = __float2half_rn(z.y * inv);
    }
    if (tid == 0) scales[h] = sc;
}

// Filter taps of the two-block precompute as one complex row: real part
// k[t] (t < min(L, 4096)), imaginary part k[4096 + t] (4096 + t < L).
template <typename T>
struct TwoBlockTaps {
    const T* k;
    int n0, n1;
    __device__ __forceinline__ float2 load(int t) const {
        return make_float2(t < n0 ? to_f32(k[t]) : 0.f, t < n1 ? to_f32(k[4096 + t]) : 0.f);
    }
};

// Two-block filter rows of the planar tensor-core kernel (sequences of
// 8192): with k0, k1 the taps [0, 4096) and [4096, 8192) of k,
// G_0 = FFT_8192([k0; 0]) and G_1 = FFT_8192([k1; k0]) = H_1 + (-1)^f H_0
// (H_b = FFT_8192([kb; 0]); the shift by 4096 is the sign (-1)^f).  One
// transform of k0 + i k1 gives both: H_0[f] = (Z[f] + conj Z[-f]) / 2,
// H_1[f] = (Z[f] - conj Z[-f]) / 2i.  Both rows in the PP layout of
// simt_precompute_tc_pp_kernel, over one scale s_h = max |Re|, |Im| of G_0
// and G_1, stored after the H row pairs.
template <typename T>
__global__ void __launch_bounds__(fused_threads<13>())
simt_precompute_tc_pp2_kernel(const T* __restrict__ k, int64_t L, __half* __restrict__ Kh,
                              float* __restrict__ scales, const float2* __restrict__ tw) {
    constexpr int LOGM = 13;
    constexpr int M = 1 << LOGM;
    constexpr int NT = fused_threads<LOGM>();
    constexpr int K = Sched<LOGM>::K;
    extern __shared__ float2 s[];
    __shared__ float red[NT / 32];
    const int tid = threadIdx.x;
    const int h = blockIdx.x;
    TwoBlockTaps<T> io;
    io.k = k + (int64_t)h * L;
    io.n0 = (int)(L < 4096 ? L : 4096);
    io.n1 = (int)(L > 4096 ? L - 4096 : 0);
    first_stage_global<LOGM, NT, T>(s, tw, io, tid);
    __syncthreads();
    fwd_stages<LOGM, 1, K, 1, NT>(s, tw, 0, tid);
    auto rows = [&](int p, int& f, float2& g0, float2& g1) {
        f = (int)perm_to_freq(p, LOGM);
        const int pm = (int)freq_to_perm((M - f) & (M - 1), LOGM);
        const float2 z = s[sidx<1>(p, 0)], zm = s[sidx<1>(pm, 0)];
        g0 = make_float2(0.5f * (z.x + zm.x), 0.5f * (z.y - zm.y));
        const float2 h1 = make_float2(0.5f * (z.y + zm.y), -0.5f * (z.x - zm.x));
        const float sg = (f & 1) ? -1.f : 1.f;
        g1 = make_float2(h1.x + sg * g0.x, h1.y + sg * g0.y);
    };
    float m = 0.f;
    for (int p = tid; p < M; p += NT) {
        int f;
        float2 g0, g1;
        rows(p, f, g0, g1);
        m = fmaxf(m, fmaxf(fmaxf(fabsf(g0.x), fabsf(g0.y)), fmaxf(fabsf(g1.x), fabsf(g1.y))));
    }
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((tid & 31) == 0) red[tid >> 5] = m;
    __syncthreads();
    m = 0.f;
    for (int i = 0; i < NT / 32; ++i) m = fmaxf(m, red[i]);
    const float sc = m > 0.f ? m : 1.f;
    const float inv = 1.f / sc;
    __half* out0 = Kh + (int64_t)h * (4 * M);
    __half* out1 = out0 + 2 * M;
    for (int p = tid; p < M; p += NT) {
        int f;
        float2 g0, g1;
        rows(p, f, g0, g1);
        const int c1 = f & 31, c2 = (f >> 5) & 31, c3 = f >> 10;
        const int word = ((c2 * 2 + (c3 >> 2)) * 32 + c1) * 4 + 2 * ((c3 & 3) >> 1);
        out0[2 * word + (c3 & 1)] = __float2half_rn(g0.x * inv);
        out0[2 * word + 2 + (c3 & 1)] = __float2half_rn(g0.y * inv);
        out1[2 * word + (c3 & 1)] = __float2half_rn(g1.x * inv);
        out1[2 * word + 2 + (c3 & 1)] = __float2half_rn(g1.y * inv);
    }
    if (tid == 0) scales[h] = sc;
}

// The 16384-point spectrum in the split tensor-core format: per channel two
// rows of 8192 complex fp16, row e holding K[2f + e] / s_h at position
// ((c2*2 + c3/4)*32 + c1)*4 + c3%4 of f = c1 + 32 c2 + 1024 c3, with
// s_h = max |Re|, |Im| over the channel stored after the 2H rows.
template <typename T>
__global__ void __launch_bounds__(fused_threads<14>())
simt_precompute_tc_split_kernel(const T* __restrict__ k, int64_t L, __half2* __restrict__ Kh,
                                float* __restrict__ scales, const float2* __restrict__ tw) {
    constexpr int LOGM = 14;
    constexpr int NT = fused_threads<LOGM>();
    constexpr int K = Sched<LOGM>::K;
    extern __shared__ float2 s[];
    __shared__ float red[NT / 32];
    const int tid = threadIdx.x;
    const int h = blockIdx.x;
    PairRows<T> io;
    io.u0 = k + (int64_t)h * L;
    io.nvalid = (int)L;
    first_stage_global<LOGM, NT, T>(s, tw, io, tid);
    __syncthreads();
    fwd_stages<LOGM, 1, K, 1, NT>(s, tw, 0, tid);
    float m = 0.f;
    for (int p = tid; p < (1 << LOGM); p += NT) {
        const float2 z = s[sidx<1>(p, 0)];
        m = fmaxf(m, fmaxf(fabsf(z.x), fabsf(z.y)));
    }
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((tid & 31) == 0) red[tid >> 5] = m;
    __syncthreads();
    m = 0.f;
    for (int i = 0; i < NT / 32; ++i) m = fmaxf(m, red[i]);
    const float sc = m > 0.f ? m : 1.f;
    const float inv = 1.f / sc;
    for (int p = tid; p < (1 << LOGM); p += NT) {
        const int f = (int)perm_to_freq(p, LOGM);
        const int e = f & 1, f8 = f >> 1;
        const int c1 = f8 & 31, c2 = (f8 >> 5) & 31, c3 = f8 >> 10;
        const float2 z = s[sidx<1>(p, 0)];
        Kh[((int64_t)(2 * h + e) << 13) + ((c2 * 2 + (c3 >> 2)) * 32 + c1) * 4 + (c3 & 3)] =
            __floats2half2_rn(z.x * inv, z.y * inv);
    }
    if (tid == 0) scales[h] = sc;
}

// Filter gradient of the backward pass: dk[h, s] = sum_b sum_t g_b[t] x_b[t-s]
// for s < L, with g = dy * v and x = u * w (gates absent: ones).  One CTA per
// (channel, chunk of batch rows): each row's g and x ride in the real and
// imaginary parts of one complex sequence z = g + i x, zero-padded to M; its
// spectrum Z gives G = (Z[f] + conj Z[M-f]) / 2 and X = (Z[f] - conj Z[M-f]) / 2i
// (g and x are real), and the CTA accumulates G conj(X) (the spectrum of the
// correlation, exact for s < N since the padding absorbs the wrap).  One
// inverse transform of the sum then gives the CTA's part of dk, added to the
// (zeroed) output with atomics.  The accumulator sits in shared memory beside
// the transform buffer and holds the bins [0, M/2] only (the sum is the
// spectrum of a real sequence, so the other half is their conjugate mirror),
// which keeps M = 16384 (N = 8192) within one CTA's shared memory.
template <int LOGM, typename T>
__global__ void __launch_bounds__(fused_threads<LOGM>())
simt_filter_grad_kernel(const T* __restrict__ u, const T* __restrict__ w, const T* __restrict__ v,
                        const T* __restrict__ dy, int64_t B, int64_t H, int64_t L, int64_t rows,
                        float* __restrict__ dk, const float2* __restrict__ tw) {
    constexpr int NT = fused_threads<LOGM>();
    constexpr int K = Sched<LOGM>::K;
    constexpr int M = 1 << LOGM;
    constexpr int64_t N = M / 2;
    extern __shared__ float2 s[];
    // the summed spectrum is Hermitian (dk is real): bins [0, M/2] only
    float2* acc = s + smem_elems<1>(M);
    const int tid = threadIdx.x;
    const int64_t h = blockIdx.x;
    const int64_t b0 = (int64_t)blockIdx.y * rows, b1 = b0 + rows < B ? b0 + rows : B;
    for (int f = tid; f <= M / 2; f += NT) acc[f] = make_float2(0.f, 0.f);
    for (int64_t b = b0; b < b1; ++b) {
        const int64_t o = (b * H + h) * N;
        PairRows<T> io;
        io.u0 = dy + o;
        io.w0 = v ? v + o : nullptr;
        io.u1 = u + o;
        io.w1 = w ? w + o : nullptr;
        io.nvalid = (int)N;
        __syncthreads();                       // the previous row's spectrum has been read
        first_stage_global<LOGM, NT, T>(s, tw, io, tid);
        __syncthreads();
        fwd_stages<LOGM, 1, K, 1, NT>(s, tw, 0, tid);
        for (int f = tid; f <= M / 2; f += NT) {
            const int p = (int)freq_to_perm(f, LOGM);
            const int pm = (int)freq_to_perm((M - f) & (M - 1), LOGM);
            const float2 zf = s[sidx<1>(p, 0)], zm = s[sidx<1>(pm, 0)];
            // G = (zf + conj zm) / 2, X = (zf - conj zm) / 2i
            const float2 G = make_float2(0.5f * (zf.x + zm.x), 0.5f * (zf.y - zm.y));
            const float2 X = make_float2(0.5f * (zf.y + zm.y), 0.5f * (zm.x - zf.x));
            acc[f] = cadd(acc[f], cmulc(G, X));
        }
    }
    __syncthreads();
    for (int p = tid; p < M; p += NT) {
        const int f = (int)perm_to_freq(p, LOGM);
        const float2 z = f <= M / 2 ? acc[f] : acc[M - f];
        s[sidx<1>(p, 0)] = f <= M / 2 ? z : make_float2(z.x, -z.y);
    }
    __syncthreads();
    inv_stages<LOGM, 0, K, 1, NT>(s, tw, 0, tid);
    const float inv = 1.0f / (float)M;
    for (int t = tid; t < L; t += NT) atomicAdd(&dk[h * L + t], s[sidx<1>(t, 0)].x * inv);
}

template <int LOGM, typename T>
cudaError_t launch_fused(const Plan& p, const ForwardArgs& a, cudaStream_t st) {
    constexpr int NT = fused_threads<LOGM>();
    const size_t smem = sizeof(float2) * smem_elems<1>(1 << LOGM);
    auto kern = simt_fused_kernel<LOGM, T>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t pairs = p.H * ((a.B + 1) / 2);
    kern<<<(unsigned)pairs, NT, smem, st>>>(a, p.H, p.tw);
    return cudaGetLastError();
}

template <int LOGM, typename T>
cudaError_t launch_fused_pre(const Plan& p, const void* k, void* Kf, cudaStream_t st) {
    constexpr int NT = fused_threads<LOGM>();
    const size_t smem = sizeof(float2) * smem_elems<1>(1 << LOGM);
    auto kern = simt_fused_precompute_kernel<LOGM, T>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)p.H, NT, smem, st>>>((const T*)k, p.L, (float2*)Kf, p.tw);
    return cudaGetLastError();
}

// ------------------------------------------------------ staged kernels ---

constexpr int kColThreads = 256;
// columns per CTA in the shared-memory column passes: 2048 / R, within
// [16, 256] (256 divides every staged C >= 256), and 8 for R >= 512.  Long
// columns need narrow tiles so that several CTAs stay resident: measured on
// B200, R = 256 (N = 2^20) ran the call 5% faster with 16 columns per CTA
// (32 KB of shared memory) than with 32 and 1.5x faster than with 64;
// R = 1024 (N = 2^22) 1.34x faster with 8 (64 KB) than with 16 (128 KB, one
// CTA per SM), and 1.30x faster than with 4 (16-byte row segments).
template <int LOGR>
constexpr int col_tile() {
    return LOGR >= 9 ? 8 : ((2048 >> LOGR) > 256 ? 256 : ((2048 >> LOGR) < 16 ? 16 : (2048 >> LOGR)));
}

template <int LOGC>
constexpr int row_threads() { return (1 << LOGC) / 32 < 128 ? 128 : ((1 << LOGC) / 32 > 512 ? 512 : (1 << LOGC) / 32); }

struct StagedArgs {
    ForwardArgs fa;
    int64_t H, N, M;
    int64_t pair0;          // first pair of this chunk
    int64_t npairs;         // pairs in this chunk
    int logC;
    float2* work;           // [npairs][R][C]
    const float2* tw;       // exp(-2 pi i e / C)
    const float2* twLo;
    const float2* twHi;
    int twSplit;
    // precompute mode: input k [H, L] instead of u/w; pair == channel
    const void* k;
    int64_t L;
    int64_t kf_pair0;       // precompute mode: channel of the first K_f row written
    // half-precision workspace (the tensor-core row pass): the forward column
    // pass stores its values times rin as fp16; the row pass leaves its
    // results unscaled; the inverse column pass multiplies row c of channel h
    // by kscale[h * R + c] * rout
    const float* kscale;
    float rin, rout;
    // the plan's status word; the inverse column passes of the half-precision
    // workspace record FFTCONV_ERR_RANGE there when the convolution came out
    // non-finite (an fp16 intermediate overflowed)
    int* status;
    // overlap-save windows (column kernels with WIN): unit u of the chunk is
    // window u % nwin of pair u / nwin; the window's position t is sequence
    // position (w - 1) winHop + t, inputs before 0 read as zero, and only its
    // second half t >= winHop is output
    int64_t nwin, winHop;
};

// pair, window and the sequence position of window position 0 of unit u
struct UnitPos {
    int64_t pair, win, base;
};
template <bool WIN>
__device__ __forceinline__ UnitPos unit_pos(const StagedArgs& A, int64_t u) {
    UnitPos p{u, 0, 0};
    if constexpr (WIN) {
        p.pair = u / A.nwin;
        p.win = u - p.pair * A.nwin;
        p.base = (p.win - 1) * A.winHop;
    }
    return p;
}

template <typename T>
__device__ __forceinline__ PairRows<T> staged_rows(const StagedArgs& A, int64_t pair, int* h) {
    if (A.k) {
        PairRows<T> r;
        r.u0 = (const T*)A.k + pair * A.L;
        r.nvalid = (int)A.L;
        *h = (int)pair;
        return r;
    }
    return pair_rows<T>(A.fa, A.H, A.N, pair, h);
}

// Column pass: length-R DFT over j of x[j*C + r] (upper half zero), twiddle
// exp(-2 pi i c r / M), stored at work[pair][c][r] in natural c order.
// Resident CTAs the shared-memory column passes ask the compiler for: at
// R = 256 five (48 registers, no spills) instead of the four that 61
// registers allow; measured on B200 (N = 2^20, B = 1, H = 128) 1% faster per
// call in the benchmark, 6% in an A/B run without it, while six or more
// spill and run slower.
template <int LOGR>
constexpr int col_min_blocks() { return LOGR == 8 ? 5 : 1; }

template <int LOGR, typename T, bool WS16, bool WIN>
__global__ void __launch_bounds__(kColThreads, col_min_blocks<LOGR>())
staged_col_fwd_kernel(StagedArgs A) {
    constexpr int R = 1 << LOGR;
    constexpr int TC = col_tile<LOGR>();
    extern __shared__ float2 s[];
    const int tid = threadIdx.x;
    const int64_t C = (int64_t)1 << A.logC;
    const int64_t pl = blockIdx.y;
    const int64_t col0 = (int64_t)blockIdx.x * TC;
    const UnitPos U = unit_pos<WIN>(A, A.pair0 + pl);
    int h;
    const PairRows<T> io = staged_rows<T>(A, U.pair, &h);
    // the nonzero rows (j < R/2; a window: all R, the first window's first
    // half zero), four consecutive columns per thread
    constexpr int JN = WIN ? R : R / 2;
    for (int idx = tid; idx < JN * (TC / 4); idx += kColThreads) {
        const int j = idx / (TC / 4), c4 = 4 * (idx % (TC / 4));
        float2 x[4];
        if (WIN && U.win == 0 && j < R / 2) {
#pragma unroll
            for (int e = 0; e < 4; ++e) x[e] = make_float2(0.f, 0.f);
        } else {
            io.load4((int)(U.base + j * C + col0 + c4), x);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) s[sidx<TC>(j, c4 + e)] = x[e];
    }
    __syncthreads();
    if constexpr (WIN) {
        fwd_stages<LOGR, 0, Sched<LOGR>::K, TC, kColThreads>(s, A.tw, A.logC - LOGR, tid);
    } else {
        // the upper half (j >= R/2) is zero: the first stage reads only the
        // lower half, so that half is never stored
        fwd_stage0_half_input<LOGR, TC, kColThreads>(s, A.tw, A.logC - LOGR, tid);
        __syncthreads();
        fwd_stages<LOGR, 1, Sched<LOGR>::K, TC, kColThreads>(s, A.tw, A.logC - LOGR, tid);
    }
    // twiddle w_M^(c r) and store: each thread keeps one column r and walks
    // CPG consecutive c (a warp writes 32 consecutive r of one c).  The
    // twiddle comes from the table at every eighth c and as a product with
    // w_M^r in between (at most seven fp32 products, a few ulps): a table
    // read per element at stride c would touch up to 32 cache lines per warp.
    constexpr int NG = kColThreads / TC, CPG = R / NG;
    static_assert(CPG % 8 == 0, "column groups walk whole runs of 8");
    const int col = tid % TC, g = tid / TC;
    const int64_t r = col0 + col;
    const float2 step = tw_M(A.twLo, A.twHi, A.twSplit, r);
    for (int i0 = 0; i0 < CPG; i0 += 8) {
        const int64_t cb = (int64_t)g * CPG + i0;
        float2 w = tw_M(A.twLo, A.twHi, A.twSplit, cb * r);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (i) w = cmul(w, step);
            const int64_t c = cb + i;
            const float2 z = cmul(s[sidx<TC>((int)freq_to_perm(c, LOGR), col)], w);
            if constexpr (WS16)
                reinterpret_cast<__half2*>(A.work)[pl * (R * C) + c * C + r] = __floats2half2_rn(z.x * A.rin, z.y * A.rin);
            else
                A.work[pl * (R * C) + c * C + r] = z;
        }
    }
}

// Row pass.  MODE 0: forward DFT over r, product with K_f row, inverse, back
// into the workspace.  MODE 1 (filter precompute): forward only, scaled by
// 1/M, into K_f[h][c][position].
template <int LOGC, int MODE>
__global__ void __launch_bounds__(row_threads<LOGC>())
staged_row_kernel(StagedArgs A) {
    constexpr int NT = row_threads<LOGC>();
    constexpr int C = 1 << LOGC;
    constexpr int K = Sched<LOGC>::K;
    extern __shared__ float2 s[];
    const int tid = threadIdx.x;
    const int64_t c = blockIdx.x;
    const int64_t R = A.M >> LOGC;
    const int64_t pl = blockIdx.y;
    float2* row = A.work + (pl * R + c) * C;
    for (int i = tid; i < C; i += NT) s[sidx<1>(i, 0)] = row[i];
    __syncthreads();
    if constexpr (MODE == 0) {
        const int64_t h = (A.pair0 + pl) / ((A.fa.B + 1) / 2);   // channel of this pair
        const float2* Krow = (const float2*)A.fa.Kf + ((int64_t)h * R + c) * C;
        const uint8_t* mrow = A.fa.mask ? A.fa.mask + (A.fa.mask_h == 1 ? 0 : h) * (A.N / kMaskBlock) : nullptr;
        fwd_stages<LOGC, 0, K - 1, 1, NT>(s, A.tw, 0, tid);
        middle_stage<LOGC, NT>(s, Krow, mrow, A.N,
                               [c, R](int p) { return c + R * perm_to_freq(p, LOGC); }, tid);
        __syncthreads();
        inv_stages<LOGC, 0, K - 1, 1, NT>(s, A.tw, 0, tid);
        for (int i = tid; i < C; i += NT) row[i] = s[sidx<1>(i, 0)];
    } else {
        fwd_stages<LOGC, 0, K, 1, NT>(s, A.tw, 0, tid);
        const float inv = 1.0f / (float)A.M;
        const int64_t h = A.pair0 + pl - A.kf_pair0;
        float2* out = (float2*)A.fa.y + (h * R + c) * C;   // fa.y carries K_f here
        for (int i = tid; i < C; i += NT) out[i] = cscale(s[sidx<1>(i, 0)], inv);
    }
}

// Inverse column pass: conjugate twiddle, inverse length-R DFT over c, and
// y = v * z for t = j*C + r < N.
template <int LOGR, typename T, bool WS16, bool WIN>
__global__ void __launch_bounds__(kColThreads, col_min_blocks<LOGR>())
staged_col_inv_kernel(StagedArgs A) {
    constexpr int R = 1 << LOGR;
    constexpr int TC = col_tile<LOGR>();
    extern __shared__ float2 s[];
    const int tid = threadIdx.x;
    const int64_t C = (int64_t)1 << A.logC;
    const int64_t pl = blockIdx.y;
    const int64_t col0 = (int64_t)blockIdx.x * TC;
    const UnitPos U = unit_pos<WIN>(A, A.pair0 + pl);
    int h;
    const PairRows<T> io = staged_rows<T>(A, U.pair, &h);
    {
        // the forward pass's walk in reverse roles: load, conjugate twiddle
        constexpr int NG = kColThreads / TC, CPG = R / NG;
        static_assert(CPG % 8 == 0, "column groups walk whole runs of 8");
        const int col = tid % TC, g = tid / TC;
        const int64_t r = col0 + col;
        const float2 step = tw_M(A.twLo, A.twHi, A.twSplit, r);
        for (int i0 = 0; i0 < CPG; i0 += 8) {
            const int64_t cb = (int64_t)g * CPG + i0;
            float2 w = tw_M(A.twLo, A.twHi, A.twSplit, cb * r);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (i) w = cmul(w, step);
                const int64_t c = cb + i;
                float2 z;
                if constexpr (WS16) {
                    z = __half22float2(reinterpret_cast<const __half2*>(A.work)[pl * (R * C) + c * C + r]);
                    z = cscale(z, __ldg(&A.kscale[(int64_t)h * R + c]) * A.rout);
                } else {
                    z = A.work[pl * (R * C) + c * C + r];
                }
                s[sidx<TC>((int)freq_to_perm(c, LOGR), col)] = cmulc(z, w);
            }
        }
    }
    __syncthreads();
    inv_stages<LOGR, 0, Sched<LOGR>::K, TC, kColThreads>(s, A.tw, A.logC - LOGR, tid);
    // outputs: the first half (t < N), or a window's second half
    constexpr int J0 = WIN ? R / 2 : 0;
    float nf = 0.f;
    for (int idx = tid; idx < (R / 2) * (TC / 4); idx += kColThreads) {
        const int j = J0 + idx / (TC / 4), c4 = 4 * (idx % (TC / 4));
        float2 z[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            z[e] = s[sidx<TC>(j, c4 + e)];
            if constexpr (WS16) { nonfinite_fold(nf, z[e].x); nonfinite_fold(nf, z[e].y); }
        }
        io.store4((int)(U.base + j * C + col0 + c4), z);
    }
    if constexpr (WS16) nonfinite_report(nf, A.status);
}

// Column passes for short columns (R <= 8) without shared memory: a thread
// takes four consecutive columns r .. r+3 of one pair, holds their R values in
// registers and does the whole length-R DFT there.  Loads and stores are
// 8- and 16-byte vectors, coalesced across the warp (consecutive threads,
// consecutive columns); measured on B200 the shared-memory kernels run these
// short columns at about a third of the memory bandwidth.
constexpr int kRegColThreads = 256;
// four resident CTAs (64 registers, a few spilled values) instead of the three
// that 80 registers allow: more loads in flight; measured on B200 (N = 32768,
// R = 8) 12% faster per call in an A/B run
constexpr int kRegColMinBlocks = 4;

template <int LOGR, typename T, bool WS16, bool WIN>
__global__ void __launch_bounds__(kRegColThreads, kRegColMinBlocks)
staged_col_fwd_reg_kernel(StagedArgs A) {
    constexpr int R = 1 << LOGR;
    const int64_t C = (int64_t)1 << A.logC;
    const int64_t pl = blockIdx.y;
    const int64_t r0 = 4 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x);
    const UnitPos U = unit_pos<WIN>(A, A.pair0 + pl);
    int h;
    const PairRows<T> io = staged_rows<T>(A, U.pair, &h);
    float2 x[4][R];
    // the nonzero rows (j < R/2; a window: all R, the first window's first
    // half zero)
#pragma unroll
    for (int j = 0; j < (WIN ? R : R / 2); ++j) {
        float2 q[4];
        if (WIN && U.win == 0 && j < R / 2) {
#pragma unroll
            for (int e = 0; e < 4; ++e) q[e] = make_float2(0.f, 0.f);
        } else {
            io.load4((int)(U.base + j * C + r0), q);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) x[e][j] = q[e];
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        if constexpr (WIN) Dft<R, -1>::run(x[e]);
        else Dft<R, -1>::run_half_input(x[e]);
    }
    // w_M^(c r) as powers of w_M^r (at most seven products)
    float2 step[4], w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        step[e] = tw_M(A.twLo, A.twHi, A.twSplit, r0 + e);
        w[e] = make_float2(1.f, 0.f);
    }
#pragma unroll
    for (int c = 0; c < R; ++c) {
        float2 z[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if (c) w[e] = cmul(w[e], step[e]);
            z[e] = cmul(x[e][c], w[e]);
        }
        const int64_t o = pl * (R * C) + c * C + r0;
        if constexpr (WS16) {
            __half2 hz[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) hz[e] = __floats2half2_rn(z[e].x * A.rin, z[e].y * A.rin);
            *reinterpret_cast<uint4*>(reinterpret_cast<__half2*>(A.work) + o) = *reinterpret_cast<const uint4*>(hz);
        } else {
            reinterpret_cast<float4*>(A.work + o)[0] = make_float4(z[0].x, z[0].y, z[1].x, z[1].y);
            reinterpret_cast<float4*>(A.work + o)[1] = make_float4(z[2].x, z[2].y, z[3].x, z[3].y);
        }
    }
}

template <int LOGR, typename T, bool WS16, bool WIN>
__global__ void __launch_bounds__(kRegColThreads, kRegColMinBlocks)
staged_col_inv_reg_kernel(StagedArgs A) {
    constexpr int R = 1 << LOGR;
    const int64_t C = (int64_t)1 << A.logC;
    const int64_t pl = blockIdx.y;
    const int64_t r0 = 4 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x);
    const UnitPos U = unit_pos<WIN>(A, A.pair0 + pl);
    int h;
    const PairRows<T> io = staged_rows<T>(A, U.pair, &h);
    float2 x[4][R];
    float2 step[4], w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        step[e] = tw_M(A.twLo, A.twHi, A.twSplit, r0 + e);
        w[e] = make_float2(1.f, 0.f);
    }
#pragma unroll
    for (int c = 0; c < R; ++c) {
        const int64_t o = pl * (R * C) + c * C + r0;
        float2 z[4];
        if constexpr (WS16) {
            const uint4 q = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const __half2*>(A.work) + o));
            const __half2* hz = reinterpret_cast<const __half2*>(&q);
            const float sc = __ldg(&A.kscale[(int64_t)h * R + c]) * A.rout;
#pragma unroll
            for (int e = 0; e < 4; ++e) z[e] = cscale(__half22float2(hz[e]), sc);
        } else {
            const float4 a = reinterpret_cast<const float4*>(A.work + o)[0];
            const float4 b = reinterpret_cast<const float4*>(A.work + o)[1];
            z[0] = make_float2(a.x, a.y); z[1] = make_float2(a.z, a.w);
            z[2] = make_float2(b.x, b.y); z[3] = make_float2(b.z, b.w);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if (c) w[e] = cmul(w[e], step[e]);
            x[e][c] = cmulc(z[e], w[e]);
        }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) Dft<R, +1>::run(x[e]);
    // outputs: the first half (t < N), or a window's second half
    float nf = 0.f;
#pragma unroll
    for (int jj = 0; jj < R / 2; ++jj) {
        const int j = (WIN ? R / 2 : 0) + jj;
        const float2 q[4] = {x[0][j], x[1][j], x[2][j], x[3][j]};
        if constexpr (WS16) {
#pragma unroll
            for (int e = 0; e < 4; ++e) { nonfinite_fold(nf, q[e].x); nonfinite_fold(nf, q[e].y); }
        }
        io.store4((int)(U.base + j * C + r0), q);
    }
    if constexpr (WS16) nonfinite_report(nf, A.status);
}

template <int LOGR, typename T, bool WS16, bool WIN>
cudaError_t launch_cols(const StagedArgs& A, int64_t C, bool inverse, cudaStream_t st) {
    if constexpr (LOGR <= 3) {
        // one thread per four columns: C / 4 threads per pair (C >= 256 a
        // power of two, so blocks of min(C / 4, 256) threads tile it exactly)
        const unsigned threads = C / 4 < kRegColThreads ? (unsigned)(C / 4) : kRegColThreads;
        dim3 grid((unsigned)(C / 4 / threads), (unsigned)A.npairs);
        if (!inverse) staged_col_fwd_reg_kernel<LOGR, T, WS16, WIN><<<grid, threads, 0, st>>>(A);
        else staged_col_inv_reg_kernel<LOGR, T, WS16, WIN><<<grid, threads, 0, st>>>(A);
        return cudaGetLastError();
    } else {
        const size_t smem = sizeof(float2) * (size_t)(1 << LOGR) * col_tile<LOGR>();
        dim3 grid((unsigned)(C / col_tile<LOGR>()), (unsigned)A.npairs);
        if (!inverse) {
            auto kern = staged_col_fwd_kernel<LOGR, T, WS16, WIN>;
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
            kern<<<grid, kColThreads, smem, st>>>(A);
        } else {
            auto kern = staged_col_inv_kernel<LOGR, T, WS16, WIN>;
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
            kern<<<grid, kColThreads, smem, st>>>(A);
        }
        return cudaGetLastError();
    }
}

template <int LOGC, int MODE>
cudaError_t launch_rows(const StagedArgs& A, int64_t R, cudaStream_t st) {
    constexpr int NT = row_threads<LOGC>();
    const size_t smem = sizeof(float2) * smem_elems<1>(1 << LOGC);
    auto kern = staged_row_kernel<LOGC, MODE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)R, (unsigned)A.npairs);
    kern<<<grid, NT, smem, st>>>(A);
    return cudaGetLastError();
}

// Runtime -> compile-time dispatch helpers.
template <typename T, bool WS16 = false, bool WIN = false>
cudaError_t cols_dispatch(int logR, const StagedArgs& A, int64_t C, bool inverse, cudaStream_t st) {
    switch (logR) {
        case 1: return launch_cols<1, T, WS16, WIN>(A, C, inverse, st);
        case 2: return launch_cols<2, T, WS16, WIN>(A, C, inverse, st);
        case 3: return launch_cols<3, T, WS16, WIN>(A, C, inverse, st);
        case 4: return launch_cols<4, T, WS16, WIN>(A, C, inverse, st);
        case 5: return launch_cols<5, T, WS16, WIN>(A, C, inverse, st);
        case 6: return launch_cols<6, T, WS16, WIN>(A, C, inverse, st);
        case 7: return launch_cols<7, T, WS16, WIN>(A, C, inverse, st);
        case 8: return launch_cols<8, T, WS16, WIN>(A, C, inverse, st);
        case 9: return launch_cols<9, T, WS16, WIN>(A, C, inverse, st);
        case 10: return launch_cols<10, T, WS16, WIN>(A, C, inverse, st);   // rows of 8192 at N = 2^22
        default: return cudaErrorInvalidValue;
    }
}

template <int MODE>
cudaError_t rows_dispatch(int logC, const StagedArgs& A, int64_t R, cudaStream_t st) {
    switch (logC) {
        case 8: return launch_rows<8, MODE>(A, R, st);
        case 9: return launch_rows<9, MODE>(A, R, st);
        case 10: return launch_rows<10, MODE>(A, R, st);
        case 11: return launch_rows<11, MODE>(A, R, st);
        case 12: return launch_rows<12, MODE>(A, R, st);
        case 13: return launch_rows<13, MODE>(A, R, st);
        case 14: return launch_rows<14, MODE>(A, R, st);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T>
cudaError_t staged_forward_t(const Plan& p, const ForwardArgs& fa, const void* k, cudaStream_t st) {
    StagedArgs A{};
    A.fa = fa;
    A.H = p.H; A.N = p.N; A.M = p.M;
    A.logC = p.logC;
    A.work = p.work;
    A.tw = p.tw; A.twLo = p.twLo; A.twHi = p.twHi; A.twSplit = p.twSplit;
    A.k = k; A.L = p.L;
    const int64_t C = (int64_t)1 << p.logC, R = (int64_t)1 << p.logR;
    const int64_t total = k ? p.H : p.H * ((fa.B + 1) / 2);
    for (int64_t first = 0; first < total; first += p.chunkPairs) {
        A.pair0 = first;
        A.npairs = total - first < p.chunkPairs ? total - first : p.chunkPairs;
        cudaError_t e = cols_dispatch<T>(p.logR, A, C, false, st);
        if (e != cudaSuccess) return e;
        e = k ? rows_dispatch<1>(p.logC, A, R, st) : rows_dispatch<0>(p.logC, A, R, st);
        if (e != cudaSuccess) return e;
        if (!k) {
            e = cols_dispatch<T>(p.logR, A, C, true, st);
            if (e != cudaSuccess) return e;
        }
    }
    return cudaSuccess;
}

// Staged path with the tensor-core row pass: per chunk of pairs the forward
// column pass, the tensor-core kernel over the chunk's rows (forward 8192-point
// transform, filter product, inverse, in place) and the inverse column pass.
template <typename T>
cudaError_t tc_staged_forward_t(const Plan& p, const ForwardArgs& fa, cudaStream_t st) {
    StagedArgs A{};
    A.fa = fa;
    A.H = p.H; A.N = p.N; A.M = p.M;
    A.logC = p.logC;
    A.work = p.work;
    A.tw = p.tw; A.twLo = p.twLo; A.twHi = p.twHi; A.twSplit = p.twSplit;
    const int64_t C = (int64_t)1 << p.logC;
    // fp16 workspace scaled by a power of two near 1/sqrt(R) (exact): the
    // column pass sums R/2 inputs per value, the scale keeps the operands in
    // the inputs' range; the unitary 8192-point pair of the row pass leaves
    // 1/8192, undone with the scale by rout
    A.kscale = (const float*)((const uint8_t*)fa.Kf + tc_staged_spectrum_bytes(p));
    A.status = p.status;
    A.rin = std::ldexp(1.0f, -(p.logR / 2));
    A.rout = (float)C * std::ldexp(1.0f, p.logR / 2);
    // workspace units: pairs, or (pair, window) with overlap-save windows
    const bool win = p.nwin > 1;
    A.nwin = p.nwin;
    A.winHop = p.winHop;
    const int64_t total = p.H * ((fa.B + 1) / 2) * p.nwin;
    for (int64_t first = 0; first < total; first += p.chunkPairs) {
        A.pair0 = first;
        A.npairs = total - first < p.chunkPairs ? total - first : p.chunkPairs;
        cudaError_t e = win ? cols_dispatch<T, true, true>(p.logR, A, C, false, st)
                            : cols_dispatch<T, true, false>(p.logR, A, C, false, st);
        if (e == cudaSuccess) e = tc_rows_forward(p, fa, first, A.npairs, st);
        if (e == cudaSuccess)
            e = win ? cols_dispatch<T, true, true>(p.logR, A, C, true, st)
                    : cols_dispatch<T, true, false>(p.logR, A, C, true, st);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// Its filter precompute: the staged forward transform of k (column pass, then
// the fp32 row pass scaled by 1/M) into the workspace, chunk by chunk, and the
// conversion of each chunk's rows to the tensor-core layout.
template <typename T>
cudaError_t tc_staged_precompute_t(const Plan& p, const void* k, void* Kf, cudaStream_t st) {
    StagedArgs A{};
    A.fa.y = p.work;        // the row pass writes the chunk's spectra in place
    A.H = p.H; A.N = p.N; A.M = p.M;
    A.logC = p.logC;
    A.work = p.work;
    A.tw = p.tw; A.twLo = p.twLo; A.twHi = p.twHi; A.twSplit = p.twSplit;
    A.k = k; A.L = p.L;
    const int64_t C = (int64_t)1 << p.logC, R = (int64_t)1 << p.logR;
    // (fp32 spectra: a chunk holds half as many channels as fp16 pairs)
    int64_t per = (int64_t)(p.workBytes / ((size_t)p.M * sizeof(float2)));
    if (per < 1) return cudaErrorInvalidValue;
    for (int64_t first = 0; first < p.H; first += per) {
        A.pair0 = first;
        A.kf_pair0 = first;
        A.npairs = p.H - first < per ? p.H - first : per;
        cudaError_t e = cols_dispatch<T>(p.logR, A, C, false, st);
        if (e == cudaSuccess) e = rows_dispatch<1>(p.logC, A, R, st);
        if (e == cudaSuccess) e = tc_rows_convert(p, first, A.npairs, Kf, st);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// ---------------------------------------------------- export (test hook) ---

__global__ void export_rfft_kernel(const float2* __restrict__ Kf, float* __restrict__ out, int64_t H,
                                   int64_t N, int logM, int staged, int logR, int logC) {
    const int64_t M = 2 * N;
    const int64_t total = H * (N + 1);
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t h = i / (N + 1), f = i % (N + 1);
        int64_t pos;
        if (!staged) {
            pos = freq_to_perm(f, logM);
        } else {
            const int64_t R = (int64_t)1 << logR;
            const int64_t c = f & (R - 1), e = f >> logR;
            pos = (c << logC) + freq_to_perm(e, logC);
        }
        const float2 z = Kf[h * M + pos];
        out[2 * i] = z.x * (float)M;
        out[2 * i + 1] = z.y * (float)M;
    }
}

}  // namespace

bool simt_fused_supported(int logM) { return logM >= 9 && logM <= 14; }

#define FFTCONV_DISPATCH_T(dtype, ...)                                   \
    switch (dtype) {                                                     \
        case kF32: { using T = float; __VA_ARGS__; }                     \
        case kF16: { using T = __half; __VA_ARGS__; }                    \
        case kBF16: { using T = __nv_bfloat16; __VA_ARGS__; }            \
        default: return cudaErrorInvalidValue;                           \
    }

cudaError_t simt_fused_forward(const Plan& p, const ForwardArgs& a, cudaStream_t st) {
    FFTCONV_DISPATCH_T(p.dtype, switch (p.logM) {
        case 9: return launch_fused<9, T>(p, a, st);
        case 10: return launch_fused<10, T>(p, a, st);
        case 11: return launch_fused<11, T>(p, a, st);
        case 12: return launch_fused<12, T>(p, a, st);
        case 13: return launch_fused<13, T>(p, a, st);
        case 14: return launch_fused<14, T>(p, a, st);
        default: return cudaErrorInvalidValue;
    })
}

cudaError_t simt_precompute_to_tc_split(const Plan& p, const void* k, void* Kf, cudaStream_t st) {
    if (p.L > 8192) return cudaErrorInvalidValue;     // the 16384-point spectrum of k (<= 8192 taps)
    const size_t smem = sizeof(float2) * smem_elems<1>(1 << 14);
    FFTCONV_DISPATCH_T(p.dtype, {
        auto kern = simt_precompute_tc_split_kernel<T>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<(unsigned)p.H, fused_threads<14>(), smem, st>>>(
            (const T*)k, p.L, (__half2*)Kf, (float*)((uint8_t*)Kf + (size_t)p.H * 2 * (8192 * 4)), p.tw);
        return cudaGetLastError();
    })
}

cudaError_t simt_precompute_to_tc_layout(const Plan& p, const void* k, void* Kf, cudaStream_t st) {
    if (p.L > 4096) return cudaErrorInvalidValue;     // the 8192-point spectrum of k (<= 4096 taps)
    const size_t smem = sizeof(float2) * smem_elems<1>(1 << 13);
    FFTCONV_DISPATCH_T(p.dtype, {
        auto kern = simt_precompute_tc8192_kernel<T>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<(unsigned)p.H, fused_threads<13>(), smem, st>>>((const T*)k, p.L, (__half2*)Kf,
                                                               (float*)((uint8_t*)Kf + (size_t)p.H * (8192 * 4)), p.tw);
        return cudaGetLastError();
    })
}

// Four-block filter rows (sequences of 16384): G_0 = H_0 and
// G_d = H_d + (-1)^f H_{d-1} for d = 1, 2, 3, with H_j = FFT_8192([k_j; 0])
// (k_j the taps [4096 j, 4096 j + 4096), zero past L).  Two transforms of
// k_0 + i k_1 and k_2 + i k_3 give the four H_j (as in the two-block
// kernel); the rows are written in the PP layout over one scale per channel
// (max |Re|, |Im| of all four rows), stored after the H row quartets.
template <typename T>
__global__ void __launch_bounds__(fused_threads<13>())
simt_precompute_tc_pp4_kernel(const T* __restrict__ k, int64_t L, __half* __restrict__ Kh,
                              float* __restrict__ scales, const float2* __restrict__ tw) {
    constexpr int LOGM = 13;
    constexpr int M = 1 << LOGM;
    constexpr int NT = fused_threads<LOGM>();
    constexpr int K = Sched<LOGM>::K;
    extern __shared__ float2 s[];
    float2* sa = s;
    float2* sb = s + smem_elems<1>(M);
    __shared__ float red[NT / 32];
    const int tid = threadIdx.x;
    const int h = blockIdx.x;
    auto clampn = [](int64_t n) { return (int)(n < 0 ? 0 : (n > 4096 ? 4096 : n)); };
    TwoBlockTaps<T> io;
    io.k = k + (int64_t)h * L;
    io.n0 = clampn(L);
    io.n1 = clampn(L - 4096);
    first_stage_global<LOGM, NT, T>(sa, tw, io, tid);
    io.k = k + (int64_t)h * L + 8192;
    io.n0 = clampn(L - 8192);
    io.n1 = clampn(L - 12288);
    first_stage_global<LOGM, NT, T>(sb, tw, io, tid);
    __syncthreads();
    fwd_stages<LOGM, 1, K, 1, NT>(sa, tw, 0, tid);
    fwd_stages<LOGM, 1, K, 1, NT>(sb, tw, 0, tid);
    auto rows = [&](int p, int& f, float2 (&g)[4]) {
        f = (int)perm_to_freq(p, LOGM);
        const int pm = (int)freq_to_perm((M - f) & (M - 1), LOGM);
        float2 hh[4];
        const float2 za = sa[sidx<1>(p, 0)], zam = sa[sidx<1>(pm, 0)];
        const float2 zb = sb[sidx<1>(p, 0)], zbm = sb[sidx<1>(pm, 0)];
        hh[0] = make_float2(0.5f * (za.x + zam.x), 0.5f * (za.y - zam.y));
        hh[1] = make_float2(0.5f * (za.y + zam.y), -0.5f * (za.x - zam.x));
        hh[2] = make_float2(0.5f * (zb.x + zbm.x), 0.5f * (zb.y - zbm.y));
        hh[3] = make_float2(0.5f * (zb.y + zbm.y), -0.5f * (zb.x - zbm.x));
        const float sg = (f & 1) ? -1.f : 1.f;
        g[0] = hh[0];
        for (int d = 1; d < 4; ++d) g[d] = make_float2(hh[d].x + sg * hh[d - 1].x, hh[d].y + sg * hh[d - 1].y);
    };
    float m = 0.f;
    for (int p = tid; p < M; p += NT) {
        int f;
        float2 g[4];
        rows(p, f, g);
        for (int d = 0; d < 4; ++d) m = fmaxf(m, fmaxf(fabsf(g[d].x), fabsf(g[d].y)));
    }
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((tid & 31) == 0) red[tid >> 5] = m;
    __syncthreads();
    m = 0.f;
    for (int i = 0; i < NT / 32; ++i) m = fmaxf(m, red[i]);
    const float sc = m > 0.f ? m : 1.f;
    const float inv = 1.f / sc;
    __half* out = Kh + (int64_t)h * (8 * M);
    for (int p = tid; p < M; p += NT) {
        int f;
        float2 g[4];
        rows(p, f, g);
        const int c1 = f & 31, c2 = (f >> 5) & 31, c3 = f >> 10;
        const int word = ((c2 * 2 + (c3 >> 2)) * 32 + c1) * 4 + 2 * ((c3 & 3) >> 1);
        for (int d = 0; d < 4; ++d) {
            out[d * 2 * M + 2 * word + (c3 & 1)] = __float2half_rn(g[d].x * inv);
            out[d * 2 * M + 2 * word + 2 + (c3 & 1)] = __float2half_rn(g[d].y * inv);
        }
    }
    if (tid == 0) scales[h] = sc;
}

cudaError_t simt_precompute_to_tc_pp4(const Plan& p, const void* k, void* Kf, const float2* tw8192, cudaStream_t st) {
    if (p.L > 16384) return cudaErrorInvalidValue;
    const size_t smem = sizeof(float2) * 2 * smem_elems<1>(1 << 13);
    FFTCONV_DISPATCH_T(p.dtype, {
        auto kern = simt_precompute_tc_pp4_kernel<T>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<(unsigned)p.H, fused_threads<13>(), smem, st>>>(
            (const T*)k, p.L, (__half*)Kf, (float*)((uint8_t*)Kf + (size_t)p.H * 4 * (8192 * 4)), tw8192);
        return cudaGetLastError();
    })
}

cudaError_t simt_precompute_to_tc_pp2(const Plan& p, const void* k, void* Kf, const float2* tw8192, cudaStream_t st) {
    if (p.L > 8192) return cudaErrorInvalidValue;
    const size_t smem = sizeof(float2) * smem_elems<1>(1 << 13);
    FFTCONV_DISPATCH_T(p.dtype, {
        auto kern = simt_precompute_tc_pp2_kernel<T>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<(unsigned)p.H, fused_threads<13>(), smem, st>>>(
            (const T*)k, p.L, (__half*)Kf, (float*)((uint8_t*)Kf + (size_t)p.H * 2 * (8192 * 4)), tw8192);
        return cudaGetLastError();
    })
}

cudaError_t simt_precompute_to_tc_pp(const Plan& p, const void* k, void* Kf, cudaStream_t st) {
    if (p.L > 4096) return cudaErrorInvalidValue;     // the 8192-point spectrum of k (<= 4096 taps)
    const size_t smem = sizeof(float2) * smem_elems<1>(1 << 13);
    FFTCONV_DISPATCH_T(p.dtype, {
        auto kern = simt_precompute_tc_pp_kernel<T>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<(unsigned)p.H, fused_threads<13>(), smem, st>>>((const T*)k, p.L, (__half*)Kf,
                                                               (float*)((uint8_t*)Kf + (size_t)p.H * (8192 * 4)), p.tw);
        return cudaGetLastError();
    })
}

template <int LOGM, typename T>
cudaError_t launch_filter_grad(const Plan& p, const void* u, const void* w, const void* v, const void* dy,
                               int64_t B, float* dk, const float2* tw, cudaStream_t st) {
    constexpr int NT = fused_threads<LOGM>();
    const size_t smem = sizeof(float2) * (smem_elems<1>(1 << LOGM) + (1 << (LOGM - 1)) + 1);
    auto kern = simt_filter_grad_kernel<LOGM, T>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // rows per CTA: enough CTAs to fill the GPU several times over, each
    // amortising its inverse transform over several rows
    int64_t rows = (B + 7) / 8;
    if (rows < 1) rows = 1;
    const int64_t chunks = (B + rows - 1) / rows;
    dim3 grid((unsigned)p.H, (unsigned)chunks);
    kern<<<grid, NT, smem, st>>>((const T*)u, (const T*)w, (const T*)v, (const T*)dy, B, p.H, p.L, rows, dk, tw);
    return cudaGetLastError();
}

// dk (fp32, [H, L]) <- the filter gradient over the batch; the plan's
// transform length M = 2N (N <= 8192) and an exp(-2 pi i e / M) table
cudaError_t simt_filter_grad(const Plan& p, const void* u, const void* w, const void* v, const void* dy, int64_t B,
                             float* dk, cudaStream_t st) {
    cudaError_t e = cudaMemsetAsync(dk, 0, sizeof(float) * (size_t)(p.H * p.L), st);
    if (e != cudaSuccess || B == 0) return e;
    const float2* tw = p.twgrad;
    switch (p.dtype) {
        case kBF16:
            switch (p.logM) {
                case 9: return launch_filter_grad<9, __nv_bfloat16>(p, u, w, v, dy, B, dk, tw, st);
                case 10: return launch_filter_grad<10, __nv_bfloat16>(p, u, w, v, dy, B, dk, tw, st);
                case 11: return launch_filter_grad<11, __nv_bfloat16>(p, u, w, v, dy, B, dk, tw, st);
                case 12: return launch_filter_grad<12, __nv_bfloat16>(p, u, w, v, dy, B, dk, tw, st);
                case 13: return launch_filter_grad<13, __nv_bfloat16>(p, u, w, v, dy, B, dk, tw, st);
                case 14: return launch_filter_grad<14, __nv_bfloat16>(p, u, w, v, dy, B, dk, tw, st);
                default: return cudaErrorInvalidValue;
            }
        case kF16:
            switch (p.logM) {
                case 9: return launch_filter_grad<9, __half>(p, u, w, v, dy, B, dk, tw, st);
                case 10: return launch_filter_grad<10, __half>(p, u, w, v, dy, B, dk, tw, st);
                case 11: return launch_filter_grad<11, __half>(p, u, w, v, dy, B, dk, tw, st);
                case 12: return launch_filter_grad<12, __half>(p, u, w, v, dy, B, dk, tw, st);
                case 13: return launch_filter_grad<13, __half>(p, u, w, v, dy, B, dk, tw, st);
                case 14: return launch_filter_grad<14, __half>(p, u, w, v, dy, B, dk, tw, st);
                default: return cudaErrorInvalidValue;
            }
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t simt_fused_precompute(const Plan& p, const void* k, void* Kf, cudaStream_t st) {
    FFTCONV_DISPATCH_T(p.dtype, switch (p.logM) {
        case 9: return launch_fused_pre<9, T>(p, k, Kf, st);
        case 10: return launch_fused_pre<10, T>(p, k, Kf, st);
        case 11: return launch_fused_pre<11, T>(p, k, Kf, st);
        case 12: return launch_fused_pre<12, T>(p, k, Kf, st);
        case 13: return launch_fused_pre<13, T>(p, k, Kf, st);
        case 14: return launch_fused_pre<14, T>(p, k, Kf, st);
        default: return cudaErrorInvalidValue;
    })
}

cudaError_t simt_staged_forward(const Plan& p, const ForwardArgs& a, cudaStream_t st) {
    FFTCONV_DISPATCH_T(p.dtype, return staged_forward_t<T>(p, a, nullptr, st))
}

cudaError_t simt_staged_precompute(const Plan& p, const void* k, void* Kf, cudaStream_t st) {
    ForwardArgs fa{};
    fa.y = Kf;      // the row pass in precompute mode writes K_f through fa.y
    FFTCONV_DISPATCH_T(p.dtype, return staged_forward_t<T>(p, fa, k, st))
}

cudaError_t tc_staged_forward(const Plan& p, const ForwardArgs& a, cudaStream_t st) {
    switch (p.dtype) {
        case kF16: return tc_staged_forward_t<__half>(p, a, st);
        case kBF16: return tc_staged_forward_t<__nv_bfloat16>(p, a, st);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t tc_staged_precompute(const Plan& p, const void* k, void* Kf, cudaStream_t st) {
    switch (p.dtype) {
        case kF16: return tc_staged_precompute_t<__half>(p, k, Kf, st);
        case kBF16: return tc_staged_precompute_t<__nv_bfloat16>(p, k, Kf, st);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t simt_export_rfft(const Plan& p, const void* Kf, float* out, cudaStream_t st) {
    const int64_t total = p.H * (p.N + 1);
    int blocks = (int)((total + 255) / 256);
    if (blocks > 65535) blocks = 65535;
    export_rfft_kernel<<<blocks, 256, 0, st>>>((const float2*)Kf, out, p.H, p.N, p.logM,
                                               p.path == kPathSimtStaged, p.logR, p.logC);
    return cudaGetLastError();
}

}  // namespace fftconv
