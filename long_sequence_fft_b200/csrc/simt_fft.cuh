// simt_fft.cuh -- fp32 FFT stages in shared memory (FP32 lanes, no tensor
// cores).  Used by the fp32 path and as the general-size path.
//
// Index algebra (mixed-radix Cooley-Tukey; the "order-p Monarch
// decomposition" of FlashFFTConv: Efficient Convolutions for Long Sequences
// with Tensor Cores, "Approach"): for a length-L transform with stage radices
// R_0 .. R_{K-1} (R_0 acts on the slowest digit), a position p of the
// in-place array is p = c_0*S_0 + c_1*S_1 + ... + c_{K-1}, S_i = L/(R_0..R_i).
// Forward stage i contracts digit j_i -> c_i (DFT of length R_i over elements
// at stride S_i) and then multiplies by exp(-2 pi i c_i r / (R_i S_i)), r the
// not-yet-contracted lower digits.  After all stages position p holds
// frequency f = c_0 + R_0*c_1 + R_0 R_1*c_2 + ... (the "Monarch-permuted"
// order; no global permutation is ever materialised).  The inverse runs the
// stages in reverse with conjugated twiddles and returns to natural order.
#pragma once

#include "common.cuh"

namespace fftconv {

// Stage schedule for a length 2^LOGL transform: a first stage of radix 4..32
// followed by radix-16 stages (a single stage when LOGL <= 5).
template <int LOGL>
struct Sched {
    static constexpr int K = (LOGL <= 5) ? 1 : (LOGL - 5 + 3) / 4 + 1;
    static constexpr int bits(int i) { return i == 0 ? LOGL - 4 * (K - 1) : 4; }
    static constexpr int stride_bits(int i) {
        int s = LOGL;
        for (int j = 0; j <= i; ++j) s -= bits(j);
        return s;
    }
};

// Host+device digit reversal for the schedule: permuted position -> frequency.
__host__ __device__ inline int64_t sched_bits(int logl, int i) {
    int K = (logl <= 5) ? 1 : (logl - 5 + 3) / 4 + 1;
    return i == 0 ? logl - 4 * (K - 1) : 4;
}
__host__ __device__ inline int sched_stages(int logl) { return (logl <= 5) ? 1 : (logl - 5 + 3) / 4 + 1; }

__host__ __device__ inline int64_t perm_to_freq(int64_t p, int logl) {
    // p = c_0 S_0 + ... ; f = c_0 + R_0 c_1 + ...
    int K = sched_stages(logl);
    int64_t f = 0;
    int shift_p = logl, shift_f = 0;
    for (int i = 0; i < K; ++i) {
        int b = (int)sched_bits(logl, i);
        shift_p -= b;
        int64_t c = (p >> shift_p) & ((1LL << b) - 1);
        f |= c << shift_f;
        shift_f += b;
    }
    return f;
}
__host__ __device__ inline int64_t freq_to_perm(int64_t f, int logl) {
    int K = sched_stages(logl);
    int64_t p = 0;
    int shift_p = logl, shift_f = 0;
    for (int i = 0; i < K; ++i) {
        int b = (int)sched_bits(logl, i);
        shift_p -= b;
        int64_t c = (f >> shift_f) & ((1LL << b) - 1);
        p |= c << shift_p;
        shift_f += b;
    }
    return p;
}

// Shared-memory index of (position p, batch column col).  With one column the
// array is padded by one element every 16 so that stride-16 and unit-stride
// stage accesses are free of bank conflicts; with TC >= 32 columns the column
// index is the fastest (conflict-free) dimension.
template <int TC>
__device__ __forceinline__ int sidx(int p, int col) {
    if constexpr (TC == 1) return p + (p >> 4);
    else return p * TC + col;
}
template <int TC>
__host__ __device__ constexpr int smem_elems(int L) { return TC == 1 ? L + L / 16 : L * TC; }

// x[c] *= w^c (or conj(w)^c) for c = 1..R-1, where w = tw[e1] is a table
// entry.  Instead of gathering R-1 table entries at stride e1 (uncoalesced
// across a warp), at most three coalesced entries w, w^4, w^16 are loaded and
// the other powers formed by products of at most four factors, which keeps
// the rounding error within a few fp32 ulps.
template <int R, bool CONJ>
__device__ __forceinline__ void twiddle_powers(float2 (&x)[R], const float2* __restrict__ tw, int e1) {
    auto mul = [](float2 a, float2 b) { return CONJ ? cmulc(a, b) : cmul(a, b); };
    const float2 w1 = __ldg(&tw[e1]);
    if constexpr (R == 2) {
        x[1] = mul(x[1], w1);
    } else {
        float2 p[4];
        p[1] = w1;
        p[2] = cmul(w1, w1);
        p[3] = cmul(p[2], w1);
        if constexpr (R == 4) {
#pragma unroll
            for (int c = 1; c < 4; ++c) x[c] = mul(x[c], p[c]);
        } else {
            constexpr int Q = R / 4;
            float2 q[Q];
            const float2 w4 = __ldg(&tw[4 * e1]);
            q[1] = w4;
            if constexpr (Q > 2) q[2] = cmul(w4, w4);
            if constexpr (Q > 3) q[3] = cmul(q[2], w4);
            if constexpr (Q > 4) {
                const float2 w16 = __ldg(&tw[16 * e1]);
                q[4] = w16;
#pragma unroll
                for (int a = 5; a < Q; ++a) q[a] = cmul(w16, q[a - 4]);
            }
#pragma unroll
            for (int c = 1; c < R; ++c) {
                const int a = c / 4, b = c % 4;
                float2 w;
                if (a == 0) w = p[b];
                else if (b == 0) w = q[a];
                else w = cmul(q[a], p[b]);
                x[c] = mul(x[c], w);
            }
        }
    }
}

// Forward stage I of a length-2^LOGL transform over TC batch columns held in
// shared memory.  tw = exp(-2 pi i e / Ltab) for e < Ltab, Ltab = L << twshift.
template <int LOGL, int I, int TC, int NT>
__device__ __forceinline__ void fwd_stage(float2* s, const float2* __restrict__ tw, int twshift, int tid) {
    constexpr int LB = Sched<LOGL>::bits(I);
    constexpr int R = 1 << LB;
    constexpr int SB = Sched<LOGL>::stride_bits(I);
    constexpr int S = 1 << SB;
    constexpr int G = ((1 << LOGL) / R) * TC;
    for (int g = tid; g < G; g += NT) {
        const int col = (TC == 1) ? 0 : (g % TC);
        const int d = (TC == 1) ? g : (g / TC);
        const int r = d & (S - 1);
        const int base = (d >> SB) * (S * R) + r;
        float2 x[R];
#pragma unroll
        for (int j = 0; j < R; ++j) x[j] = s[sidx<TC>(base + j * S, col)];
        Dft<R, -1>::run(x);
        if constexpr (S > 1) twiddle_powers<R, false>(x, tw, r << (twshift + (LOGL - SB - LB)));
#pragma unroll
        for (int c = 0; c < R; ++c) s[sidx<TC>(base + c * S, col)] = x[c];
    }
}

// Forward stage 0 of a transform whose upper half is zero (x[p] = 0 for
// p >= L/2, i.e. for the slowest digit j_0 >= R_0/2): reads only the nonzero
// half of each butterfly's inputs and skips the first butterfly level
// (Dft::run_half_input).  The zero half need not be stored.
template <int LOGL, int TC, int NT>
__device__ __forceinline__ void fwd_stage0_half_input(float2* s, const float2* __restrict__ tw, int twshift,
                                                      int tid) {
    constexpr int LB = Sched<LOGL>::bits(0);
    constexpr int R = 1 << LB;
    constexpr int SB = Sched<LOGL>::stride_bits(0);
    constexpr int S = 1 << SB;
    constexpr int G = S * TC;                    // stage 0: one butterfly per (r < S, column)
    for (int g = tid; g < G; g += NT) {
        const int col = (TC == 1) ? 0 : (g % TC);
        const int r = (TC == 1) ? g : (g / TC);
        float2 x[R];
#pragma unroll
        for (int j = 0; j < R / 2; ++j) x[j] = s[sidx<TC>(r + j * S, col)];
#pragma unroll
        for (int j = R / 2; j < R; ++j) x[j] = make_float2(0.f, 0.f);
        Dft<R, -1>::run_half_input(x);
        if constexpr (S > 1) twiddle_powers<R, false>(x, tw, r << (twshift + (LOGL - SB - LB)));
#pragma unroll
        for (int c = 0; c < R; ++c) s[sidx<TC>(r + c * S, col)] = x[c];
    }
}

// Inverse of fwd_stage (conjugate twiddle, then inverse DFT).  Unnormalised.
template <int LOGL, int I, int TC, int NT>
__device__ __forceinline__ void inv_stage(float2* s, const float2* __restrict__ tw, int twshift, int tid) {
    constexpr int LB = Sched<LOGL>::bits(I);
    constexpr int R = 1 << LB;
    constexpr int SB = Sched<LOGL>::stride_bits(I);
    constexpr int S = 1 << SB;
    constexpr int G = ((1 << LOGL) / R) * TC;
    for (int g = tid; g < G; g += NT) {
        const int col = (TC == 1) ? 0 : (g % TC);
        const int d = (TC == 1) ? g : (g / TC);
        const int r = d & (S - 1);
        const int base = (d >> SB) * (S * R) + r;
        float2 x[R];
#pragma unroll
        for (int c = 0; c < R; ++c) x[c] = s[sidx<TC>(base + c * S, col)];
        if constexpr (S > 1) twiddle_powers<R, true>(x, tw, r << (twshift + (LOGL - SB - LB)));
        Dft<R, +1>::run(x);
#pragma unroll
        for (int j = 0; j < R; ++j) s[sidx<TC>(base + j * S, col)] = x[j];
    }
}

// Forward stages [FIRST, LAST) in order, with a barrier after each.
template <int LOGL, int FIRST, int LAST, int TC, int NT>
__device__ __forceinline__ void fwd_stages(float2* s, const float2* __restrict__ tw, int twshift, int tid) {
    if constexpr (FIRST < LAST) {
        fwd_stage<LOGL, FIRST, TC, NT>(s, tw, twshift, tid);
        __syncthreads();
        fwd_stages<LOGL, FIRST + 1, LAST, TC, NT>(s, tw, twshift, tid);
    }
}
// Inverse stages LAST-1 down to FIRST, with a barrier after each.
template <int LOGL, int FIRST, int LAST, int TC, int NT>
__device__ __forceinline__ void inv_stages(float2* s, const float2* __restrict__ tw, int twshift, int tid) {
    if constexpr (FIRST < LAST) {
        inv_stage<LOGL, LAST - 1, TC, NT>(s, tw, twshift, tid);
        __syncthreads();
        inv_stages<LOGL, FIRST, LAST - 1, TC, NT>(s, tw, twshift, tid);
    }
}

}  // namespace fftconv
