// tc_kernels.cu -- tensor-core (tcgen05) fused FFT convolution, sm_100a.
//
// FlashFFTConv: Efficient Convolutions for Long Sequences with Tensor Cores,
// "Approach": the FFT convolution is rewritten as an order-p Monarch
// decomposition -- matrix-matrix products with small DFT factors applied
// along one digit of the sequence index -- so the transform runs on tensor
// cores, permutations become on-chip transposes, and the whole convolution
// (gates included, "Key results") is one kernel.
//
// This kernel: sequence length N = 4096, transform length M = 8192.
//   t = 256*j1 + 8*l + j3   (j1 < 32, zero for j1 >= 16;  l < 32;  j3 < 8)
//   f = c1 + 32*c2 + 1024*c3
//   exp(-2 pi i f t / M) = w32^(c1 j1) w1024^(c1 l) wM^(c1 j3) w32^(c2 l) w256^(c2 j3) w8^(c3 j3)
// Forward: S1 contracts j1 (DFT-32 on 16 nonzero inputs), twiddle w1024^(c1 l),
// S2 contracts l (DFT-32), twiddle wM^(c1 j3), S3 contracts j3 with the
// per-c2 factor w8^(c3 j3) w256^(c2 j3) (the second twiddle folded into the
// matrix).  Product with the filter spectrum, then the mirror image with
// conjugate factors; the last inverse stage emits only t < N.
//
// Data layout.  One CTA tile = 4 pairs of batch rows (the two real sequences
// of a pair are the real and imaginary parts of one complex sequence; the
// filter is real, so both come back exact).  Pair q owns TMEM lanes
// [32q, 32q+32).  Every stage is a tcgen05.mma with M = 128 rows (the 4 pairs
// x 32 values of one digit), complex numbers as interleaved (re, im) pairs of
// fp16 and the DFT factor as the real 2n x 2n matrix [[Re, Im], [-Im, Re]] in
// shared memory.  Stages whose contracted digit already sits inside a TMEM
// lane (S1, S3 and their inverses) take A from TMEM; the two stages that
// contract the lane digit (S2, S2') and the last inverse stage take A from
// shared memory, written by the previous epilogue in the transposed order
// (the "on-chip transpose").  Accumulators are fp32 in TMEM; twiddles and the
// filter product are applied in fp32 by the epilogue warps, which round to
// fp16 for the next stage.  Each DFT factor carries 1/sqrt(n), so the forward
// and inverse transforms are unitary and the filter spectrum is used
// unnormalised.
//
// Warp roles: warps 0..15 are epilogue warps (warp w serves lane quarter
// w % 4 and the column slice w / 4), warp 16 issues the MMAs.  Accumulators
// are double-buffered (two 128-column TMEM buffers); mbarriers hand chunks
// between the MMA warp and the epilogue warps.  Every wait is bounded: on
// timeout the kernel records FFTCONV_ERR_TIMEOUT in the plan's status word,
// drains, frees its TMEM and returns.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cmath>
#include <complex>
#include <cstring>
#include <vector>

#include "common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

namespace fftconv {

cudaError_t simt_precompute_to_tc_layout(const Plan& p, const void* k, void* Kf, cudaStream_t s);

namespace {

using namespace tc;

constexpr int kN = 4096;
constexpr int kM = 8192;
constexpr int kEpiWarps = 16;
constexpr int kThreads = (kEpiWarps + 1) * 32;
constexpr int kChunksPerUnit = 22;   // 4 chunks in each of S1..S2', 2 in S1'
constexpr uint32_t kWaitLimit = 1u << 20;

// shared-memory map (bytes from a 1024-aligned base)
constexpr int kTile = 16384;                 // 128 rows x 128 B, 128-byte swizzle
constexpr int kOffData = 0;                  // 8 tiles (one per j3)
constexpr int kOffBS1 = 8 * kTile;           // K=32 N=64   4 KB
constexpr int kOffBS2 = kOffBS1 + 4096;      // K=64 N=64   8 KB
constexpr int kOffBS3 = kOffBS2 + 8192;      // 32 x (K=16 N=16)  16 KB
constexpr int kOffBS3i = kOffBS3 + 16384;    // 32 x (K=16 N=16)  16 KB
constexpr int kOffBS2i = kOffBS3i + 16384;   // K=64 N=64   8 KB
constexpr int kOffBS1i = kOffBS2i + 8192;    // K=64 N=32   4 KB
constexpr int kOffBEnd = kOffBS1i + 4096;
constexpr int kBImageBytes = kOffBEnd - kOffBS1;   // 57344
constexpr int kOffBars = kOffBEnd;           // 8 mbarriers
constexpr int kOffMisc = kOffBars + 64;      // tmem base, abort flag
constexpr int kSmemBytes = kOffMisc + 64 + 1024;    // + alignment slack

// byte offset of element (n, k) of a K x N B operand in the no-swizzle
// K-major layout used for every DFT factor: 8x8 core matrices, K-halves
// LBO = (N/8)*128 bytes apart, 8-row groups 128 bytes apart.
inline size_t bimg_offset(int n, int k, int N) {
    return (size_t)(k / 8) * (N / 8) * 128 + (size_t)(n / 8) * 128 + (n % 8) * 16 + (k % 8) * 2;
}

struct TcArgs {
    const void* u;
    const void* w;
    const void* v;
    void* y;
    const float2* Kf;          // [H][c2][c3][c1] complex fp32, unnormalised
    const uint8_t* mask;
    int64_t mask_h;
    int64_t B, H;
    int64_t npairs;            // H * ceil(B/2)
    int64_t nunits;            // ceil(npairs / 4)
    const uint4* bimg;         // DFT factors, image of the shared-memory region
    const float2* tw1024;      // exp(-2 pi i e/1024), e < 1024
    const float2* twM;         // exp(-2 pi i e/8192), e < 256
    int* status;
};

template <typename T>
struct IO;
template <>
struct IO<__nv_bfloat16> {
    static __device__ __forceinline__ float2 unpack2(uint32_t v) {
        return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
    }
    static __device__ __forceinline__ uint32_t pack2(float a, float b) {
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<uint32_t*>(&h);
    }
};
template <>
struct IO<__half> {
    static __device__ __forceinline__ float2 unpack2(uint32_t v) {
        __half2 h = *reinterpret_cast<__half2*>(&v);
        return __half22float2(h);
    }
    static __device__ __forceinline__ uint32_t pack2(float a, float b) {
        __half2 h = __floats2half2_rn(a, b);
        return *reinterpret_cast<uint32_t*>(&h);
    }
};

__device__ __forceinline__ uint32_t pack_h2(float re, float im) {
    __half2 h = __floats2half2_rn(re, im);
    return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float2 f2(uint32_t a, uint32_t b) { return make_float2(__uint_as_float(a), __uint_as_float(b)); }

// 128-byte swizzle of a logical byte offset inside a 1024-byte-aligned tile
__device__ __forceinline__ uint32_t swz(uint32_t off) { return off ^ (((off >> 7) & 7u) << 4); }

struct PairInfo {
    int64_t o0, o1;      // element offsets of rows b0 and b1 (o1 < 0: absent)
    int64_t h;
    bool valid;
};

__device__ __forceinline__ PairInfo pair_info(const TcArgs& a, int64_t pair) {
    PairInfo p;
    p.valid = pair < a.npairs;
    const int64_t PB = (a.B + 1) / 2;
    const int64_t pp = p.valid ? pair : 0;
    p.h = pp / PB;
    const int64_t b0 = 2 * (pp % PB), b1 = b0 + 1;
    p.o0 = (b0 * a.H + p.h) * kN;
    p.o1 = b1 < a.B ? (b1 * a.H + p.h) * kN : -1;
    return p;
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 1) tc_fftconv_n4096_kernel(TcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t* bar = (uint64_t*)(smem + kOffBars);
    uint64_t* bar_in = bar + 0;
    uint64_t* dfull = bar + 1;   // [2]
    uint64_t* dfree = bar + 3;   // [2]
    uint64_t* bar_fin = bar + 5;
    uint32_t* tmem_base_sh = (uint32_t*)(smem + kOffMisc);
    volatile int* abort_flag = (volatile int*)(smem + kOffMisc + 4);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const uint32_t sbase = smem_u32(smem);

    if (tid == 0) {
        mbar_init(bar_in, kEpiWarps);
        mbar_init(&dfull[0], 1);
        mbar_init(&dfull[1], 1);
        mbar_init(&dfree[0], kEpiWarps);
        mbar_init(&dfree[1], kEpiWarps);
        mbar_init(bar_fin, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kEpiWarps) tmem_alloc(tmem_base_sh, 512);
    // DFT factors into shared memory
    {
        uint4* dst = (uint4*)(smem + kOffBS1);
        for (int i = tid; i < kBImageBytes / 16; i += kThreads) dst[i] = __ldg(&a.bimg[i]);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_base_sh;

    // Bounded wait, made warp-uniform so that warp-collective tcgen05
    // instructions are never reached by only part of a warp.
    auto wait = [&](uint64_t* b, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, mbar_wait_bounded(b, parity, abort_flag, kWaitLimit));
    };
    auto fail = [&](void) {
        if (!*abort_flag) {
            *abort_flag = 1;
            atomicExch(a.status, kStatusTimeout);
        }
    };

    if (warp == kEpiWarps) {
        // ============================ MMA issuer ============================
        const uint32_t id64 = idesc_f16_f32(128, 64);
        const uint32_t id16 = idesc_f16_f32(128, 16);
        uint32_t g = 0;          // global chunk counter
        int iter = 0;
        bool ok = true;
        for (int64_t unit = blockIdx.x; unit < a.nunits && ok; unit += gridDim.x, ++iter) {
            if (!wait(bar_in, iter & 1)) { ok = false; fail(); break; }
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < kChunksPerUnit && ok; ++c, ++g) {
                const int stage = c < 20 ? (c >> 2) : 5, k = c < 20 ? (c & 3) : c - 20;
                const uint32_t b = g & 1;
                if (g >= 2 && !wait(&dfree[b], ((g - 2) >> 1) & 1)) {
                    ok = false; fail(); break;
                }
                // stages whose chunks regroup the data need every epilogue of
                // the previous stage, including the one on the other buffer
                if ((stage == 2 || stage == 4 || stage == 5) && k == 0 &&
                    !wait(&dfree[b ^ 1], ((g - 1) >> 1) & 1)) {
                    ok = false; fail(); break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t d = tbase + 256 + 128 * b;
                    if (stage == 0) {            // S1: A1 (TMEM) cols j3*16 + j1
                        for (int jj = 0; jj < 2; ++jj) {
                            const int j3 = 2 * k + jj;
                            for (int s = 0; s < 2; ++s)
                                mma_ts(d + jj * 64, tbase + j3 * 16 + s * 8,
                                       make_desc(sbase + kOffBS1 + s * 2 * 1024, 1024, 128, 0), id64, s);
                        }
                    } else if (stage == 1) {     // S2: A2 (smem tile j3)
                        for (int jj = 0; jj < 2; ++jj) {
                            const int j3 = 2 * k + jj;
                            for (int s = 0; s < 4; ++s)
                                mma_ss(d + jj * 64, make_desc(sbase + kOffData + j3 * kTile + 32 * s, 16, 1024, 2),
                                       make_desc(sbase + kOffBS2 + s * 2 * 1024, 1024, 128, 0), id64, s);
                        }
                    } else if (stage == 2 || stage == 3) {   // S3 / S3': A (TMEM) cols c2*8 + j3|c3
                        const int off = stage == 2 ? kOffBS3 : kOffBS3i;
                        for (int cl = 0; cl < 8; ++cl) {
                            const int c2 = 8 * k + cl;
                            mma_ts(d + cl * 16, tbase + c2 * 8,
                                   make_desc(sbase + off + c2 * 512, 256, 128, 0), id16, 0);
                        }
                    } else if (stage == 4) {     // S2': A5 (smem tile j3), K = c2
                        for (int jj = 0; jj < 2; ++jj) {
                            const int j3 = 2 * k + jj;
                            for (int s = 0; s < 4; ++s)
                                mma_ss(d + jj * 64, make_desc(sbase + kOffData + j3 * kTile + 32 * s, 16, 1024, 2),
                                       make_desc(sbase + kOffBS2i + s * 2 * 1024, 1024, 128, 0), id64, s);
                        }
                    } else {                     // S1': A6 (smem tile j3), K = c1; chunk k: j1 in [8k, 8k+8)
                        for (int j3 = 0; j3 < 8; ++j3) {
                            for (int s = 0; s < 4; ++s)
                                mma_ss(d + j3 * 16, make_desc(sbase + kOffData + j3 * kTile + 32 * s, 16, 1024, 2),
                                       make_desc(sbase + kOffBS1i + 256 * k + s * 2 * 512, 512, 128, 0), id16, s);
                        }
                    }
                    tc_commit(&dfull[b]);
                }
                __syncwarp();
            }
        }
        // drain: every issued MMA must finish before TMEM is released
        if (lane == 0) tc_commit(bar_fin);
        __syncwarp();
        if (!wait(bar_fin, 0)) fail();
    } else {
        // ========================== epilogue warps ==========================
        const int q = warp & 3;          // lane quarter = pair within the tile
        const int s = warp >> 2;         // column slice
        const uint32_t lq = (uint32_t)(32 * q) << 16;
        const int64_t N = kN;
        const int64_t nblk = N / 32;

        // loop-invariant twiddles
        // (the wM^(c1 j3) twiddles are read from the L1-resident table per use)
        float2 tw1[8], tw3[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            tw1[i] = __ldg(&a.tw1024[((8 * s + i) * lane) & 1023]);   // w1024^(c1 l), l = lane
            tw3[i] = __ldg(&a.tw1024[(lane * (8 * s + i)) & 1023]);   // w1024^(c1 l), c1 = lane
        }

        uint32_t g = 0;
        int iter = 0;
        bool ok = true;
        for (int64_t unit = blockIdx.x; unit < a.nunits && ok; unit += gridDim.x, ++iter) {
            const PairInfo P = pair_info(a, unit * 4 + q);
            const T* u0 = (const T*)a.u + P.o0;
            const T* w0 = a.w ? (const T*)a.w + P.o0 : nullptr;
            const bool has1 = P.o1 >= 0;
            const T* u1 = has1 ? (const T*)a.u + P.o1 : nullptr;
            const T* w1 = (has1 && a.w) ? (const T*)a.w + P.o1 : nullptr;

            // ---- load: x = u*w for t = 256*j1 + 8*l + j3, j1 in [4s, 4s+4)
            {
                uint32_t packed[8][4];   // [j3][j1 - 4s]
#pragma unroll
                for (int jl = 0; jl < 4; ++jl) {
                    const int j1 = 4 * s + jl;
                    const int64_t t0 = 256 * j1 + 8 * lane;
                    float xa[8], xb[8];
                    if (P.valid) {
                        const uint4 ua = __ldg((const uint4*)(u0 + t0));
                        const uint32_t uw[4] = {ua.x, ua.y, ua.z, ua.w};
                        uint32_t ww[4] = {0x3f803f80u, 0x3f803f80u, 0x3f803f80u, 0x3f803f80u};
                        if (w0) { const uint4 wa = __ldg((const uint4*)(w0 + t0)); ww[0] = wa.x; ww[1] = wa.y; ww[2] = wa.z; ww[3] = wa.w; }
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 uu = IO<T>::unpack2(uw[e]);
                            const float2 gg = w0 ? IO<T>::unpack2(ww[e]) : make_float2(1.f, 1.f);
                            xa[2 * e] = uu.x * gg.x;
                            xa[2 * e + 1] = uu.y * gg.y;
                        }
                        if (u1) {
                            const uint4 ub = __ldg((const uint4*)(u1 + t0));
                            const uint32_t ubw[4] = {ub.x, ub.y, ub.z, ub.w};
                            uint32_t wb[4];
                            if (w1) { const uint4 t4 = __ldg((const uint4*)(w1 + t0)); wb[0] = t4.x; wb[1] = t4.y; wb[2] = t4.z; wb[3] = t4.w; }
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 uu = IO<T>::unpack2(ubw[e]);
                                const float2 gg = w1 ? IO<T>::unpack2(wb[e]) : make_float2(1.f, 1.f);
                                xb[2 * e] = uu.x * gg.x;
                                xb[2 * e + 1] = uu.y * gg.y;
                            }
                        } else {
#pragma unroll
                            for (int e = 0; e < 8; ++e) xb[e] = 0.f;
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 8; ++e) { xa[e] = 0.f; xb[e] = 0.f; }
                    }
#pragma unroll
                    for (int j3 = 0; j3 < 8; ++j3) packed[j3][jl] = pack_h2(xa[j3], xb[j3]);
                }
#pragma unroll
                for (int j3 = 0; j3 < 8; ++j3) tmem_st4(tbase + lq + j3 * 16 + 4 * s, packed[j3]);
                tc_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_in);
            }

            // warm L2 with the next tile's rows (u, w, v of both sequences and
            // the filter spectrum) while this tile is being transformed
            if (s == 0 && lane < 7) {
                const int64_t nu = unit + gridDim.x;
                if (nu < a.nunits) {
                    const PairInfo Q = pair_info(a, nu * 4 + q);
                    if (Q.valid) {
                        const void* src = nullptr;
                        uint32_t bytes = kN * sizeof(T);
                        if (lane == 0) src = (const T*)a.u + Q.o0;
                        else if (lane == 1 && a.w) src = (const T*)a.w + Q.o0;
                        else if (lane == 2 && a.v) src = (const T*)a.v + Q.o0;
                        else if (lane == 3 && Q.o1 >= 0) src = (const T*)a.u + Q.o1;
                        else if (lane == 4 && Q.o1 >= 0 && a.w) src = (const T*)a.w + Q.o1;
                        else if (lane == 5 && Q.o1 >= 0 && a.v) src = (const T*)a.v + Q.o1;
                        else if (lane == 6) { src = a.Kf + Q.h * (int64_t)kM; bytes = kM * sizeof(float2); }
                        if (src) prefetch_l2(src, bytes);
                    }
                }
            }

            // per-tile epilogue state
            const float2* Kh = a.Kf + P.h * (int64_t)kM;
            const uint8_t* mrow = a.mask ? a.mask + (a.mask_h == 1 ? 0 : P.h) * nblk : nullptr;
            T* y0 = (T*)a.y + P.o0;
            T* y1 = has1 ? (T*)a.y + P.o1 : nullptr;
            const T* v0 = a.v ? (const T*)a.v + P.o0 : nullptr;
            const T* v1 = (has1 && a.v) ? (const T*)a.v + P.o1 : nullptr;

#pragma unroll 1
            for (int c = 0; c < kChunksPerUnit; ++c, ++g) {
                const int stage = c < 20 ? (c >> 2) : 5, k = c < 20 ? (c & 3) : c - 20;
                const uint32_t b = g & 1;
                if (!wait(&dfull[b], (g >> 1) & 1)) { ok = false; fail(); break; }
                tc_fence_after();
                const uint32_t dcol = tbase + lq + 256 + 128 * b;

                if (stage == 0) {
                    // E1: lane = l; columns (jj, c1 = 8s + i); twiddle w1024^(c1 l);
                    // write A2 tile j3, row 32q + c1, K element pair 2l
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) {
                        uint32_t r[16];
                        tmem_ld16(dcol + jj * 64 + 16 * s, r);
                        tc_wait_ld();
                        uint8_t* tile = smem + kOffData + (2 * k + jj) * kTile;
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const float2 z = cmul(f2(r[2 * i], r[2 * i + 1]), tw1[i]);
                            const uint32_t off = (uint32_t)(4 * q + s) * 1024 + i * 128 + ((4 * lane) ^ (i << 4));
                            *(uint32_t*)(tile + off) = pack_h2(z.x, z.y);
                        }
                    }
                    fence_proxy_async_smem();
                } else if (stage == 1) {
                    // E2: lane = c1; columns (jj, c2 = 8s + i); twiddle wM^(c1 j3);
                    // write A3 (TMEM) col c2*8 + j3
                    uint32_t h[2][8];
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) {
                        uint32_t r[16];
                        tmem_ld16(dcol + jj * 64 + 16 * s, r);
                        tc_wait_ld();
                        const float2 t = __ldg(&a.twM[lane * (2 * k + jj)]);
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const float2 z = cmul(f2(r[2 * i], r[2 * i + 1]), t);
                            h[jj][i] = pack_h2(z.x, z.y);
                        }
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i) tmem_st2(tbase + lq + (8 * s + i) * 8 + 2 * k, h[0][i], h[1][i]);
                    tc_wait_st();
                } else if (stage == 2) {
                    // EK: lane = c1; columns (c2 = 8k + 2s + cc, c3); times K_f;
                    // write A4 (TMEM) col c2*8 + c3 (in place)
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        const int c2 = 8 * k + 2 * s + cc;
                        uint32_t r[16];
                        tmem_ld16(dcol + (2 * s + cc) * 16, r);
                        float2 kv[8];
#pragma unroll
                        for (int c3 = 0; c3 < 8; ++c3) kv[c3] = __ldg(&Kh[(c2 * 8 + c3) * 32 + lane]);
                        tc_wait_ld();
                        uint32_t h8[8];
#pragma unroll
                        for (int c3 = 0; c3 < 8; ++c3) {
                            float2 kk = kv[c3];
                            if (mrow) {
                                const int64_t f = lane + 32 * c2 + 1024 * c3;
                                const int64_t gb = f <= N ? f : kM - f;
                                int64_t blk = gb >> 5;
                                if (blk >= nblk) blk = nblk - 1;
                                if (__ldg(&mrow[blk]) == 0) kk = make_float2(0.f, 0.f);
                            }
                            const float2 z = cmul(f2(r[2 * c3], r[2 * c3 + 1]), kk);
                            h8[c3] = pack_h2(z.x, z.y);
                        }
                        tmem_st8(tbase + lq + c2 * 8, h8);
                    }
                    tc_wait_st();
                } else if (stage == 3) {
                    // E3': lane = c1; columns (c2 = 8k + cl, j3 = 2s + jj); twiddle
                    // conj wM^(c1 j3); write A5 tile j3, row 32q + c1, K pair 2*c2
                    uint32_t h[2][8];
                    const float2 t0 = __ldg(&a.twM[lane * (2 * s)]), t1 = __ldg(&a.twM[lane * (2 * s + 1)]);
#pragma unroll
                    for (int cl = 0; cl < 8; ++cl) {
                        uint32_t r[4];
                        tmem_ld4(dcol + cl * 16 + 4 * s, r);
                        tc_wait_ld();
#pragma unroll
                        for (int jj = 0; jj < 2; ++jj) {
                            const float2 z = cmulc(f2(r[2 * jj], r[2 * jj + 1]), jj ? t1 : t0);
                            h[jj][cl] = pack_h2(z.x, z.y);
                        }
                    }
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) {
                        uint8_t* tile = smem + kOffData + (2 * s + jj) * kTile;
                        const uint32_t m = 32 * q + lane;
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const uint32_t off = (m >> 3) * 1024 + (m & 7) * 128 + (32 * k + 16 * hh);
                            *(uint4*)(tile + swz(off)) =
                                make_uint4(h[jj][4 * hh], h[jj][4 * hh + 1], h[jj][4 * hh + 2], h[jj][4 * hh + 3]);
                        }
                    }
                    fence_proxy_async_smem();
                } else if (stage == 4) {
                    // E2': lane = c1; columns (jj, l = 8s + i); twiddle conj w1024^(c1 l);
                    // write A6 tile j3 (in place), row 32q + l, K pair 2*c1
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) {
                        uint32_t r[16];
                        tmem_ld16(dcol + jj * 64 + 16 * s, r);
                        tc_wait_ld();
                        uint8_t* tile = smem + kOffData + (2 * k + jj) * kTile;
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const float2 z = cmulc(f2(r[2 * i], r[2 * i + 1]), tw3[i]);
                            const uint32_t off = (uint32_t)(4 * q + s) * 1024 + i * 128 + ((4 * lane) ^ (i << 4));
                            *(uint32_t*)(tile + off) = pack_h2(z.x, z.y);
                        }
                    }
                    fence_proxy_async_smem();
                } else {
                    // EO: lane = l; chunk k holds j1 in [8k, 8k+8) for every j3 at
                    // columns j3*16 + 2*(j1 - 8k); this warp takes j1 = 8k + 2s + jj
                    // and writes y = v * z at t = 256 j1 + 8 l + j3, 8 consecutive t
                    // per (row, j1) as one 16-byte store.
                    if (P.valid) {
                        uint4 va[2], vb[2];
#pragma unroll
                        for (int jj = 0; jj < 2; ++jj) {
                            const int64_t t0 = 256 * (8 * k + 2 * s + jj) + 8 * lane;
                            va[jj] = v0 ? __ldg((const uint4*)(v0 + t0)) : make_uint4(0, 0, 0, 0);
                            vb[jj] = v1 ? __ldg((const uint4*)(v1 + t0)) : make_uint4(0, 0, 0, 0);
                        }
                        uint32_t r[8][4];
#pragma unroll
                        for (int j3 = 0; j3 < 8; ++j3) tmem_ld4(dcol + j3 * 16 + 4 * s, r[j3]);
                        tc_wait_ld();
#pragma unroll
                        for (int jj = 0; jj < 2; ++jj) {
                            const int64_t t0 = 256 * (8 * k + 2 * s + jj) + 8 * lane;
                            const uint32_t vaw[4] = {va[jj].x, va[jj].y, va[jj].z, va[jj].w};
                            const uint32_t vbw[4] = {vb[jj].x, vb[jj].y, vb[jj].z, vb[jj].w};
                            uint32_t oa[4], ob[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                float a0 = __uint_as_float(r[2 * e][2 * jj]), a1 = __uint_as_float(r[2 * e + 1][2 * jj]);
                                float b0 = __uint_as_float(r[2 * e][2 * jj + 1]), b1 = __uint_as_float(r[2 * e + 1][2 * jj + 1]);
                                if (v0) { const float2 g = IO<T>::unpack2(vaw[e]); a0 *= g.x; a1 *= g.y; }
                                if (v1) { const float2 g = IO<T>::unpack2(vbw[e]); b0 *= g.x; b1 *= g.y; }
                                oa[e] = IO<T>::pack2(a0, a1);
                                ob[e] = IO<T>::pack2(b0, b1);
                            }
                            *(uint4*)(y0 + t0) = make_uint4(oa[0], oa[1], oa[2], oa[3]);
                            if (y1) *(uint4*)(y1 + t0) = make_uint4(ob[0], ob[1], ob[2], ob[3]);
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&dfree[b]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kEpiWarps) {
        tc_fence_after();
        tmem_dealloc(tbase, 512);
        tmem_relinquish();
    }
}

// ----------------------------------------------------------- host side ---

struct TcResources {
    uint8_t* bimg = nullptr;
    float2* tw1024 = nullptr;
    float2* twM = nullptr;
    int num_sms = 0;
};

std::complex<double> wpow(long long e, long long n, int sign) {
    const double two_pi = 6.283185307179586476925286766559;
    const long long r = ((e % n) + n) % n;
    const double a = two_pi * (double)r / (double)n;
    return std::complex<double>(std::cos(a), sign * std::sin(a));
}

void put_f16(std::vector<uint8_t>& img, size_t off, double v) {
    const __half h = __double2half(v);
    std::memcpy(&img[off], &h, 2);
}

// Real-pair image of complex F (n_out x n_in) as a K x N B operand:
// K = 2*n_in (input re/im interleaved), N = 2*n_out.
void put_complex_matrix(std::vector<uint8_t>& img, size_t base, int n_out, int n_in,
                        const std::vector<std::complex<double>>& F) {
    const int N = 2 * n_out;
    for (int c = 0; c < n_out; ++c)
        for (int j = 0; j < n_in; ++j) {
            const std::complex<double> f = F[(size_t)c * n_in + j];
            put_f16(img, base + bimg_offset(2 * c, 2 * j, N), f.real());
            put_f16(img, base + bimg_offset(2 * c, 2 * j + 1, N), -f.imag());
            put_f16(img, base + bimg_offset(2 * c + 1, 2 * j, N), f.imag());
            put_f16(img, base + bimg_offset(2 * c + 1, 2 * j + 1, N), f.real());
        }
}

std::vector<uint8_t> build_bimage() {
    std::vector<uint8_t> img(kBImageBytes, 0);
    const double r32 = 1.0 / std::sqrt(32.0), r8 = 1.0 / std::sqrt(8.0);
    auto off = [](int o) { return (size_t)(o - kOffBS1); };
    std::vector<std::complex<double>> F;
    // S1: c1 <- j1 (j1 < 16)
    F.assign(32 * 16, 0);
    for (int c = 0; c < 32; ++c) for (int j = 0; j < 16; ++j) F[c * 16 + j] = wpow((long long)c * j, 32, -1) * r32;
    put_complex_matrix(img, off(kOffBS1), 32, 16, F);
    // S2: c2 <- l
    F.assign(32 * 32, 0);
    for (int c = 0; c < 32; ++c) for (int j = 0; j < 32; ++j) F[c * 32 + j] = wpow((long long)c * j, 32, -1) * r32;
    put_complex_matrix(img, off(kOffBS2), 32, 32, F);
    // S3 (per c2): c3 <- j3 with w8^(c3 j3) w256^(c2 j3);  S3': j3 <- c3, conjugate
    for (int c2 = 0; c2 < 32; ++c2) {
        std::vector<std::complex<double>> G(64), Gi(64);
        for (int c3 = 0; c3 < 8; ++c3)
            for (int j3 = 0; j3 < 8; ++j3) {
                const std::complex<double> gv = wpow((long long)c3 * j3, 8, -1) * wpow((long long)c2 * j3, 256, -1) * r8;
                G[c3 * 8 + j3] = gv;
                Gi[j3 * 8 + c3] = std::conj(gv);
            }
        put_complex_matrix(img, off(kOffBS3) + c2 * 512, 8, 8, G);
        put_complex_matrix(img, off(kOffBS3i) + c2 * 512, 8, 8, Gi);
    }
    // S2': l <- c2
    F.assign(32 * 32, 0);
    for (int l = 0; l < 32; ++l) for (int c = 0; c < 32; ++c) F[l * 32 + c] = wpow((long long)c * l, 32, +1) * r32;
    put_complex_matrix(img, off(kOffBS2i), 32, 32, F);
    // S1': j1 <- c1 (j1 < 16)
    F.assign(16 * 32, 0);
    for (int j = 0; j < 16; ++j) for (int c = 0; c < 32; ++c) F[j * 32 + c] = wpow((long long)c * j, 32, +1) * r32;
    put_complex_matrix(img, off(kOffBS1i), 16, 32, F);
    return img;
}

std::vector<float2> twiddle_table(int n, int count) {
    std::vector<float2> t(count);
    for (int e = 0; e < count; ++e) {
        const std::complex<double> z = wpow(e, n, -1);
        t[e] = make_float2((float)z.real(), (float)z.imag());
    }
    return t;
}

__global__ void tc_export_kernel(const float2* __restrict__ Kf, float* __restrict__ out, int64_t H) {
    const int64_t total = H * (kN + 1);
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t h = i / (kN + 1), f = i % (kN + 1);
        const int64_t c1 = f & 31, c2 = (f >> 5) & 31, c3 = f >> 10;
        const float2 z = Kf[h * kM + (c2 * 8 + c3) * 32 + c1];
        out[2 * i] = z.x;
        out[2 * i + 1] = z.y;
    }
}

}  // namespace

bool tc_supported(int64_t N, int64_t /*L*/, int dtype) {
    return N == kN && (dtype == kF16 || dtype == kBF16);
}

cudaError_t tc_plan_init(Plan& p) {
    TcResources* r = new TcResources();
    p.tc = r;
    const std::vector<uint8_t> img = build_bimage();
    cudaError_t e = cudaMalloc((void**)&r->bimg, img.size());
    if (e == cudaSuccess) e = cudaMemcpy(r->bimg, img.data(), img.size(), cudaMemcpyHostToDevice);
    const std::vector<float2> t1 = twiddle_table(1024, 1024), t2 = twiddle_table(kM, 256);
    if (e == cudaSuccess) e = cudaMalloc((void**)&r->tw1024, t1.size() * sizeof(float2));
    if (e == cudaSuccess) e = cudaMemcpy(r->tw1024, t1.data(), t1.size() * sizeof(float2), cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMalloc((void**)&r->twM, t2.size() * sizeof(float2));
    if (e == cudaSuccess) e = cudaMemcpy(r->twM, t2.data(), t2.size() * sizeof(float2), cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&r->num_sms, cudaDevAttrMultiProcessorCount, p.device);
    // the SIMT engine computes the filter spectrum (any length), so the plan
    // also carries its twiddle table
    p.logTab = p.logM;
    if (e == cudaSuccess) {
        std::vector<float2> tw(p.M);
        for (int64_t i = 0; i < p.M; ++i) {
            const std::complex<double> z = wpow(i, p.M, -1);
            tw[i] = make_float2((float)z.real(), (float)z.imag());
        }
        e = cudaMalloc((void**)&p.tw, tw.size() * sizeof(float2));
        if (e == cudaSuccess) e = cudaMemcpy(p.tw, tw.data(), tw.size() * sizeof(float2), cudaMemcpyHostToDevice);
    }
    if (e == cudaSuccess) {
        e = cudaFuncSetAttribute(tc_fftconv_n4096_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kSmemBytes);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(tc_fftconv_n4096_kernel<__half>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kSmemBytes);
    }
    return e;
}

void tc_plan_free(Plan& p) {
    TcResources* r = (TcResources*)p.tc;
    if (!r) return;
    cudaFree(r->bimg);
    cudaFree(r->tw1024);
    cudaFree(r->twM);
    delete r;
    p.tc = nullptr;
}

size_t tc_filter_bytes(const Plan& p) { return (size_t)p.H * kM * sizeof(float2); }

cudaError_t tc_precompute(const Plan& p, const void* k, void* Kf, cudaStream_t s) {
    return simt_precompute_to_tc_layout(p, k, Kf, s);
}

cudaError_t tc_forward(const Plan& p, const ForwardArgs& fa, cudaStream_t s) {
    const TcResources* r = (const TcResources*)p.tc;
    TcArgs a{};
    a.u = fa.u; a.w = fa.w; a.v = fa.v; a.y = fa.y;
    a.Kf = (const float2*)fa.Kf;
    a.mask = fa.mask; a.mask_h = fa.mask_h;
    a.B = fa.B; a.H = p.H;
    a.npairs = p.H * ((fa.B + 1) / 2);
    a.nunits = (a.npairs + 3) / 4;
    a.bimg = (const uint4*)r->bimg;
    a.tw1024 = r->tw1024;
    a.twM = r->twM;
    a.status = p.status;
    const int64_t grid = a.nunits < r->num_sms ? a.nunits : r->num_sms;
    if (p.dtype == kBF16)
        tc_fftconv_n4096_kernel<__nv_bfloat16><<<(unsigned)grid, kThreads, kSmemBytes, s>>>(a);
    else
        tc_fftconv_n4096_kernel<__half><<<(unsigned)grid, kThreads, kSmemBytes, s>>>(a);
    return cudaGetLastError();
}

cudaError_t tc_export_rfft(const Plan& p, const void* Kf, float* out, cudaStream_t s) {
    const int64_t total = p.H * (kN + 1);
    int blocks = (int)((total + 255) / 256);
    if (blocks > 65535) blocks = 65535;
    tc_export_kernel<<<blocks, 256, 0, s>>>((const float2*)Kf, out, p.H);
    return cudaGetLastError();
}

}  // namespace fftconv
