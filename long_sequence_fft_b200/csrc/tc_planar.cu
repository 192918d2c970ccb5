// tc_planar.cu -- tensor-core (tcgen05) fused FFT convolution with planar
// complex data, sm_100a: sequences of 4096 (one zero-padded 8192-point
// transform per sequence; shorter ones packed several to a transform),
// sequences of 8192 and 16384 as two and four blocks of 4096 (a
// block-partitioned convolution: block b's output is sum_{j <= b} X_j G_{b-j}
// in the 8192-point domain), and longer sequences with filters of at most
// 2049 taps (overlap-save windows of 4096 inputs, hop 2048).
//
// FlashFFTConv: Efficient Convolutions for Long Sequences with Tensor Cores,
// "Approach": the FFT convolution as an order-p Monarch decomposition --
// matrix products with small DFT factors along one digit of the index, so
// the transform runs on tensor cores, permutations become on-chip
// transposes, and the whole convolution (gates included, "Key results") is
// one kernel.
//
// The transform and the tiling are those of tc_kernels.cu (8192 = 32 x 32 x
// 8, a CTA tile = 4 pairs of batch rows of one channel, pair q in TMEM lanes
// [32q, 32q+32), six tcgen05.mma stages S1, S2, S3, S3', S2', S1' with a ring
// of four 64-column fp32 accumulator buffers, four MMA issuer warps and
// sixteen epilogue warps).  What differs is how complex numbers are laid out:
//
//   - "pair-planar" (PP): the values of a complex vector are taken two at a
//     time; the real parts of values 2p and 2p+1 share one 32-bit word
//     (fp16 pair) and their imaginary parts the next word.  A half2
//     instruction then applies a twiddle or the filter to two values at
//     once, with no shuffling of real and imaginary halves (a complex
//     product of two values costs four half2 instructions);
//   - "planar" (PL): all real parts, then all imaginary parts.
//
// The DFT factors are stored as real 2n x 2n matrices whose row (K) and
// column (N) orders follow the operand layouts below, so the MMAs read and
// write these layouts directly.  Every accumulator's column order is PP.
//
//   operand              where             K order          written by
//   S1  A1               TMEM              PP(j1)           load (u*w)
//   S2  A2  (MN-major)   shared, 128B sw.  PL(l)            E1: 16-byte stores
//   S3  A3               TMEM              PP(j3)           E2
//   S3' A4               TMEM              PP(c3)           EK (filter product)
//   S2' A5  (K-major)    shared, 128B sw.  PP(c2)           E3': 16-byte stores
//   S1' A6  (MN-major)   shared, 128B sw.  PL(c1)           E2': 16-byte stores
//
// The two stages that contract the TMEM lane digit (S2: l, S1': c1) read an
// MN-major ("transposed") shared-memory operand: the epilogue thread that
// holds one lane's values for consecutive output indices writes them as
// consecutive rows of the next operand -- the on-chip transpose is a plain
// 16-byte vector store.  Every wait is bounded: on timeout the kernel records
// FFTCONV_ERR_TIMEOUT in the plan's status word, drains, frees its TMEM and
// returns.
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

cudaError_t simt_precompute_to_tc_pp(const Plan& p, const void* k, void* Kf, cudaStream_t s);
cudaError_t simt_precompute_to_tc_pp2(const Plan& p, const void* k, void* Kf, const float2* tw8192, cudaStream_t s);
cudaError_t simt_precompute_to_tc_pp4(const Plan& p, const void* k, void* Kf, const float2* tw8192, cudaStream_t s);

namespace {

using namespace tc;

constexpr int kN = 4096;          // window length (inputs and outputs per transform)
constexpr int kM = 8192;          // transform length
constexpr int kHop = 2048;        // overlap-save hop for longer sequences
constexpr int kEpiWarps = 16;
constexpr int kMmaWarps = 4;
constexpr int kThreads = (kEpiWarps + kMmaWarps) * 32;
constexpr int kDBuf = 4;
constexpr int kChunks = 44;       // 8 per stage S1..S2', 4 for S1'
constexpr uint32_t kWaitLimit = 1u << 20;

// shared memory (bytes from a 1024-aligned base)
constexpr int kTile = 16384;                  // one data tile: 128 rows x 64 fp16
constexpr int OffData = 0;                    // 8 tiles (one per j3)
constexpr int OffBS1 = 8 * kTile;             // K=32  N=64   4 KB
constexpr int OffBS2 = OffBS1 + 4096;         // K=64  N=64   8 KB
constexpr int OffBS3 = OffBS2 + 8192;         // 32 x (K=16 N=16)  16 KB
constexpr int OffBS3i = OffBS3 + 16384;       // 32 x (K=16 N=16)  16 KB
constexpr int OffBS2i = OffBS3i + 16384;      // K=64  N=64   8 KB
constexpr int OffBS1i = OffBS2i + 8192;       // K=64  N=32   4 KB
constexpr int OffBEnd = OffBS1i + 4096;
constexpr int BImageBytes = OffBEnd - OffBS1;
constexpr int kKBytes = kM * 4;               // one filter spectrum row, 8192 complex fp16
constexpr int OffK = OffBEnd;
constexpr int OffTw = OffK + kKBytes;         // w8192^e, e < 256, as half2
constexpr int OffBars = OffTw + 1024;
constexpr int OffXBars = OffBars + 128;       // block-mode hand-over barriers [4 steps][4 slices][<= 3]
constexpr int OffMisc = OffXBars + 512;
constexpr int SmemBytes = OffMisc + 64 + 1024;   // + alignment slack
static_assert(SmemBytes <= 232448, "shared memory");

// chunk c of a tile -> stage (0 S1, 1 S2, 2 S3, 3 S3', 4 S2', 5 S1') and index
__host__ __device__ __forceinline__ int chunk_stage(int c) { return c < 40 ? (c >> 3) : 5; }
__host__ __device__ __forceinline__ int chunk_index(int c) { return c < 40 ? (c & 7) : c - 40; }
// Chunks that need a whole earlier stage (not just the chunks that the
// accumulator ring already orders before them): the first S3 chunks need
// all of E2, the first S2' chunks all of E3', the last S1' chunk the last E2'
// pair.
__host__ __device__ __forceinline__ int chunk_stage_barrier(int c) {
    if (c >= 16 && c < 20) return 0;
    if (c >= 32 && c < 36) return 1;
    if (c == 43) return 2;
    return -1;
}

// Monarch mode: bit m of empty_groups(keep) is set when the eight c2 of group m
// (8m .. 8m + 7) are all masked; the S3 and S3' chunk pairs of such a group
// (chunks 16 + 2m, 17 + 2m and 24 + 2m, 25 + 2m) are not run.  The ring runs
// over the remaining chunks in order: chunk c takes slot chunk_slot(c) of the
// tile's 44 - 4 popc(empty) slots, whose buffer is slot % 4.
__host__ __device__ __forceinline__ uint32_t empty_groups(uint32_t keep) {
    uint32_t e = 0;
    for (int m = 0; m < 4; ++m)
        if (((keep >> (8 * m)) & 0xffu) == 0) e |= 1u << m;
    return e;
}
__host__ __device__ __forceinline__ int popc4(uint32_t x) { return (x & 1) + ((x >> 1) & 1) + ((x >> 2) & 1) + ((x >> 3) & 1); }
__host__ __device__ __forceinline__ bool chunk_skipped(int c, uint32_t empty) {
    return c >= 16 && c < 32 && ((empty >> (((c - 16) & 7) >> 1)) & 1u);
}
__host__ __device__ __forceinline__ int chunk_slot(int c, uint32_t empty) {
    if (c < 16) return c;
    if (c < 24) return c - 2 * popc4(empty & ((1u << ((c - 16) >> 1)) - 1u));
    if (c < 32) return c - 2 * popc4(empty) - 2 * popc4(empty & ((1u << ((c - 24) >> 1)) - 1u));
    return c - 4 * popc4(empty);
}

// fp16 element index of the real (comp 0) or imaginary (comp 1) part of
// value i in pair-planar and planar order (n values)
__host__ __device__ constexpr int pp_index(int comp, int i) { return 4 * (i >> 1) + 2 * comp + (i & 1); }
__host__ __device__ constexpr int pl_index(int comp, int i, int n) { return comp * n + i; }

// byte offset of element (n, k) of a K x N B operand, K-major, no swizzle:
// 8x8 core matrices, K-groups of 8 LBO = (N/8)*128 bytes apart
inline size_t bimg_offset(int n, int k, int N) {
    return (size_t)(k / 8) * (N / 8) * 128 + (size_t)(n / 8) * 128 + (n % 8) * 16 + (k % 8) * 2;
}

// 128-byte swizzle of a byte offset (1024-byte aligned atoms)
__device__ __forceinline__ uint32_t swz(uint32_t off) { return off ^ (((off >> 7) & 7u) << 4); }
// MN-major operand tile, 128-byte swizzle: element (m, k) of 128 x 64; the
// two 64-row halves 8192 bytes apart (LBO), the K-groups of 8 1024 bytes
// apart (SBO)
__device__ __forceinline__ uint32_t mn_off(int m, int k) {
    return swz((uint32_t)((m >> 6) * 8192 + (k >> 3) * 1024 + (k & 7) * 128 + (m & 63) * 2));
}
// K-major operand tile, 128-byte swizzle: row m holds K = 64 fp16 (128 bytes)
__device__ __forceinline__ uint32_t k_off(int m, int kbyte) {
    return swz((uint32_t)((m >> 3) * 1024 + (m & 7) * 128 + kbyte));
}

// kernel modes: one transform per row (N <= 4096, packed below), overlap-save
// windows (N >= 16384, filters of at most 2049 taps), two blocks (N = 8192),
// and the plain mode with a Monarch-aligned frequency mask (N = 4096)
constexpr int kPlain = kPlanarPlain, kWin = kPlanarWindows, kTwo = kPlanarTwoBlock, kMonarch = kPlanarMonarch;
constexpr int kFour = 4;          // the block mode with four blocks (N = 16384)
// block modes: P blocks of 4096 per pair, quarter q = block q >> kShift of
// pair q & ((1 << kShift) - 1)
template <int MODE>
struct Blocks {
    static constexpr bool on = MODE == kTwo || MODE == kFour;
    static constexpr int P = MODE == kFour ? 4 : 2;
    static constexpr int kShift = MODE == kFour ? 0 : 1;
};

struct PArgs {
    const void* u;
    const void* w;
    const void* v;
    void* y;
    const uint32_t* K;          // [H][kstride] words: the spectrum / scale, PP layout (k_word)
    int64_t kstride;            // words per channel: 8192, or 8192 P (block modes: G_0 .. G_{P-1})
    int g1_from_g0;             // two blocks, L <= 4096: G_1 = (-1)^f G_0 (not read)
    int ng;                     // block mode: filter rows G_d that are not zero (d < ng)
    uint32_t keep_c2;           // Monarch mode: bit c2 keeps the bins with that middle digit
    const float* Kscale;        // [H]
    const uint8_t* mask;
    int64_t mask_h;
    int64_t B, H, N;
    int64_t nwin;               // windows per sequence (1 for N <= 4096)
    int lseg;                   // log2(N / 256) for N <= 4096: 4096 / N sequences share a transform
    int64_t pb;                 // pairs per channel, ceil(B/2)
    int64_t tpc;                // tiles per window, ceil(pb/4)
    int64_t nunits;             // H * nwin * tpc
    const uint4* bimg;          // DFT factor images
    const uint32_t* tw1024;     // exp(-2 pi i e/1024) as half2, e < 1024
    const uint32_t* tw8192;     // exp(-2 pi i e/8192) as half2, e < 256
    int* status;
    // backward (correlation) launches: a second output y2 = s_h v2 z beside
    // y = s_h v z (y2 may be NULL)
    void* y2;
    const void* v2;
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

__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u2h(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }
// two fp32 accumulator values (as raw bits) -> one fp16 pair
__device__ __forceinline__ uint32_t pk(uint32_t a, uint32_t b) {
    return h2u(__floats2half2_rn(__uint_as_float(a), __uint_as_float(b)));
}
__device__ __forceinline__ uint32_t pkf(float a, float b) { return h2u(__floats2half2_rn(a, b)); }

// (xr + i xi) (tr + i ti) for two values at once: xr, xi, tr, ti are the PP
// words (fp16 pairs) of the real and imaginary parts
__device__ __forceinline__ void cmul_pp(uint32_t& xr, uint32_t& xi, uint32_t tr, uint32_t ti) {
    const __half2 a = u2h(xr), b = u2h(xi), c = u2h(tr), d = u2h(ti);
    xr = h2u(__hfma2(__hneg2(b), d, __hmul2(a, c)));
    xi = h2u(__hfma2(b, c, __hmul2(a, d)));
}
// (yr + i yi) += (xr + i xi) (tr + i ti), two values at once (PP words)
__device__ __forceinline__ void cfma_pp(uint32_t& yr, uint32_t& yi, uint32_t xr, uint32_t xi, uint32_t tr,
                                        uint32_t ti) {
    const __half2 a = u2h(xr), b = u2h(xi), c = u2h(tr), d = u2h(ti);
    yr = h2u(__hfma2(__hneg2(b), d, __hfma2(a, c, u2h(yr))));
    yi = h2u(__hfma2(b, c, __hfma2(a, d, u2h(yi))));
}
constexpr uint32_t kNegPair = 0x80008000u;   // sign bits of both halves

// Block-mode hand-over slots of EK step st (byte offsets from the data
// tiles): the bytes that E3' writes in the same step (K bytes [32 st,
// 32 st + 32) of every row of every tile), 64 slots of 16 bytes per lane,
// consecutive lanes on consecutive rows so that a warp's 16-byte accesses hit
// distinct banks.  Slot z = (s np + i) 4 + piece: piece < 4 of the values of
// the giving warp i (of np per slice) of slice s; with two blocks, slot
// 32 + (2 s + pq) 4 + piece: the G_1 words the block-1 warp of pair pq reads.
__device__ __forceinline__ uint32_t xoff(int st, int z, int lane) {
    return (uint32_t)((z >> 3) * kTile) + k_off(32 * (z & 3) + lane, 32 * st + 16 * ((z >> 2) & 1));
}

// word index of the filter spectrum value f = c1 + 32 c2 + 1024 c3 (its real
// part; the imaginary part is the next word), and which half: 16-byte groups
// of four c3 values (two PP pairs), consecutive c1 in consecutive groups, so
// a warp (c1 = lane) reads 512 contiguous bytes per (c2, c3 half)
__host__ __device__ __forceinline__ int k_word(int c1, int c2, int c3) {
    return ((c2 * 2 + (c3 >> 2)) * 32 + c1) * 4 + 2 * ((c3 & 3) >> 1);
}

struct PairInfo {
    int64_t o0, o1;      // element offsets of the window in rows b0 and b1 (o1 < 0: absent)
    bool valid;
    bool tail_only;      // only window positions t >= kHop are outputs
};

// A tile holds 4 transform rows of one channel and one window; each row is
// the complex sequence of a pair of batch rows (the two real sequences are its
// real and imaginary parts).  Sequences of N = 4096: unit u covers channel
// u / (nwin*tpc), window j = (u / tpc) % nwin and pairs 4*(u % tpc) + q,
// q < 4 (pairs past ceil(B/2) are empty); window j starts at 2048 j; window
// 0 keeps all 4096 outputs, window j > 0 keeps positions [2048, 4096) (the
// overlap-save rule: its transform is exact from window position L - 1 on,
// and L <= 2049).
// Shorter sequences (N = 256 .. 2048) are packed: transform row q holds the
// S = 4096 / N pairs q S + sigma (sigma < S) at positions [2N sigma,
// 2N sigma + N), each followed by N zeros, so a tile covers 4 S pairs.  The
// 8192-point circular convolution of such a row is the causal convolution of
// each pair, exactly: a filter of at most N taps reaches back at most N - 1
// positions, into that pair's own zeros (or, for sigma = 0, around the end
// of the row into the last pair's zeros).
// Sequences of 8192 and 16384 (block modes, P = N / 4096 blocks): a tile
// holds 4 / P pairs; transform row q is block b = q >> log2(4 / P) (inputs
// and outputs [4096 b, 4096 b + 4096)) of the tile's pair q mod (4 / P),
// zero-padded to 8192 points.
struct TileBase {
    int64_t h, bp0, j;   // channel, first pair of the tile, window
};
template <int MODE>
__device__ __forceinline__ TileBase tile_base(const PArgs& a, int64_t unit) {
    TileBase t;
    if constexpr (MODE == kPlain || MODE == kMonarch) {
        t.h = unit / a.tpc;
        t.j = 0;
        t.bp0 = (unit - t.h * a.tpc) * (64 >> a.lseg);
    } else if constexpr (Blocks<MODE>::on) {
        t.h = unit / a.tpc;
        t.j = 0;
        t.bp0 = (unit - t.h * a.tpc) << Blocks<MODE>::kShift;
    } else {
        const uint32_t un = (uint32_t)unit, tpc = (uint32_t)a.tpc, per_ch = (uint32_t)a.nwin * tpc;
        const uint32_t hh = un / per_ch, rem = un - hh * per_ch, jj = rem / tpc;
        t.h = hh;
        t.j = jj;
        t.bp0 = 4 * (int64_t)(rem - jj * tpc);
    }
    return t;
}
// rows of transform row q, segment sigma of a tile
template <int MODE>
__device__ __forceinline__ PairInfo pair_rows(const PArgs& a, const TileBase& t, int q, int sigma) {
    PairInfo p;
    const int64_t bp = Blocks<MODE>::on ? t.bp0 + (q & ((1 << Blocks<MODE>::kShift) - 1))
                                        : t.bp0 + ((int64_t)q << (4 - a.lseg)) + sigma;
    p.valid = bp < a.pb;
    p.tail_only = t.j > 0;
    const int64_t b0 = 2 * (p.valid ? bp : 0), b1 = b0 + 1;
    const int64_t base = MODE == kWin ? kHop * t.j : (Blocks<MODE>::on ? (int64_t)kN * (q >> Blocks<MODE>::kShift) : 0);
    p.o0 = (b0 * a.H + t.h) * a.N + base;
    p.o1 = (p.valid && b1 < a.B) ? (b1 * a.H + t.h) * a.N + base : -1;
    return p;
}
// kept stage-1 index i (< 16) -> its segment and the position of its first
// element in the segment: j1 = the i-th digit with (j1 mod 2^(lseg+1)) <
// 2^lseg, t = 256 j1 + 8 l + j3
__device__ __forceinline__ int seg_of(const PArgs& a, int i) { return i >> a.lseg; }
__device__ __forceinline__ int tau_of(const PArgs& a, int i) { return 256 * (i & ((1 << a.lseg) - 1)); }

template <int MODE>
__device__ __forceinline__ int64_t unit_channel(const PArgs& a, int64_t u) {
    if constexpr (MODE == kWin) return (int64_t)((uint32_t)u / ((uint32_t)a.nwin * (uint32_t)a.tpc));
    return u / a.tpc;
}

// BWD: the correlation of the backward pass -- the product with conj(K)
// instead of K (the filter is real, so that is correlation with k) and the
// second output y2.  UNGATED: the forward build for calls without the input
// gate w (no gate loads, normal L2 policy for u).  Against the gated build
// given w = NULL it measured 6% faster on plain and packed sequences, 5% on
// two blocks and 1-3% on four.
template <typename T, int MODE, bool BWD = false, bool UNGATED = false>
__global__ void __launch_bounds__(kThreads, 1) tc_fftconv_planar_kernel(PArgs a) {
    static_assert(!BWD || MODE == kPlain || MODE == kTwo, "the correlation pass runs on plain and two-block plans");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t* bar = (uint64_t*)(smem + OffBars);
    uint64_t* bar_in = bar + 0;    // the tile's input is in TMEM (16 epilogue warps)
    uint64_t* dfull = bar + 1;     // [kDBuf] accumulator buffer written (tcgen05.commit)
    uint64_t* dfree = bar + 5;     // [kDBuf] accumulator buffer drained (16 epilogue warps)
    uint64_t* bar_fin = bar + 9;   // every MMA has completed (drain before exit)
    uint64_t* bar_k = bar + 10;    // the tile's filter row has landed in shared memory
    uint64_t* bar_stage = bar + 11;   // [3] E2, E3', E2' done for the tile (16 epilogue warps)
    // block modes: [EK step][slice][giving warp] that warp's spectrum values
    // are in the hand-over slots (its 32 threads)
    uint64_t* xfull = (uint64_t*)(smem + OffXBars);
    // Monarch mode (same space): [4] the EK of c2 group m is done (16 epilogue warps)
    uint64_t* ek_done = (uint64_t*)(smem + OffXBars);
    uint32_t* tmem_base_sh = (uint32_t*)(smem + OffMisc);
    volatile int* abort_flag = (volatile int*)(smem + OffMisc + 4);

    const int tid = threadIdx.x;
    // the warp index through a shuffle, so the compiler knows it is the same
    // for all lanes: everything derived from it (TMEM and shared-memory
    // addresses, descriptors) stays in uniform registers
    const int warp = __shfl_sync(0xffffffffu, tid >> 5, 0);
    const int lane = tid & 31;
    const uint32_t sbase = smem_u32(smem);

    if (tid == 0) {
        mbar_init(bar_in, kEpiWarps);
        for (int i = 0; i < kDBuf; ++i) {
            mbar_init(&dfull[i], 1);
            mbar_init(&dfree[i], kEpiWarps);
        }
        mbar_init(bar_fin, kMmaWarps);
        mbar_init(bar_k, 1);
        for (int i = 0; i < 3; ++i) mbar_init(&bar_stage[i], kEpiWarps);
        if constexpr (Blocks<MODE>::on)
            for (int i = 0; i < 48; ++i) mbar_init(&xfull[i], 32);
        if constexpr (MODE == kMonarch)
            for (int i = 0; i < 4; ++i) mbar_init(&ek_done[i], kEpiWarps);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kEpiWarps) tmem_alloc(tmem_base_sh, 512);   // the first MMA warp owns TMEM
    {
        uint4* dst = (uint4*)(smem + OffBS1);
        for (int i = tid; i < BImageBytes / 16; i += kThreads) dst[i] = __ldg(&a.bimg[i]);
        uint32_t* t = (uint32_t*)(smem + OffTw);
        for (int i = tid; i < 256; i += kThreads) t[i] = __ldg(&a.tw8192[i]);
    }
    const uint32_t* stw = (const uint32_t*)(smem + OffTw);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = __shfl_sync(0xffffffffu, *tmem_base_sh, 0);

    auto wait = [&](uint64_t* b, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, mbar_wait_bounded(b, parity, abort_flag, kWaitLimit));
    };
    auto fail = [&](void) {
        if (!*abort_flag) {
            *abort_flag = 1;
            atomicExch(a.status, kStatusTimeout);
        }
    };

    if (warp >= kEpiWarps) {
        // ============================ MMA issuers ===========================
        // issuer i handles the chunks c = i (mod 4) of every tile, which all
        // use accumulator buffer i
        const int issuer = warp - kEpiWarps;
        constexpr uint32_t kTransA = 1u << 15;        // A operand MN-major
        const uint32_t id64 = idesc_f16_f32(128, 64);
        const uint32_t id64t = id64 | kTransA;
        const uint32_t id16 = idesc_f16_f32(128, 16);
        const uint32_t id32t = idesc_f16_f32(128, 32) | kTransA;
        // B operands: K-major, no swizzle; K-groups (N/8)*128 bytes apart
        const uint64_t dS1 = make_desc(sbase + OffBS1, 1024, 128, 0);      // K step: +2048 B
        const uint64_t dS2 = make_desc(sbase + OffBS2, 1024, 128, 0);      // K step: +2048 B
        const uint64_t dS2i = make_desc(sbase + OffBS2i, 1024, 128, 0);
        const uint64_t dS3 = make_desc(sbase + OffBS3, 256, 128, 0);       // per c2: +512 B
        const uint64_t dS3i = make_desc(sbase + OffBS3i, 256, 128, 0);
        const uint64_t dS1i = make_desc(sbase + OffBS1i, 512, 128, 0);     // K step: +1024 B
        // A operands in shared memory: MN-major (S2, S1') and K-major (S2')
        const uint64_t dAmn = make_desc(sbase + OffData, 8192, 1024, 2);   // K step: +2048 B
        const uint64_t dAk = make_desc(sbase + OffData, 16, 1024, 2);      // K step: +32 B
        int iter = 0;
        int k_issued = 0;
        bool ok = true;
        uint32_t g = issuer;
        // Monarch mode: the S3 / S3' products of a masked c2 and the S2' K
        // steps whose eight c2 are all masked are not issued (their outputs
        // would be zero); a chunk with some kept c2 is still committed, a
        // chunk pair whose eight c2 are all masked is not run at all
        const uint32_t keep = MODE == kMonarch ? a.keep_c2 : 0xffffffffu;
        const uint32_t empty = MODE == kMonarch ? empty_groups(keep) : 0u;
        // the chunks this issuer runs (Monarch mode: the slot decides; the same every tile)
        uint64_t mine = 0;
        for (int c = 0; c < kChunks; ++c)
            if (!chunk_skipped(c, empty) && (chunk_slot(c, empty) & 3) == issuer) mine |= 1ull << c;
        for (int64_t unit = blockIdx.x; unit < a.nunits && ok; unit += gridDim.x, ++iter) {
            if (!wait(bar_in, iter & 1)) { ok = false; fail(); break; }
            tc_fence_after();
            if (issuer == 0) {
                if (lane == 0) {
                    // the previous tile is finished with the filter buffer (its
                    // epilogue warps arrived on bar_in after all their reads)
                    mbar_expect_tx(bar_k, kKBytes);
                    bulk_copy_g2s(smem + OffK, a.K + unit_channel<MODE>(a, unit) * a.kstride, kKBytes, bar_k);
                }
                ++k_issued;
                __syncwarp();
            }
#pragma unroll 1
            for (int c = MODE == kMonarch ? 0 : issuer; c < kChunks && ok; c += MODE == kMonarch ? 1 : kMmaWarps) {
                // (Monarch mode: this issuer runs the chunks whose slot is issuer mod 4)
                if (MODE == kMonarch && !((mine >> c) & 1ull)) continue;
                const int stage = chunk_stage(c), k = chunk_index(c);
                const uint32_t b = g % kDBuf;
                if (g >= kDBuf && !wait(&dfree[b], ((g - kDBuf) / kDBuf) & 1)) { ok = false; fail(); break; }
                g += kMmaWarps;
                int sb = chunk_stage_barrier(c);
                if (MODE == kMonarch && stage == 2) sb = 0;      // every S3 chunk after all of E2
                if (sb >= 0 && !wait(&bar_stage[sb], iter & 1)) { ok = false; fail(); break; }
                // Monarch mode: an S3' chunk after the EK of its c2 group (with
                // chunks skipped, the ring no longer orders the two)
                if (MODE == kMonarch && stage == 3 && !wait(&ek_done[k >> 1], iter & 1)) {
                    ok = false;
                    fail();
                    break;
                }
                tc_fence_after();
                {
                    // the whole warp evaluates the operands; one elected lane issues
                    const uint32_t d = tbase + 256 + 64 * b;
                    if (stage == 0) {            // S1: A1 cols 16 j3 + (PP j1), j3 = k
#pragma unroll
                        for (int ks = 0; ks < 2; ++ks)
                            mma_ts_warp(d, tbase + 16 * k + 8 * ks, dS1 + 128 * ks, id64, ks);
                    } else if (stage == 1) {     // S2: MN-major tile j3 = k
                        const uint64_t da = dAmn + (uint64_t)(k * (kTile >> 4));
#pragma unroll
                        for (int s = 0; s < 4; ++s) mma_ss_warp(d, da + 128 * s, dS2 + 128 * s, id64t, s);
                    } else if (stage == 2 || stage == 3) {   // S3 / S3': c2 = 4k + cl, A cols 8 c2
                        const uint64_t db = (stage == 2 ? dS3 : dS3i) + (uint64_t)(4 * k * 32);
#pragma unroll
                        for (int cl = 0; cl < 4; ++cl)
                            if ((keep >> (4 * k + cl)) & 1u)
                                mma_ts_warp(d + 16 * cl, tbase + 8 * (4 * k + cl), db + 32 * cl, id16, 0);
                    } else if (stage == 4) {     // S2': K-major tile j3 = k, K step s = c2 8s .. 8s + 7
                        const uint64_t da = dAk + (uint64_t)(k * (kTile >> 4));
                        uint32_t acc = 0;
#pragma unroll
                        for (int s = 0; s < 4; ++s)
                            if ((keep >> (8 * s)) & 0xffu) {
                                mma_ss_warp(d, da + 2 * s, dS2i + 128 * s, id64, acc);
                                acc = 1;
                            }
                    } else {                     // S1': j3 = 2k + jl, MN-major tiles, N = 32 (16 kept j1)
#pragma unroll
                        for (int jl = 0; jl < 2; ++jl) {
                            const uint64_t da = dAmn + (uint64_t)((2 * k + jl) * (kTile >> 4));
#pragma unroll
                            for (int s = 0; s < 4; ++s) mma_ss_warp(d + 32 * jl, da + 128 * s, dS1i + 64 * s, id32t, s);
                        }
                    }
                    tc_commit_warp(&dfull[b]);
                }
                __syncwarp();
                if (c == issuer + 12) {
                    // warm L2 with the next tile's rows (u, w, v of both
                    // sequences of each pair, and the filter spectrum): issuer i
                    // takes pair i
                    const void* pf_src = nullptr;
                    uint32_t pf_bytes = (uint32_t)(a.N < kN ? a.N : kN) * sizeof(T);
                    const int64_t nu = unit + gridDim.x;
                    // (packed short sequences: the row's first segments only)
                    if (nu < a.nunits && (lane >> 3) < (16 >> a.lseg)) {
                        const TileBase tb = tile_base<MODE>(a, nu);
                        const int64_t hn = tb.h;
                        const PairInfo Q = pair_rows<MODE>(a, tb, issuer, lane >> 3);
                        const int which = lane & 7;
                        if (Q.valid) {
                            if (which == 0) pf_src = (const T*)a.u + Q.o0;
                            else if (which == 1 && a.w) pf_src = (const T*)a.w + Q.o0;
                            else if (which == 2 && a.v) pf_src = (const T*)a.v + Q.o0;
                            else if (which == 3 && Q.o1 >= 0) pf_src = (const T*)a.u + Q.o1;
                            else if (which == 4 && Q.o1 >= 0 && a.w) pf_src = (const T*)a.w + Q.o1;
                            else if (which == 5 && Q.o1 >= 0 && a.v) pf_src = (const T*)a.v + Q.o1;
                            else if (which == 6 && issuer == 0 && (lane >> 3) == 0) {
                                pf_src = a.K + hn * a.kstride;
                                pf_bytes = kKBytes;
                            } else if (Blocks<MODE>::on && which == 7 && issuer >= 1 && issuer < a.ng &&
                                       (lane >> 3) == 0 && !a.g1_from_g0) {
                                pf_src = a.K + hn * a.kstride + issuer * kM;    // G_issuer (block modes)
                                pf_bytes = kKBytes;
                            }
                        }
                    }
                    if (pf_src) prefetch_l2(pf_src, pf_bytes);
                    __syncwarp();
                }
            }
        }
        // drain: every issued MMA and the last filter copy must finish before
        // TMEM and shared memory are released -- bounded, and regardless of
        // an abort
        if (lane == 0) tc_commit(bar_fin);
        __syncwarp();
        bool drained = false;
        for (uint32_t i = 0; i < kWaitLimit && !drained; ++i) drained = mbar_try_wait(bar_fin, 0);
        if (!drained) fail();
        if (issuer == 0 && k_issued > 0) {
            drained = false;
            for (uint32_t i = 0; i < kWaitLimit && !drained; ++i) drained = mbar_try_wait(bar_k, (k_issued - 1) & 1);
            if (!drained) fail();
        }
        __syncwarp();
    } else {
        // ========================== epilogue warps ==========================
        const int q = warp & 3;          // lane quarter = pair within the tile
        const int s = warp >> 2;         // column slice
        const uint32_t lq = (uint32_t)(32 * q) << 16;
        const int64_t nblk = kN / 32;    // mask blocks (plain mode: N = 4096)

        // w1024^(x (8s + i)), x = lane, i < 8, as PP pairs over i: the E1
        // twiddle (x = l, c1 = 8s + i) and, conjugated, the E2' twiddle
        // (x = c1, l = 8s + i)
        uint32_t twr[4], twi[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const __half2 t0 = u2h(__ldg(&a.tw1024[(lane * (8 * s + 2 * p)) & 1023]));
            const __half2 t1 = u2h(__ldg(&a.tw1024[(lane * (8 * s + 2 * p + 1)) & 1023]));
            twr[p] = h2u(__lows2half2(t0, t1));
            twi[p] = h2u(__highs2half2(t0, t1));
        }

        // ---- load: x = u*w for t = 256 j1 + 8 l + j3 (l = lane), j1 the kept
        // stage-1 digits of index 2P and 2P+1 with P = 2s + part, into the TMEM
        // A1 columns 16 j3 + 2P (real pair) and 16 j3 + 2P + 1 (imaginary
        // pair: the pair's second row); part 1 then arrives on bar_in.  A
        // tile's input is loaded while the previous tile's last stages run
        // (the A columns are free once S3' is done).  Absent rows or gates read
        // a present row and are masked.
        struct LoadPart {
            uint4 ld[2][4];
            bool keep0[2], keep1[2];
        };
        auto load_issue = [&](int64_t lu, int part, LoadPart& lp) {
            const TileBase tb = tile_base<MODE>(a, lu);
            const bool has_w = !UNGATED && a.w != nullptr;
            const int P = 2 * s + part;
#pragma unroll
            for (int jh = 0; jh < 2; ++jh) {
                // kept stage-1 index 2P + jh: its segment's rows and position
                const int i = 2 * P + jh;
                const PairInfo LP = pair_rows<MODE>(a, tb, q, seg_of(a, i));
                const bool hasL = LP.o1 >= 0;
                lp.keep0[jh] = LP.valid;
                lp.keep1[jh] = hasL;
                const int64_t oo1 = hasL ? LP.o1 : LP.o0;
                const int64_t t0 = tau_of(a, i) + 8 * lane;
                const T* pu0 = (const T*)a.u + LP.o0;
                const T* pu1 = (const T*)a.u + oo1;
                // read once: evict-first leaves L2 to the prefetched next rows
                // (measured 1.3% faster on the flagship); overlap-save windows
                // re-read half of each window and the four-block mode measured
                // slower with it: normal policy there
                const uint64_t pol =
                    (MODE == kWin || MODE == kFour || UNGATED) ? l2_evict_normal() : l2_evict_first();
                lp.ld[jh][0] = ldg_nc_hint(pu0 + t0, pol);
                lp.ld[jh][2] = ldg_nc_hint(pu1 + t0, pol);
                if constexpr (UNGATED) {
                    lp.ld[jh][1] = lp.ld[jh][3] = make_uint4(0u, 0u, 0u, 0u);
                } else {
                    lp.ld[jh][1] = ldg_nc_hint((has_w ? (const T*)a.w + LP.o0 : pu0) + t0, pol);
                    lp.ld[jh][3] = ldg_nc_hint((has_w ? (const T*)a.w + oo1 : pu1) + t0, pol);
                }
            }
        };
        auto load_finish = [&](int part, const LoadPart& lp) {
            const bool has_w = !UNGATED && a.w != nullptr;
            const int P = 2 * s + part;
            float xa[2][8], xb[2][8];
#pragma unroll
            for (int jh = 0; jh < 2; ++jh) {
                const uint32_t ua[4] = {lp.ld[jh][0].x, lp.ld[jh][0].y, lp.ld[jh][0].z, lp.ld[jh][0].w};
                const uint32_t wa[4] = {lp.ld[jh][1].x, lp.ld[jh][1].y, lp.ld[jh][1].z, lp.ld[jh][1].w};
                const uint32_t ub[4] = {lp.ld[jh][2].x, lp.ld[jh][2].y, lp.ld[jh][2].z, lp.ld[jh][2].w};
                const uint32_t wb[4] = {lp.ld[jh][3].x, lp.ld[jh][3].y, lp.ld[jh][3].z, lp.ld[jh][3].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float2 p0 = IO<T>::unpack2(ua[e]), p1 = IO<T>::unpack2(ub[e]);
                    if (has_w) {
                        const float2 g0 = IO<T>::unpack2(wa[e]), g1 = IO<T>::unpack2(wb[e]);
                        p0.x *= g0.x; p0.y *= g0.y; p1.x *= g1.x; p1.y *= g1.y;
                    }
                    if (!lp.keep0[jh]) p0 = make_float2(0.f, 0.f);
                    if (!lp.keep1[jh]) p1 = make_float2(0.f, 0.f);
                    xa[jh][2 * e] = p0.x; xa[jh][2 * e + 1] = p0.y;
                    xb[jh][2 * e] = p1.x; xb[jh][2 * e + 1] = p1.y;
                }
            }
#pragma unroll
            for (int j3 = 0; j3 < 8; ++j3)
                tmem_st2(tbase + lq + 16 * j3 + 2 * P, pkf(xa[0][j3], xa[1][j3]), pkf(xb[0][j3], xb[1][j3]));
            if (part == 1) {
                tc_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_in);
            }
        };
        auto load_tile = [&](int64_t lu, int part) {
            LoadPart lp;
            load_issue(lu, part, lp);
            load_finish(part, lp);
        };

        int iter = 0;
        bool ok = true;
        float nf = 0.f;          // non-finite detector over the outputs (fp16 range)
        if ((int64_t)blockIdx.x < a.nunits) {
            load_tile(blockIdx.x, 0);
            load_tile(blockIdx.x, 1);
        }
        for (int64_t unit = blockIdx.x; unit < a.nunits && ok; unit += gridDim.x, ++iter) {
            const TileBase TB = tile_base<MODE>(a, unit);
            const int64_t hch = TB.h;
            const uint32_t* Ks = (const uint32_t*)(smem + OffK);
            float kscale = __ldg(&a.Kscale[hch]);
            asm volatile("mov.b32 %0, %0;" : "+f"(kscale));
            const uint8_t* mrow = a.mask ? a.mask + (a.mask_h == 1 ? 0 : hch) * nblk : nullptr;

            // Monarch mode: the keep set, its empty c2 groups (their S3 and
            // S3' chunk pairs are not run) and the ring slot of each chunk
            const uint32_t keep = MODE == kMonarch ? a.keep_c2 : 0xffffffffu;
            const uint32_t empty = MODE == kMonarch ? empty_groups(keep) : 0u;
            const int slots4 = kChunks / 4 - popc4(empty);      // ring rounds per tile
            const int off_late = 4 * popc4(empty);               // slot = chunk - off_late from S2' on
            // the ring helpers take the chunk's slot (its chunk index outside
            // the Monarch mode)
            auto begin_pair = [&](int sl) -> bool {
                const uint32_t par = (uint32_t)(iter * slots4 + (sl >> 2)) & 1u;
                if (!wait(&dfull[sl & 3], par) || !wait(&dfull[(sl & 3) + 1], par)) {
                    fail();
                    return false;
                }
                tc_fence_after();
                return true;
            };
            auto release = [&](int sl) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&dfree[sl & 3]);
                    mbar_arrive(&dfree[(sl & 3) + 1]);
                }
            };
            auto stage_done = [&](int i) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar_stage[i]);
            };
            auto dcol = [&](int sl) -> uint32_t { return tbase + lq + 256 + 64 * (sl & 3); };

            // E1 (S1 -> S2), chunks j3 = k, k+1: lane = l; PP columns of
            // c1 = 8s .. 8s+7; twiddle w1024^(c1 l); MN-major A2 tile j3,
            // rows 32q + c1, K = l (real) and 32 + l (imaginary).
            // E2' (S2' -> S1'): lane = c1; PP columns of l = 8s .. 8s+7;
            // twiddle conj w1024^(c1 l); MN-major A6 tile j3, rows 32q + l,
            // K = c1 and 32 + c1.  The same twiddles and the same stores.
            auto e_transpose = [&](int sl, int k, bool conj) {
                uint32_t r[2][16];
                tmem_ld16(dcol(sl) + 16 * s, r[0]);
                tmem_ld16(dcol(sl + 1) + 16 * s, r[1]);
                tc_wait_ld();
                release(sl);
                const uint32_t flip = conj ? kNegPair : 0u;
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    uint32_t wr[4], wi[4];
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        wr[p] = pk(r[cc][4 * p], r[cc][4 * p + 1]);
                        wi[p] = pk(r[cc][4 * p + 2], r[cc][4 * p + 3]);
                        cmul_pp(wr[p], wi[p], twr[p], twi[p] ^ flip);
                    }
                    uint8_t* tile = smem + OffData + (k + cc) * kTile;
                    *(uint4*)(tile + mn_off(32 * q + 8 * s, lane)) = make_uint4(wr[0], wr[1], wr[2], wr[3]);
                    *(uint4*)(tile + mn_off(32 * q + 8 * s, 32 + lane)) = make_uint4(wi[0], wi[1], wi[2], wi[3]);
                }
                fence_proxy_async_smem();
            };

#pragma unroll 1
            for (int k = 0; k < 8; k += 2) {
                if (!(ok = begin_pair(k))) break;
                e_transpose(k, k, false);
            }
            // E2, chunks j3 = k, k+1: lane = c1; PP columns of c2 = 8s .. 8s+7;
            // twiddle w8192^(c1 j3) (one PP pair over j3 = k, k+1); A3 TMEM
            // columns 8 c2 + k (real pair), 8 c2 + k + 1 (imaginary pair)
            // (Monarch mode: the A3 columns of a masked c2 are not needed)
            const uint32_t keep_e2 = (keep >> (8 * s)) & 0xffu;     // this slice's c2
#pragma unroll 1
            for (int k = 0; k < 8 && ok; k += 2) {
                const int c = 8 + k;
                if (!(ok = begin_pair(c))) break;
                uint32_t r[2][16];
                // (loads are unconditional: loads under a branch spill the array)
                tmem_ld16(dcol(c) + 16 * s, r[0]);
                tmem_ld16(dcol(c + 1) + 16 * s, r[1]);
                const __half2 t0 = u2h(stw[lane * k]), t1 = u2h(stw[lane * (k + 1)]);
                const uint32_t tr = h2u(__lows2half2(t0, t1)), ti = h2u(__highs2half2(t0, t1));
                tc_wait_ld();
                release(c);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    if ((keep_e2 >> i) & 1u) {
                        const int ire = 4 * (i >> 1) + (i & 1);
                        uint32_t wr = pk(r[0][ire], r[1][ire]), wi = pk(r[0][ire + 2], r[1][ire + 2]);
                        cmul_pp(wr, wi, tr, ti);
                        tmem_st2(tbase + lq + 8 * (8 * s + i) + k, wr, wi);
                    }
                }
                tc_wait_st();
            }
            if (ok) stage_done(0);
            // EK: lane = c1; the PP columns of c3 (all eight) of c2 = 4(k+cc) + s;
            // times the filter spectrum K/scale (|K/scale| <= 1); A4 TMEM
            // columns 8 c2 .. 8 c2 + 7 in place.
            // Block mode (P = 2 or 4 blocks of 4096 per pair): quarter q holds
            // block b = q >> blk_shift of pair q & (pairs per tile - 1).  Block
            // b's output is sum_{j <= b} X_j G_{b-j}, G_d the spectrum of
            // [k_d; k_{d-1}] (k_d the filter taps [4096 d, 4096 d + 4096),
            // k_{-1} = 0): G_d holds both the taps that reach d blocks ahead
            // and the wrap-around of the 8192-point product.  The warps of
            // blocks b < P - 1 hand their values over through the data tiles
            // (free between S2 and E3') before their own product; G_0 is in
            // shared memory, G_1 of P = 2 arrives by cp.async (or is
            // (-1)^f G_0 when k_1 = 0), the G_d of P = 4 come from L2.
            if (ok && !(ok = wait(bar_k, iter & 1))) fail();
            using BM = Blocks<MODE>;
            const int blk = BM::on ? q >> BM::kShift : 0;
            const int pq = BM::on ? q & ((1 << BM::kShift) - 1) : 0;
            constexpr int np = BM::on ? (BM::P - 1) << BM::kShift : 1;      // producers per slice
            // (the correlation of the backward pass runs the other way: block b
            // takes sum_{j > b} X_j conj(G_{j-b}), so the later blocks give)
            const bool x_give = BM::on && (BWD ? blk > 0 : blk < BM::P - 1);
            const bool x_take = BM::on && (BWD ? blk < BM::P - 1 : blk > 0);
            const int gi = BWD ? blk - 1 : blk;                        // giving index among the blocks
            const int xz = (s * np + (gi << BM::kShift) + pq) * 4;    // this warp's slots when giving
            const int xg = 32 + (2 * s + pq) * 4;                      // P = 2: the G_1 slots
            const bool g1_async = x_take && BM::P == 2 && !a.g1_from_g0;
            uint8_t* const xs = smem + OffData;
            if (g1_async && ok) {
                // the block-1 warps fetch their G_1 words of all four steps into
                // their slots (the data tiles are free: this warp's E2 waited for
                // every S2 chunk)
                const uint32_t* G1 = a.K + hch * a.kstride + kM;
#pragma unroll
                for (int st = 0; st < 4; ++st) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int c2 = 4 * (2 * st + (e >> 1)) + s;
                        cp_async16(xs + xoff(st, xg + e, lane), G1 + k_word(lane, c2, 4 * (e & 1)));
                    }
                    cp_async_commit();
                }
            }
#pragma unroll 1
            for (int k = 0; k < 8 && ok; k += 2) {
                const int c = 16 + k;
                const int st = k >> 1;
                if (MODE == kMonarch && ((empty >> st) & 1u)) continue;     // group st: S3 not run
                const int sl = c - 2 * popc4(empty & ((1u << st) - 1u));
                // this warp's two c2 (4k + s, 4k + 4 + s); Monarch mode skips a masked one
                const bool kc0 = (keep >> (4 * k + s)) & 1u, kc1 = (keep >> (4 * k + 4 + s)) & 1u;
                if (!(ok = begin_pair(sl))) break;
                uint32_t r[2][16];
                tmem_ld16(dcol(sl) + 16 * s, r[0]);
                tmem_ld16(dcol(sl + 1) + 16 * s, r[1]);
                tc_wait_ld();
                release(sl);
                // h[cc]: the PP words of c2 = 4(k+cc) + s (all eight c3)
                uint32_t h[2][8];
#pragma unroll
                for (int cc = 0; cc < 2; ++cc)
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        h[cc][2 * p] = pk(r[cc][4 * p], r[cc][4 * p + 1]);
                        h[cc][2 * p + 1] = pk(r[cc][4 * p + 2], r[cc][4 * p + 3]);
                    }
                uint64_t* const xrow = &xfull[(st * 4 + s) * np];       // this step and slice
                if (x_give) {
                    // hand this block's values over before this warp's own product
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        *(uint4*)(xs + xoff(st, xz + 2 * cc, lane)) = make_uint4(h[cc][0], h[cc][1], h[cc][2], h[cc][3]);
                        *(uint4*)(xs + xoff(st, xz + 2 * cc + 1, lane)) =
                            make_uint4(h[cc][4], h[cc][5], h[cc][6], h[cc][7]);
                    }
                    mbar_arrive(&xrow[(gi << BM::kShift) + pq]);
                }
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    if (!(cc ? kc1 : kc0)) continue;       // (Monarch mode) masked c2: no product
                    const int c2 = 4 * (k + cc) + s;
                    const uint4 k0 = *(const uint4*)(Ks + k_word(lane, c2, 0));
                    const uint4 k1 = *(const uint4*)(Ks + k_word(lane, c2, 4));
                    uint32_t kw[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
                    if (!BM::on && mrow) {
                        // frequency-sparse filter: zero the masked bins (f and
                        // its mirror 8192 - f share one rfft bin)
#pragma unroll
                        for (int c3 = 0; c3 < 8; ++c3) {
                            const int f = lane + 32 * c2 + 1024 * c3;
                            int blk = (f <= kN ? f : kM - f) >> 5;
                            blk = blk < (int)nblk ? blk : (int)nblk - 1;
                            if (__ldg(&mrow[blk]) == 0) {
                                const uint32_t keep = (c3 & 1) ? 0x0000ffffu : 0xffff0000u;
                                kw[2 * (c3 >> 1)] &= keep;
                                kw[2 * (c3 >> 1) + 1] &= keep;
                            }
                        }
                    }
                    if constexpr (MODE == kMonarch) {
                        // a kept bin whose Hermitian mirror 8192 - f has a masked
                        // c2 is zeroed too, so the spectrum stays symmetric
#pragma unroll
                        for (int c3 = 0; c3 < 8; ++c3) {
                            const int f = lane + 32 * c2 + 1024 * c3;
                            const int c2m = (((kM - f) & (kM - 1)) >> 5) & 31;
                            if (!((keep >> c2m) & 1u)) {
                                const uint32_t keepw = (c3 & 1) ? 0x0000ffffu : 0xffff0000u;
                                kw[2 * (c3 >> 1)] &= keepw;
                                kw[2 * (c3 >> 1) + 1] &= keepw;
                            }
                        }
                    }
                    if constexpr (BWD) {
#pragma unroll
                        for (int p = 0; p < 4; ++p) kw[2 * p + 1] ^= kNegPair;   // conj(K)
                    }
#pragma unroll
                    for (int p = 0; p < 4; ++p) cmul_pp(h[cc][2 * p], h[cc][2 * p + 1], kw[2 * p], kw[2 * p + 1]);
                }
                if (BM::P == 4 && x_take) {
                    // + X_j G_{b-j} for the earlier blocks j of this pair (G_d
                    // words from L2, requested before the hand-over wait)
#pragma unroll 1
                    for (int j = 0; j < blk && ok; ++j) {
                        const int d = blk - j;
                        if (d >= a.ng) continue;                  // G_d = 0: the filter is shorter
                        const uint32_t* Gd = a.K + hch * a.kstride + d * kM;
                        uint4 gq0 = __ldg((const uint4*)(Gd + k_word(lane, 4 * k + s, 0)));
                        uint4 gq1 = __ldg((const uint4*)(Gd + k_word(lane, 4 * k + s, 4)));
                        if (!(ok = wait(&xrow[j], iter & 1))) {
                            fail();
                            break;
                        }
                        const int zj = (s * np + j) * 4;
#pragma unroll
                        for (int cc = 0; cc < 2; ++cc) {
                            if (cc == 1) {
                                gq0 = __ldg((const uint4*)(Gd + k_word(lane, 4 * k + 4 + s, 0)));
                                gq1 = __ldg((const uint4*)(Gd + k_word(lane, 4 * k + 4 + s, 4)));
                            }
                            const uint4 x0 = *(const uint4*)(xs + xoff(st, zj + 2 * cc, lane));
                            const uint4 x1 = *(const uint4*)(xs + xoff(st, zj + 2 * cc + 1, lane));
                            const uint32_t xw[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                            const uint32_t gw[8] = {gq0.x, gq0.y, gq0.z, gq0.w, gq1.x, gq1.y, gq1.z, gq1.w};
#pragma unroll
                            for (int p = 0; p < 4; ++p)
                                cfma_pp(h[cc][2 * p], h[cc][2 * p + 1], xw[2 * p], xw[2 * p + 1], gw[2 * p],
                                        gw[2 * p + 1]);
                        }
                    }
                    if (!ok) break;
                } else if (x_take) {
                    // P = 2: + X_0 G_1 (backward: + X_1 conj(G_1)), once the
                    // other block's warp has handed its values over
                    if (!(ok = wait(&xrow[pq], iter & 1))) {
                        fail();
                        break;
                    }
                    if (!a.g1_from_g0) {      // this thread's G_1 copies of steps <= st have landed
                        if (st == 0) cp_async_wait<3>();
                        else if (st == 1) cp_async_wait<2>();
                        else if (st == 2) cp_async_wait<1>();
                        else cp_async_wait<0>();
                    }
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        const int z0 = (s * np + pq) * 4;              // the giving warp of this pair
                        const uint4 x0 = *(const uint4*)(xs + xoff(st, z0 + 2 * cc, lane));
                        const uint4 x1 = *(const uint4*)(xs + xoff(st, z0 + 2 * cc + 1, lane));
                        const uint32_t xw[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                        uint32_t gw[8];
                        if (a.g1_from_g0) {
                            // k1 = 0: G_1 = (-1)^f G_0, and f = c1 (mod 2) = lane (mod 2)
                            const int c2 = 4 * (k + cc) + s;
                            const uint4 k0 = *(const uint4*)(Ks + k_word(lane, c2, 0));
                            const uint4 k1 = *(const uint4*)(Ks + k_word(lane, c2, 4));
                            const uint32_t sg = (lane & 1) ? kNegPair : 0u;
                            gw[0] = k0.x ^ sg; gw[1] = k0.y ^ sg; gw[2] = k0.z ^ sg; gw[3] = k0.w ^ sg;
                            gw[4] = k1.x ^ sg; gw[5] = k1.y ^ sg; gw[6] = k1.z ^ sg; gw[7] = k1.w ^ sg;
                        } else {
                            const uint4 g0 = *(const uint4*)(xs + xoff(st, xg + 2 * cc, lane));
                            const uint4 g1 = *(const uint4*)(xs + xoff(st, xg + 2 * cc + 1, lane));
                            gw[0] = g0.x; gw[1] = g0.y; gw[2] = g0.z; gw[3] = g0.w;
                            gw[4] = g1.x; gw[5] = g1.y; gw[6] = g1.z; gw[7] = g1.w;
                        }
                        if constexpr (BWD) {
#pragma unroll
                            for (int p = 0; p < 4; ++p) gw[2 * p + 1] ^= kNegPair;   // conj(G_1)
                        }
#pragma unroll
                        for (int p = 0; p < 4; ++p)
                            cfma_pp(h[cc][2 * p], h[cc][2 * p + 1], xw[2 * p], xw[2 * p + 1], gw[2 * p], gw[2 * p + 1]);
                    }
                }
                if (kc0) tmem_st8(tbase + lq + 8 * (4 * k + s), h[0]);
                if (kc1) tmem_st8(tbase + lq + 8 * (4 * k + 4 + s), h[1]);
                tc_wait_st();
                if constexpr (MODE == kMonarch) {
                    // this group's A4 columns are written: its S3' chunks may run
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&ek_done[st]);
                }
            }
            if (g1_async) cp_async_wait<0>();     // nothing in flight past here (also after an abort)
            // E3': lane = c1; chunk c + (s >> 1), its c2 = 4(k + cc) + cl for
            // cl < 4, j3 = 4h + jj with h = s & 1 (PP columns 16 cl + 8h ..
            // + 7); twiddle conj w8192^(c1 j3); K-major A5 tile j3, row
            // 32q + c1, the PP K words of c2 = 4(k+cc) .. + 3 (16 bytes)
#pragma unroll 1
            for (int k = 0; k < 8 && ok; k += 2) {
                const int c = 24 + k;
                if (MODE == kMonarch && ((empty >> (k >> 1)) & 1u)) continue;   // S3' of this group not run
                const int sl = c - off_late / 2 - 2 * popc4(empty & ((1u << (k >> 1)) - 1u));
                if (!(ok = begin_pair(sl))) break;
                const int cc = s >> 1, h = s & 1;
                // Monarch mode: the S3' products of masked c2 were not issued,
                // so their accumulator columns are stale: a quadruple with a
                // masked c2 stores zeros there (S2' reads them unless its
                // whole K step of eight c2 is masked, then nothing is stored)
                const uint32_t kq = (keep >> (4 * (k + cc))) & 0xfu;
                const bool kstep = (keep >> (8 * ((k + cc) >> 1))) & 0xffu;
                uint32_t r[4][8];
#pragma unroll
                for (int cl = 0; cl < 4; ++cl) tmem_ld8(dcol(sl + cc) + 16 * cl + 8 * h, r[cl]);
                tc_wait_ld();
                release(sl);
                if (!kstep) {
                    fence_proxy_async_smem();
                    continue;
                }
                if (kq != 0xfu) {
#pragma unroll
                    for (int cl = 0; cl < 4; ++cl)
                        if (!((kq >> cl) & 1u))
#pragma unroll
                            for (int i = 0; i < 8; ++i) r[cl][i] = 0u;
                }
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const int j3 = 4 * h + jj;
                    const __half2 t = u2h(stw[lane * j3]);
                    const uint32_t trb = h2u(__low2half2(t)), tib = h2u(__high2half2(t)) ^ kNegPair;
                    const int ire = 4 * (jj >> 1) + (jj & 1);
                    uint32_t w0r = pk(r[0][ire], r[1][ire]), w0i = pk(r[0][ire + 2], r[1][ire + 2]);
                    uint32_t w1r = pk(r[2][ire], r[3][ire]), w1i = pk(r[2][ire + 2], r[3][ire + 2]);
                    cmul_pp(w0r, w0i, trb, tib);
                    cmul_pp(w1r, w1i, trb, tib);
                    uint8_t* tile = smem + OffData + j3 * kTile;
                    *(uint4*)(tile + k_off(32 * q + lane, 16 * (k + cc))) =
                        make_uint4(w0r, w0i, w1r, w1i);
                }
                fence_proxy_async_smem();
            }
            if (ok) stage_done(1);
            if (ok && unit + gridDim.x < a.nunits) load_tile(unit + gridDim.x, 0);
#pragma unroll 1
            for (int k = 0; k < 8 && ok; k += 2) {
                const int c = 32 + k;
                if (!(ok = begin_pair(c - off_late))) break;
                e_transpose(c - off_late, k, true);
            }
            if (ok) stage_done(2);
            if (ok && unit + gridDim.x < a.nunits) load_tile(unit + gridDim.x, 1);
            // EO: lane = l; chunk 40 + k holds j3 = 2k + jl (jl = 0, 1) at
            // columns 32 jl + PP(i) for the kept stage-1 indices i < 16.  This
            // warp takes i = 4s + 2hf + jj in two halves hf: the PP words of
            // index pair 2s + hf (columns 32 jl + 8s + 4hf .. + 3) of all four
            // chunks give the eight consecutive t = 256 j1 + 8 l + j3 of each
            // row: one 16-byte store.  y = s_h v z; in a window after the
            // first, positions t < 2048 (i < 8: warps with s < 2) are not
            // outputs.
            {
                // the output gates of both halves, requested before the
                // accumulator wait so that their latency overlaps it
                uint4 vg[2][2][2];            // [hf][jj][row]
                {
                    const T* vr = a.v ? (const T*)a.v : (const T*)a.u;   // any readable row if no gate
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf)
#pragma unroll
                        for (int jj = 0; jj < 2; ++jj) {
                            const int i = 4 * s + 2 * hf + jj;
                            const PairInfo Pg = pair_rows<MODE>(a, TB, q, seg_of(a, i));
                            const int64_t tg = tau_of(a, i) + 8 * lane;
                            const uint64_t pol = l2_evict_first();      // the gate is read once
                            vg[hf][jj][0] = ldg_nc_hint(vr + Pg.o0 + tg, pol);
                            vg[hf][jj][1] = ldg_nc_hint(vr + (Pg.o1 >= 0 ? Pg.o1 : Pg.o0) + tg, pol);
                        }
                }
#pragma unroll
                for (int hf = 0; hf < 2 && ok; ++hf) {
                    const int jb = 4 * s + 2 * hf;            // this pass's first kept index
                    PairInfo P[2];
                    int64_t t0[2];
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) {
                        P[jj] = pair_rows<MODE>(a, TB, q, seg_of(a, jb + jj));
                        t0[jj] = tau_of(a, jb + jj) + 8 * lane;
                    }
                    if (hf == 0 && (!(ok = begin_pair(40 - off_late)) || !(ok = begin_pair(42 - off_late)))) break;
                    // r[cc][jl][0..3] = re(jb), re(jb+1), im(jb), im(jb+1) of j3 = 2cc + jl
                    uint32_t r[4][2][4];
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc)
#pragma unroll
                        for (int jl = 0; jl < 2; ++jl)
                            tmem_ld4(dcol(40 - off_late + cc) + 32 * jl + 2 * jb, r[cc][jl]);
                    tc_wait_ld();
                    if (hf == 1) {
                        release(40 - off_late);
                        release(42 - off_late);
                    }
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) {
                        if (!P[jj].valid || (P[jj].tail_only && s < 2)) continue;
                        const bool has1 = P[jj].o1 >= 0;
                        const uint32_t vaw[4] = {vg[hf][jj][0].x, vg[hf][jj][0].y, vg[hf][jj][0].z, vg[hf][jj][0].w};
                        const uint32_t vbw[4] = {vg[hf][jj][1].x, vg[hf][jj][1].y, vg[hf][jj][1].z, vg[hf][jj][1].w};
                        uint32_t oa[4], ob[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            // j3 = 2e (chunk 40 + e, jl 0) and 2e + 1 (jl 1)
                            float a0 = __uint_as_float(r[e][0][jj]) * kscale;
                            float a1 = __uint_as_float(r[e][1][jj]) * kscale;
                            float b0 = __uint_as_float(r[e][0][2 + jj]) * kscale;
                            float b1 = __uint_as_float(r[e][1][2 + jj]) * kscale;
                            // fp16 range (t = 256 j1 + 8 l + j3): a non-finite
                            // value in a forward stage or the filter product
                            // reaches every output of the transform, one after
                            // S3' every output of its j3 and one after S2' every
                            // j1 of its (l, j3), in the real or the imaginary
                            // part.  So each warp checks both sequences at every
                            // (l, j3) of its pair for one kept j1 (hf = jj = 0:
                            // the first segment, valid whenever any is; in a
                            // later window the warps s >= 2; the four-block
                            // build measured faster checking every value)
                            if (MODE == kFour || (hf == 0 && jj == 0)) {
                                nonfinite_fold(nf, a0); nonfinite_fold(nf, a1);
                                nonfinite_fold(nf, b0); nonfinite_fold(nf, b1);
                            }
                            if (a.v) {
                                const float2 g0 = IO<T>::unpack2(vaw[e]), g1 = IO<T>::unpack2(vbw[e]);
                                a0 *= g0.x; a1 *= g0.y; b0 *= g1.x; b1 *= g1.y;
                            }
                            oa[e] = IO<T>::pack2(a0, a1);
                            ob[e] = IO<T>::pack2(b0, b1);
                        }
                        *(uint4*)((T*)a.y + P[jj].o0 + t0[jj]) = make_uint4(oa[0], oa[1], oa[2], oa[3]);
                        if (has1) *(uint4*)((T*)a.y + P[jj].o1 + t0[jj]) = make_uint4(ob[0], ob[1], ob[2], ob[3]);
                        if constexpr (BWD) {
                            if (a.y2) {
                                // y2 = s_h v2 z: the same z, the second gate
                                const uint4 ga = __ldg((const uint4*)((const T*)a.v2 + P[jj].o0 + t0[jj]));
                                const uint4 gb = __ldg((const uint4*)((const T*)a.v2 + (has1 ? P[jj].o1 : P[jj].o0) +
                                                                      t0[jj]));
                                const uint32_t gaw[4] = {ga.x, ga.y, ga.z, ga.w};
                                const uint32_t gbw[4] = {gb.x, gb.y, gb.z, gb.w};
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const float a0 = __uint_as_float(r[e][0][jj]) * kscale;
                                    const float a1 = __uint_as_float(r[e][1][jj]) * kscale;
                                    const float b0 = __uint_as_float(r[e][0][2 + jj]) * kscale;
                                    const float b1 = __uint_as_float(r[e][1][2 + jj]) * kscale;
                                    const float2 g0 = IO<T>::unpack2(gaw[e]), g1 = IO<T>::unpack2(gbw[e]);
                                    oa[e] = IO<T>::pack2(a0 * g0.x, a1 * g0.y);
                                    ob[e] = IO<T>::pack2(b0 * g1.x, b1 * g1.y);
                                }
                                *(uint4*)((T*)a.y2 + P[jj].o0 + t0[jj]) = make_uint4(oa[0], oa[1], oa[2], oa[3]);
                                if (has1)
                                    *(uint4*)((T*)a.y2 + P[jj].o1 + t0[jj]) = make_uint4(ob[0], ob[1], ob[2], ob[3]);
                            }
                        }
                    }
                }
            }
        }
        nonfinite_report(nf, a.status);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kEpiWarps) {     // the warp that allocated
        tc_fence_after();
        tmem_dealloc(tbase, 512);
        tmem_relinquish();
    }
}

// ----------------------------------------------------------- host side ---

struct Resources {
    uint8_t* bimg = nullptr;
    uint32_t* tw1024 = nullptr;
    uint32_t* tw8192 = nullptr;
    float2* twf8192 = nullptr;     // fp32 exp(-2 pi i e/8192), e < 8192 (two-block filter precompute)
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

// Real-pair image of the complex n_out x n_in matrix F as a K x N B operand
// (N = Ntot columns): input value j's real and imaginary parts sit at K rows
// kidx(0, j), kidx(1, j), output value c's at N columns nidx(0, c), nidx(1, c)
template <class KI, class NI>
void put_matrix(std::vector<uint8_t>& img, size_t base, int n_out, int n_in, int Ntot,
                const std::vector<std::complex<double>>& F, KI kidx, NI nidx) {
    for (int c = 0; c < n_out; ++c)
        for (int j = 0; j < n_in; ++j) {
            const std::complex<double> f = F[(size_t)c * n_in + j];
            put_f16(img, base + bimg_offset(nidx(0, c), kidx(0, j), Ntot), f.real());
            put_f16(img, base + bimg_offset(nidx(0, c), kidx(1, j), Ntot), -f.imag());
            put_f16(img, base + bimg_offset(nidx(1, c), kidx(0, j), Ntot), f.imag());
            put_f16(img, base + bimg_offset(nidx(1, c), kidx(1, j), Ntot), f.real());
        }
}

// the stage-1 digit j1 of kept index i (< 16): the transform's inputs and the
// kept outputs are the positions t = 256 j1 + 8 l + j3 with
// (j1 mod 2^(lseg+1)) < 2^lseg (for N = 4096, lseg = 4: j1 < 16)
int kept_j1(int i, int lseg) { return ((i >> lseg) << (lseg + 1)) | (i & ((1 << lseg) - 1)); }

std::vector<uint8_t> build_bimage(int lseg) {
    std::vector<uint8_t> img(BImageBytes, 0);
    const double r32 = 1.0 / std::sqrt(32.0), r8 = 1.0 / std::sqrt(8.0);
    auto off = [](int o) { return (size_t)(o - OffBS1); };
    auto pp = [](int comp, int i) { return pp_index(comp, i); };
    auto pl32 = [](int comp, int i) { return pl_index(comp, i, 32); };
    std::vector<std::complex<double>> F;
    // S1: c1 <- j1 (the 16 kept digits: the nonzero inputs)
    F.assign(32 * 16, 0);
    for (int c = 0; c < 32; ++c)
        for (int j = 0; j < 16; ++j) F[c * 16 + j] = wpow((long long)c * kept_j1(j, lseg), 32, -1) * r32;
    put_matrix(img, off(OffBS1), 32, 16, 64, F, pp, pp);
    // S2: c2 <- l
    F.assign(32 * 32, 0);
    for (int c = 0; c < 32; ++c) for (int j = 0; j < 32; ++j) F[c * 32 + j] = wpow((long long)c * j, 32, -1) * r32;
    put_matrix(img, off(OffBS2), 32, 32, 64, F, pl32, pp);
    // S3 (per c2): c3 <- j3 with w8^(c3 j3) w256^(c2 j3);  S3': j3 <- c3, conjugate
    for (int c2 = 0; c2 < 32; ++c2) {
        std::vector<std::complex<double>> G(64), Gi(64);
        for (int c3 = 0; c3 < 8; ++c3)
            for (int j3 = 0; j3 < 8; ++j3) {
                const std::complex<double> gv = wpow((long long)c3 * j3, 8, -1) * wpow((long long)c2 * j3, 256, -1) * r8;
                G[c3 * 8 + j3] = gv;
                Gi[j3 * 8 + c3] = std::conj(gv);
            }
        put_matrix(img, off(OffBS3) + c2 * 512, 8, 8, 16, G, pp, pp);
        put_matrix(img, off(OffBS3i) + c2 * 512, 8, 8, 16, Gi, pp, pp);
    }
    // S2': l <- c2
    F.assign(32 * 32, 0);
    for (int l = 0; l < 32; ++l) for (int c = 0; c < 32; ++c) F[l * 32 + c] = wpow((long long)c * l, 32, +1) * r32;
    put_matrix(img, off(OffBS2i), 32, 32, 64, F, pp, pp);
    // S1': j1 <- c1 (the 16 kept digits: the outputs)
    F.assign(16 * 32, 0);
    for (int j = 0; j < 16; ++j)
        for (int c = 0; c < 32; ++c) F[j * 32 + c] = wpow((long long)c * kept_j1(j, lseg), 32, +1) * r32;
    put_matrix(img, off(OffBS1i), 16, 32, 32, F, pl32, pp);
    return img;
}

uint32_t half2_bits(double re, double im) {
    const __half2 h = __floats2half2_rn((float)re, (float)im);
    uint32_t b;
    std::memcpy(&b, &h, 4);
    return b;
}

std::vector<uint32_t> twiddles_h2(int n, int count) {
    std::vector<uint32_t> t(count);
    for (int e = 0; e < count; ++e) {
        const std::complex<double> z = wpow(e, n, -1);
        t[e] = half2_bits(z.real(), z.imag());
    }
    return t;
}

template <typename V>
cudaError_t upload_vec(V** dst, const std::vector<V>& v) {
    cudaError_t e = cudaMalloc((void**)dst, v.size() * sizeof(V));
    if (e == cudaSuccess) e = cudaMemcpy(*dst, v.data(), v.size() * sizeof(V), cudaMemcpyHostToDevice);
    return e;
}

template <typename T, int MODE, bool BWD = false, bool UNGATED = false>
void launch(const PArgs& a, int64_t grid, cudaStream_t s) {
    tc_fftconv_planar_kernel<T, MODE, BWD, UNGATED><<<(unsigned)grid, kThreads, SmemBytes, s>>>(a);
}

template <typename T, int MODE, bool BWD = false, bool UNGATED = false>
cudaError_t allow_smem() {
    return cudaFuncSetAttribute(tc_fftconv_planar_kernel<T, MODE, BWD, UNGATED>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, SmemBytes);
}

// K_f (PP layout) -> rfft bins [0, N] of each channel's 2N-point spectrum:
// bin f is bin f * (4096 / N) of the 8192-point spectrum of the zero-padded
// filter (N <= 4096)
__global__ void planar_export_kernel(const uint32_t* __restrict__ K, const float* __restrict__ scale,
                                     float* __restrict__ out, int64_t H, int64_t N) {
    const int64_t nb = N + 1, total = H * nb, stride = kN / N;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t h = i / nb, f = (i % nb) * stride;
        const int c1 = (int)(f & 31), c2 = (int)((f >> 5) & 31), c3 = (int)(f >> 10);
        const uint32_t* row = K + h * kM;
        const int wd = k_word(c1, c2, c3), half = c3 & 1;
        const __half re = __ushort_as_half((unsigned short)(row[wd] >> (16 * half)));
        const __half im = __ushort_as_half((unsigned short)(row[wd + 1] >> (16 * half)));
        out[2 * i] = __half2float(re) * scale[h];
        out[2 * i + 1] = __half2float(im) * scale[h];
    }
}

}  // namespace

// log2(N / 256) for packed and single sequences (N <= 4096); overlap-save
// windows (N > 4096) transform 4096 inputs each, like N = 4096
static int plan_lseg(int64_t N) {
    if (N > kN) return 4;
    int l = 0;
    while ((int64_t(256) << l) < N) ++l;
    return l;
}

cudaError_t tc_planar_init(Plan& p) {
    Resources* r = new Resources();
    p.tcp = r;
    cudaError_t e = upload_vec(&r->bimg, build_bimage(plan_lseg(p.N)));
    if (e == cudaSuccess) e = upload_vec(&r->tw1024, twiddles_h2(1024, 1024));
    if (e == cudaSuccess) e = upload_vec(&r->tw8192, twiddles_h2(kM, 256));
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&r->num_sms, cudaDevAttrMultiProcessorCount, p.device);
    if (e == cudaSuccess && (p.N == 2 * kN || p.N == 4 * kN)) {
        std::vector<float2> t(kM);
        for (int i = 0; i < kM; ++i) {
            const std::complex<double> z = wpow(i, kM, -1);
            t[i] = make_float2((float)z.real(), (float)z.imag());
        }
        e = upload_vec(&r->twf8192, t);
    }
    if (e == cudaSuccess) e = allow_smem<__nv_bfloat16, kPlain>();
    if (e == cudaSuccess) e = allow_smem<__nv_bfloat16, kWin>();
    if (e == cudaSuccess) e = allow_smem<__nv_bfloat16, kTwo>();
    if (e == cudaSuccess) e = allow_smem<__nv_bfloat16, kFour>();
    if (e == cudaSuccess) e = allow_smem<__half, kPlain>();
    if (e == cudaSuccess) e = allow_smem<__half, kWin>();
    if (e == cudaSuccess) e = allow_smem<__half, kTwo>();
    if (e == cudaSuccess) e = allow_smem<__half, kFour>();
    if (e == cudaSuccess) e = allow_smem<__nv_bfloat16, kMonarch>();
    if (e == cudaSuccess) e = allow_smem<__half, kMonarch>();
    if (e == cudaSuccess) e = allow_smem<__nv_bfloat16, kPlain, true>();
    if (e == cudaSuccess) e = allow_smem<__half, kPlain, true>();
    if (e == cudaSuccess) e = allow_smem<__nv_bfloat16, kTwo, true>();
    if (e == cudaSuccess) e = allow_smem<__half, kTwo, true>();
    if (e == cudaSuccess) e = allow_smem<__nv_bfloat16, kPlain, false, true>();
    if (e == cudaSuccess) e = allow_smem<__half, kPlain, false, true>();
    if (e == cudaSuccess) e = allow_smem<__nv_bfloat16, kTwo, false, true>();
    if (e == cudaSuccess) e = allow_smem<__half, kTwo, false, true>();
    if (e == cudaSuccess) e = allow_smem<__nv_bfloat16, kFour, false, true>();
    if (e == cudaSuccess) e = allow_smem<__half, kFour, false, true>();
    return e;
}

void tc_planar_free(Plan& p) {
    Resources* r = (Resources*)p.tcp;
    if (!r) return;
    cudaFree(r->bimg);
    cudaFree(r->tw1024);
    cudaFree(r->tw8192);
    cudaFree(r->twf8192);
    delete r;
    p.tcp = nullptr;
}

// K_f: H rows of 8192 complex fp16 (the spectrum over each channel's largest
// component, PP layout), then [H] fp32 scales
size_t tc_planar_filter_bytes(const Plan& p) {
    return (size_t)p.H * kKBytes + (((size_t)p.H * 4 + 15) & ~size_t(15));
}

// Block-mode K_f (sequences of 8192 or 16384, P = N / 4096 blocks): per
// channel the P rows G_0 = FFT_8192([k0; 0]), G_d = FFT_8192([k_d; k_{d-1}])
// (k_d the taps [4096 d, 4096 d + 4096) of k, zero past L), PP layout over one
// common scale, then [H] fp32 scales
size_t tc_planar_two_block_bytes(const Plan& p) {
    return (size_t)p.H * (size_t)(p.N / kN) * kKBytes + (((size_t)p.H * 4 + 15) & ~size_t(15));
}

cudaError_t tc_planar_precompute(const Plan& p, const void* k, void* Kf, cudaStream_t s) {
    return simt_precompute_to_tc_pp(p, k, Kf, s);
}

cudaError_t tc_planar_precompute_two_block(const Plan& p, const void* k, void* Kf, cudaStream_t s) {
    const Resources* r = (const Resources*)p.tcp;
    if ((p.N != 2 * kN && p.N != 4 * kN) || !r->twf8192) return cudaErrorInvalidValue;
    return p.N == 2 * kN ? simt_precompute_to_tc_pp2(p, k, Kf, r->twf8192, s)
                         : simt_precompute_to_tc_pp4(p, k, Kf, r->twf8192, s);
}

// mode: kPlain (N <= 4096), kWin (overlap-save windows), kTwo (block modes,
// N = 8192 or 16384; fa.Kf the block filter rows)
cudaError_t tc_planar_forward(const Plan& p, const ForwardArgs& fa, int mode, cudaStream_t s) {
    const Resources* r = (const Resources*)p.tcp;
    if (mode == kTwo && ((p.N != 2 * kN && p.N != 4 * kN) || fa.mask)) return cudaErrorInvalidValue;
    PArgs a{};
    a.u = fa.u; a.w = fa.w; a.v = fa.v; a.y = fa.y;
    a.K = (const uint32_t*)fa.Kf;
    const int rows = mode == kTwo ? (int)(p.N / kN) : 1;       // filter rows per channel
    a.kstride = (int64_t)rows * kM;
    a.g1_from_g0 = mode == kTwo && rows == 2 && p.L <= kN;
    a.ng = (int)((p.L + kN - 1) / kN) + 1;                      // G_d = 0 for d > ceil(L / 4096)
    if (a.ng > rows) a.ng = rows;
    a.Kscale = (const float*)((const uint8_t*)fa.Kf + (size_t)p.H * rows * kKBytes);
    a.mask = fa.mask; a.mask_h = fa.mask_h;
    a.B = fa.B; a.H = p.H; a.N = p.N;
    a.nwin = mode == kWin ? p.N / kHop - 1 : 1;
    a.lseg = plan_lseg(p.N);
    a.pb = (fa.B + 1) / 2;
    const int64_t pairs_per_tile = mode == kTwo ? 4 / rows : int64_t(64) >> a.lseg;   // 4 rows x 4096 / N pairs
    a.tpc = (a.pb + pairs_per_tile - 1) / pairs_per_tile;
    a.nunits = p.H * a.nwin * a.tpc;
    a.bimg = (const uint4*)r->bimg;
    a.tw1024 = r->tw1024;
    a.tw8192 = r->tw8192;
    a.status = p.status;
    const int64_t grid = a.nunits < r->num_sms ? a.nunits : r->num_sms;
    if (p.dtype == kBF16) {
        if (mode == kWin) launch<__nv_bfloat16, kWin>(a, grid, s);
        else if (mode == kTwo && rows == 4 && !a.w) launch<__nv_bfloat16, kFour, false, true>(a, grid, s);
        else if (mode == kTwo && rows == 4) launch<__nv_bfloat16, kFour>(a, grid, s);
        else if (mode == kTwo && !a.w) launch<__nv_bfloat16, kTwo, false, true>(a, grid, s);
        else if (mode == kTwo) launch<__nv_bfloat16, kTwo>(a, grid, s);
        else if (!a.w) launch<__nv_bfloat16, kPlain, false, true>(a, grid, s);
        else launch<__nv_bfloat16, kPlain>(a, grid, s);
    } else {
        if (mode == kWin) launch<__half, kWin>(a, grid, s);
        else if (mode == kTwo && rows == 4 && !a.w) launch<__half, kFour, false, true>(a, grid, s);
        else if (mode == kTwo && rows == 4) launch<__half, kFour>(a, grid, s);
        else if (mode == kTwo && !a.w) launch<__half, kTwo, false, true>(a, grid, s);
        else if (mode == kTwo) launch<__half, kTwo>(a, grid, s);
        else if (!a.w) launch<__half, kPlain, false, true>(a, grid, s);
        else launch<__half, kPlain>(a, grid, s);
    }
    return cudaGetLastError();
}

cudaError_t tc_planar_forward_monarch(const Plan& p, const ForwardArgs& fa, uint32_t keep_c2, cudaStream_t s) {
    const Resources* r = (const Resources*)p.tcp;
    if (p.N != kN || fa.mask || keep_c2 == 0) return cudaErrorInvalidValue;
    PArgs a{};
    a.u = fa.u; a.w = fa.w; a.v = fa.v; a.y = fa.y;
    a.K = (const uint32_t*)fa.Kf;
    a.kstride = kM;
    a.Kscale = (const float*)((const uint8_t*)fa.Kf + (size_t)p.H * kKBytes);
    a.keep_c2 = keep_c2;
    a.B = fa.B; a.H = p.H; a.N = p.N;
    a.nwin = 1;
    a.lseg = plan_lseg(p.N);
    a.pb = (fa.B + 1) / 2;
    a.tpc = (a.pb + 3) / 4;
    a.nunits = p.H * a.tpc;
    a.bimg = (const uint4*)r->bimg;
    a.tw1024 = r->tw1024;
    a.tw8192 = r->tw8192;
    a.status = p.status;
    const int64_t grid = a.nunits < r->num_sms ? a.nunits : r->num_sms;
    if (p.dtype == kBF16) launch<__nv_bfloat16, kMonarch>(a, grid, s);
    else launch<__half, kMonarch>(a, grid, s);
    return cudaGetLastError();
}

// Correlation pass of the backward (N <= 4096): y = v * corr(u * w, k),
// y2 = v2 * corr(u * w, k) (y2 may be NULL), i.e. the forward kernel with the
// product by conj(K) and a second gated output.
cudaError_t tc_planar_correlate(const Plan& p, const ForwardArgs& fa, void* y2, const void* v2, cudaStream_t s) {
    if (p.N > 2 * kN) return cudaErrorInvalidValue;
    const bool two = p.N == 2 * kN;              // fa.Kf: the two-block rows G_0, G_1
    const Resources* r = (const Resources*)p.tcp;
    PArgs a{};
    a.u = fa.u; a.w = fa.w; a.v = fa.v; a.y = fa.y;
    a.y2 = y2; a.v2 = v2;
    a.K = (const uint32_t*)fa.Kf;
    a.kstride = two ? 2 * kM : kM;
    a.Kscale = (const float*)((const uint8_t*)fa.Kf + (size_t)p.H * (two ? 2 : 1) * kKBytes);
    a.g1_from_g0 = two && p.L <= kN;
    a.ng = two ? 2 : 1;
    a.B = fa.B; a.H = p.H; a.N = p.N;
    a.nwin = 1;
    a.lseg = plan_lseg(p.N);
    a.pb = (fa.B + 1) / 2;
    const int64_t pairs_per_tile = two ? 2 : int64_t(64) >> a.lseg;
    a.tpc = (a.pb + pairs_per_tile - 1) / pairs_per_tile;
    a.nunits = p.H * a.tpc;
    a.bimg = (const uint4*)r->bimg;
    a.tw1024 = r->tw1024;
    a.tw8192 = r->tw8192;
    a.status = p.status;
    const int64_t grid = a.nunits < r->num_sms ? a.nunits : r->num_sms;
    if (p.dtype == kBF16) {
        if (two) launch<__nv_bfloat16, kTwo, true>(a, grid, s);
        else launch<__nv_bfloat16, kPlain, true>(a, grid, s);
    } else {
        if (two) launch<__half, kTwo, true>(a, grid, s);
        else launch<__half, kPlain, true>(a, grid, s);
    }
    return cudaGetLastError();
}

cudaError_t tc_planar_export(const Plan& p, const void* Kf, float* out, cudaStream_t s) {
    if (p.N > kN) return cudaErrorInvalidValue;      // overlap-save plans store the 8192-point spectrum only
    const int64_t total = p.H * (p.N + 1);
    int blocks = (int)((total + 255) / 256);
    if (blocks > 65535) blocks = 65535;
    planar_export_kernel<<<blocks, 256, 0, s>>>((const uint32_t*)Kf,
                                                (const float*)((const uint8_t*)Kf + (size_t)p.H * kKBytes), out, p.H,
                                                p.N);
    return cudaGetLastError();
}

}  // namespace fftconv
