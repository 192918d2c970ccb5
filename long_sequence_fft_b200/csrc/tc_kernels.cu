// tc_kernels.cu -- tensor-core (tcgen05) fused FFT convolution, sm_100a.
//
// FlashFFTConv: Efficient Convolutions for Long Sequences with Tensor Cores,
// "Approach": the FFT convolution is rewritten as an order-p Monarch
// decomposition -- matrix-matrix products with small DFT factors applied
// along one digit of the sequence index -- so the transform runs on tensor
// cores, permutations become on-chip transposes, and the whole convolution
// (gates included, "Key results") is one kernel.
//
// The transform engine: 8192-point transforms of 4-pair tiles.
//   t = 256*j1 + 8*l + j3   (j1 < 32, l < 32, j3 < 8)
//   f = c1 + 32*c2 + 1024*c3
//   exp(-2 pi i f t / 8192) = w32^(c1 j1) w1024^(c1 l) w8192^(c1 j3) w32^(c2 l) w256^(c2 j3) w8^(c3 j3)
// Forward: S1 contracts j1 (DFT-32), twiddle w1024^(c1 l), S2 contracts l
// (DFT-32), twiddle w8192^(c1 j3), S3 contracts j3 with the per-c2 factor
// w8^(c3 j3) w256^(c2 j3) (the second twiddle folded into the matrix).
// Product with the filter spectrum, then the mirror image with conjugate
// factors (S3', S2', S1').
//
// Four modes use it (see Lay and pair_info):
//   plain    N = 4096: x zero for t >= 4096 (S1 sees 16 nonzero j1), S1' emits
//            only t < 4096;
//   windows  N > 4096 with filters of at most 2049 taps: overlap-save windows
//            of 4096 inputs, hop 2048;
//   split    N = 8192 with longer filters: the 16384-point spectrum split by
//            bin parity into two 8192-point transforms of all 8192 inputs;
//   rows     the row pass of the staged path for longer sequences (M = R x
//            8192): a tile is four complex fp16 workspace rows of one pair,
//            each transformed, multiplied by its own filter row and
//            transformed back in place (the column passes are SIMT kernels).
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
// (the "on-chip transpose").  Accumulators are fp32 in TMEM.  The epilogue
// warps round them to fp16 and apply the twiddles and the filter product
// (K / s_h, |K / s_h| <= 1) in packed half precision; the channel scale s_h
// is applied to y in fp32.  Each DFT factor carries 1/sqrt(n), so the forward
// and inverse transforms are unitary and the filter spectrum is used
// unnormalised.
//
// Warp roles: warps 0..15 are epilogue warps (warp w serves lane quarter
// w % 4 and the column slice w / 4); warps 16..19 issue the MMAs, one per SM
// sub-partition.  A tile's work is a sequence of 64-column accumulator
// chunks (44, or 48 in the split and rows modes) cycled through a ring of four TMEM
// buffers; mbarriers hand chunks between the MMA warps and the epilogue
// warps, and the epilogue hands a buffer back as soon as its TMEM loads have
// landed.  The next tile's input is loaded while the current tile's last
// stages run.  Every wait is bounded: on timeout the kernel records
// FFTCONV_ERR_TIMEOUT in the plan's status word, drains, frees its TMEM and
// returns.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cmath>
#include <complex>
#include <cstring>
#include <type_traits>
#include <vector>

#include "common.cuh"
#include "internal.h"
#include "simt_fft.cuh"   // perm_to_freq: the order of the staged row pass
#include "tc_ptx.cuh"

namespace fftconv {

cudaError_t simt_precompute_to_tc_layout(const Plan& p, const void* k, void* Kf, cudaStream_t s);
cudaError_t simt_precompute_to_tc_split(const Plan& p, const void* k, void* Kf, cudaStream_t s);

namespace {

using namespace tc;

constexpr int kN = 4096;          // window length (inputs and outputs per transform)
constexpr int kM = 8192;          // transform length
constexpr int kHop = 2048;        // overlap-save hop for longer sequences
constexpr int kEpiWarps = 16;
constexpr int kMmaWarps = 4;     // one MMA issuer per SMSP; issuer i owns accumulator buffer i
constexpr int kThreads = (kEpiWarps + kMmaWarps) * 32;
constexpr int kDBuf = 4;             // accumulator ring: 4 buffers of 64 TMEM columns

// Kernel modes.  0: sequences of 4096 (one zero-padded 8192-point transform
// per sequence, first 4096 outputs).  1: overlap-save windows of 4096 for
// longer sequences with short filters.  2: sequences of 8192 with full-length
// filters through the 16384-point spectrum split by bin parity (see
// pair_info): the 8192-point transform then takes all 8192 inputs and returns
// all 8192 outputs.
// 3 (rows): the row pass of the staged path, M = R x 8192: full-length
// 8192-point transforms of complex workspace rows, product with that row's
// part of the spectrum, inverse, written back in place.
constexpr int kModePlain = 0, kModeWindows = 1, kModeSplit = 2, kModeRows = 3;
constexpr int kModeBlocks4 = 4;     // N = 16384: four blocks of 4096 per pair (tc_planar.cu)

// chunk c of a tile -> stage (0 S1, 1 S2, 2 S3, 3 S3', 4 S2', 5 S1') and index
__host__ __device__ __forceinline__ int chunk_stage(int c) { return c < 40 ? (c >> 3) : 5; }
__host__ __device__ __forceinline__ int chunk_index(int c) { return c < 40 ? (c & 7) : c - 40; }
// Ordering.  An epilogue warp releases an accumulator buffer as soon as its
// TMEM loads have landed in registers, before the math and the stores, so
// the MMA for chunk c + 4 can start early.  Because every epilogue warp works
// through its chunks in order, "buffer of chunk c released" still implies
// that all the work of the chunks before c's pair is done (stores fenced),
// which covers most data dependencies.  The chunks that regroup the data
// need whole stages instead, signalled by per-tile stage barriers: the first
// S3 chunks (16..19) need all of E2, the first S2' chunks (32..35) all of
// E3', and the S1' chunk for j3 = 6, 7 (43) the last E2' pair.  Returns
// the stage barrier chunk c waits for, or -1.  With several MMA issuers this
// must be explicit: chunks of one stage are issued independently.
__host__ __device__ __forceinline__ int chunk_stage_barrier(int c) {
    if (c >= 16 && c < 20) return 0;
    if (c >= 32 && c < 36) return 1;
    if (c == 43) return 2;
    return -1;
}
constexpr uint32_t kWaitLimit = 1u << 20;

// shared-memory map (bytes from a 1024-aligned base) and per-mode sizes
constexpr int kTile = 16384;                 // 128 rows x 128 B, 128-byte swizzle
constexpr int kKBytes = kM * 4;              // one filter spectrum row, 8192 x half2
template <int MODE>
struct Lay {
    static constexpr bool kFull = MODE == kModeSplit || MODE == kModeRows;   // all 8192 inputs and outputs
    static constexpr bool kSplit = MODE == kModeSplit;  // even/odd bin tiles
    static constexpr int kJ1 = kFull ? 32 : 16;         // nonzero inputs / kept outputs per j3
    static constexpr int OffData = 0;                   // 8 tiles (one per j3)
    static constexpr int OffBS1 = 8 * kTile;            // K=2*kJ1 N=64        4 / 8 KB
    static constexpr int OffBS2 = OffBS1 + kJ1 * 256;   // K=64 N=64           8 KB
    static constexpr int OffBS3 = OffBS2 + 8192;        // 32 x (K=16 N=16)    16 KB
    static constexpr int OffBS3i = OffBS3 + 16384;      // 32 x (K=16 N=16)    16 KB
    static constexpr int OffBS2i = OffBS3i + 16384;     // K=64 N=64           8 KB
    static constexpr int OffBS1i = OffBS2i + 8192;      // K=64 N=2*kJ1        4 / 8 KB
    static constexpr int OffBEnd = OffBS1i + kJ1 * 256;
    static constexpr int BImageBytes = OffBEnd - OffBS1;
    static constexpr int OffK = OffBEnd;                // the tile's filter spectrum row
    // (the rows mode has four filter rows per tile, read through L2)
    static constexpr bool kKShared = MODE != kModeRows;
    // the 256-entry w8192 twiddle table lives in shared memory except in the
    // split mode, whose larger factors leave no room (it is read through L1)
    static constexpr bool kTwShared = !kSplit;
    static constexpr int OffTwM = OffK + (kKShared ? kKBytes : 0);
    static constexpr int OffBars = OffTwM + (kTwShared ? 2048 : 0);   // 16 mbarrier slots
    static constexpr int OffMisc = OffBars + 128;       // tmem base, abort flag
    static constexpr int SmemBytes = OffMisc + 64 + 1024;              // + alignment slack
    static constexpr int Chunks = kFull ? 48 : 44;      // 8 per stage S1..S2', S1' 4 or 8
};
static_assert(Lay<kModeSplit>::SmemBytes <= 232448, "shared memory");
static_assert(Lay<kModeRows>::SmemBytes <= 232448, "shared memory");
static_assert(Lay<kModePlain>::SmemBytes <= 232448, "shared memory");

// byte offset of element (n, k) of a K x N B operand in the no-swizzle
// K-major layout used for every DFT factor: 8x8 core matrices, K-halves
// LBO = (N/8)*128 bytes apart, 8-row groups 128 bytes apart.
inline size_t bimg_offset(int n, int k, int N) {
    return (size_t)(k / 8) * (N / 8) * 128 + (size_t)(n / 8) * 128 + (n % 8) * 16 + (k % 8) * 2;
}

// A twiddle in packed half precision (see cmul_h).
struct Tw16 {
    uint32_t p, q;
};

struct TcArgs {
    const void* u;
    const void* w;
    const void* v;
    void* y;
    const __half2* Kh16;       // rows of 8192 complex fp16 (see k16_index): [H] unnormalised / scale;
                               // split mode [2H] (even, odd bins); rows mode [H * R], spectrum / M / scale
    const float* Kscale;       // the rows' scales: [H] per channel ([H * R] per row in rows mode)
    const uint8_t* mask;
    int64_t mask_h;
    int64_t B, H;
    int64_t N;                 // sequence length (row stride of u, w, v, y)
    int64_t nwin;              // windows per sequence (1 for N = 4096)
    int64_t pb;                // pairs per channel, ceil(B/2)
    int64_t tpc;               // tiles per window, ceil(pb/4)
    int64_t nunits;            // H * nwin * tpc
    const uint4* bimg;         // DFT factors, image of the shared-memory region
    const float2* tw1024;      // exp(-2 pi i e/1024), e < 1024
    const Tw16* twM16;         // exp(-2 pi i e/8192), e < 256, as half2 pairs
    const float2* tw16k;       // split mode: exp(-2 pi i t/16384), t < 8192
    float2 w16k_j3[8];         // split mode: exp(-2 pi i j/16384), j < 8
    uint4* scratch;            // split mode: [CTAs][4 pairs][8192] half2, z_even of the group
    uint4* work;               // rows mode: the staged workspace [pairs][R][8192] complex fp16
    int64_t R;                 // rows mode: rows per pair
    int64_t pair0;             // rows mode: first pair of this chunk
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

// Twiddle products in packed half precision.  A twiddle t = (tr, ti) is held
// as the two half2 values tp = (tr, ti) and tq = (-ti, tr); then
//   x t = re(x) tp + im(x) tq,   x conj(t) = re(x) tp* + im(x) tq*
// with tp* = (tr, -ti) and tq* = (ti, tr), each a sign flip of one half.
__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u2h(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }
__device__ __forceinline__ Tw16 tw16(float2 t) {
    return {h2u(__floats2half2_rn(t.x, t.y)), h2u(__floats2half2_rn(-t.y, t.x))};
}
__device__ __forceinline__ Tw16 tw16_conj(Tw16 t) { return {t.p ^ 0x80000000u, t.q ^ 0x00008000u}; }
// x (fp32 accumulator pair) rounded to fp16, times t; returns packed fp16
__device__ __forceinline__ uint32_t cmul_h(uint32_t xr, uint32_t xi, Tw16 t) {
    const __half2 x = __floats2half2_rn(__uint_as_float(xr), __uint_as_float(xi));
    return h2u(__hfma2(__low2half2(x), u2h(t.p), __hmul2(__high2half2(x), u2h(t.q))));
}

// 128-byte swizzle of a logical byte offset inside a 1024-byte-aligned tile
__device__ __forceinline__ uint32_t swz(uint32_t off) { return off ^ (((off >> 7) & 7u) << 4); }

struct PairInfo {
    int64_t o0, o1;      // element offsets of the window in rows b0 and b1 (o1 < 0: absent)
    int64_t h;
    bool valid;
    bool tail_only;      // only window positions t >= kHop are outputs
    bool odd;            // split mode: the tile of odd spectrum bins
    int64_t krow;        // rows mode: this quarter's filter row (channel * R + row)
};

// A tile holds 4 pairs of batch rows of ONE channel and one window: unit u
// covers channel u / (nwin*tpc), window j = (u / tpc) % nwin and pairs
// 4*(u % tpc) + q, q < 4 (pairs past ceil(B/2) are empty).
//
// Overlap-save (sequences longer than 4096, filters of L <= 2049 taps): the
// kernel's transform gives the first 4096 outputs of the linear convolution
// of a 4096-sample window with the filter, exact wherever the filter's whole
// history lies inside the window, i.e. from window position L - 1 on.
// Window j starts at 2048 j; window 0 keeps all 4096 outputs (there is no
// history before t = 0), window j > 0 keeps positions [2048, 4096), i.e.
// y[2048 (j+1), 2048 (j+2)).  N / 2048 - 1 windows cover the sequence.
// Tile indices fit in 32 bits (the host rejects launches of 2^31 tiles or
// more), so the decomposition uses 32-bit division.  In the plain mode the
// row stride and the window are fixed.
template <int MODE>
__device__ __forceinline__ PairInfo pair_info(const TcArgs& a, int64_t unit, int q) {
    PairInfo p;
    if constexpr (MODE == kModePlain) {
        p.h = unit / a.tpc;
        const int64_t bp = 4 * (unit % a.tpc) + q;
        p.valid = bp < a.pb;
        p.tail_only = false;
        p.odd = false;
        const int64_t b0 = 2 * (p.valid ? bp : 0), b1 = b0 + 1;
        p.o0 = (b0 * a.H + p.h) * kN;
        p.o1 = (p.valid && b1 < a.B) ? (b1 * a.H + p.h) * kN : -1;
        return p;
    }
    if constexpr (MODE == kModeRows) {
        // Rows mode: unit u is pair u / (R/4) of the chunk and rows
        // c = 4 (u % (R/4)) + q; o0 indexes the workspace row (complex).
        const int64_t qpr = a.R / 4;
        const int64_t pl = unit / qpr, c = 4 * (unit - pl * qpr) + q;
        p.h = (a.pair0 + pl) / a.pb;
        p.valid = true;
        p.tail_only = false;
        p.odd = false;
        p.o0 = (pl * a.R + c) * (int64_t)kM;
        p.o1 = -1;
        p.krow = p.h * a.R + c;
        return p;
    }
    if constexpr (MODE == kModeSplit) {
        // Split mode (N = 8192, full-length filter).  With M = 16384 and x zero
        // for t >= 8192, X(2f) is the 8192-point transform of x and X(2f+1)
        // that of x[t] w16384^t; the output is
        //   y[t] = (z_even[t] + w16384^-t z_odd[t]) / 2,
        // z_e the inverse 8192-point transform of X(2f+e) K(2f+e) (unitary
        // factors, unnormalised K).  Unit u is group u / 2 (4 pairs of one
        // channel) and parity u % 2; a CTA takes both parities of a group
        // back to back, parking z_even in its scratch slot for the odd tile.
        const int64_t g = unit >> 1;
        p.h = g / a.tpc;
        const int64_t bp = 4 * (g % a.tpc) + q;
        p.valid = bp < a.pb;
        p.tail_only = false;
        p.odd = unit & 1;
        const int64_t b0 = 2 * (p.valid ? bp : 0), b1 = b0 + 1;
        p.o0 = (b0 * a.H + p.h) * a.N;
        p.o1 = (p.valid && b1 < a.B) ? (b1 * a.H + p.h) * a.N : -1;
        return p;
    }
    const uint32_t un = (uint32_t)unit, tpc = (uint32_t)a.tpc, per_ch = (uint32_t)a.nwin * tpc;
    const uint32_t h = un / per_ch;
    const uint32_t rem = un - h * per_ch;
    const uint32_t j = rem / tpc;
    p.h = h;
    const int64_t bp = 4 * (int64_t)(rem - j * tpc) + q;
    p.valid = bp < a.pb;
    p.tail_only = j > 0;
    p.odd = false;
    const int64_t b0 = 2 * (p.valid ? bp : 0), b1 = b0 + 1;
    p.o0 = (b0 * a.H + p.h) * a.N + kHop * j;
    p.o1 = (p.valid && b1 < a.B) ? (b1 * a.H + p.h) * a.N + kHop * j : -1;
    return p;
}

// A CTA's first unit and the one after `u` (the split mode takes the two
// parity tiles of a group back to back).
template <int MODE>
__device__ __forceinline__ int64_t first_unit() {
    return MODE == kModeSplit ? 2 * (int64_t)blockIdx.x : (int64_t)blockIdx.x;
}
template <int MODE>
__device__ __forceinline__ int64_t next_unit(int64_t u) {
    if constexpr (MODE == kModeSplit) return (u & 1) ? u + 2 * (int64_t)gridDim.x - 1 : u + 1;
    return u + gridDim.x;
}
// The tile's channel, and its filter row in K_f (the split mode stores the
// even and the odd bins of each channel as two rows).
template <int MODE>
__device__ __forceinline__ int64_t unit_channel(const TcArgs& a, int64_t u) {
    if constexpr (MODE == kModeRows) return (a.pair0 + u / (a.R / 4)) / a.pb;
    if constexpr (MODE == kModeWindows) return (int64_t)((uint32_t)u / ((uint32_t)a.nwin * (uint32_t)a.tpc));
    if constexpr (MODE == kModeSplit) return (u >> 1) / a.tpc;
    return u / a.tpc;
}
template <int MODE>
__device__ __forceinline__ int64_t unit_filter_row(const TcArgs& a, int64_t u) {
    return MODE == kModeSplit ? 2 * unit_channel<MODE>(a, u) + (u & 1) : unit_channel<MODE>(a, u);
}

// position of spectrum value f = c1 + 32 c2 + 1024 c3 in a channel's fp16 row:
// 16-byte groups of four c3 values, consecutive c1 in consecutive groups, so a
// warp (c1 = lane) reads 512 contiguous bytes per (c2, c3 half)
__host__ __device__ __forceinline__ int k16_index(int c1, int c2, int c3) {
    return ((c2 * 2 + (c3 >> 2)) * 32 + c1) * 4 + (c3 & 3);
}

template <typename T, int MODE>
__global__ void __launch_bounds__(kThreads, 1) tc_fftconv_n4096_kernel(TcArgs a) {
    using LY = Lay<MODE>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t* bar = (uint64_t*)(smem + LY::OffBars);
    uint64_t* bar_in = bar + 0;    // the tile's input is in TMEM (16 epilogue warps)
    uint64_t* dfull = bar + 1;     // [kDBuf] accumulator buffer written (tcgen05.commit)
    uint64_t* dfree = bar + 5;     // [kDBuf] accumulator buffer drained (16 epilogue warps)
    uint64_t* bar_fin = bar + 9;   // every MMA has completed (drain before exit)
    uint64_t* bar_k = bar + 10;    // the tile's filter row has landed in shared memory
    uint64_t* bar_stage = bar + 11;   // [3] E2, E3', E2' done for the tile (16 epilogue warps)
    uint32_t* tmem_base_sh = (uint32_t*)(smem + LY::OffMisc);
    volatile int* abort_flag = (volatile int*)(smem + LY::OffMisc + 4);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
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
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kEpiWarps) tmem_alloc(tmem_base_sh, 512);   // the first MMA warp owns TMEM
    // DFT factors and the w8192 twiddle table into shared memory
    {
        uint4* dst = (uint4*)(smem + LY::OffBS1);
        for (int i = tid; i < LY::BImageBytes / 16; i += kThreads) dst[i] = __ldg(&a.bimg[i]);
        if constexpr (LY::kTwShared) {
            Tw16* t2 = (Tw16*)(smem + LY::OffTwM);
            for (int i = tid; i < 256; i += kThreads) t2[i] = a.twM16[i];
        }
    }
    const Tw16* stwM = LY::kTwShared ? (const Tw16*)(smem + LY::OffTwM) : a.twM16;
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

    if (warp >= kEpiWarps) {
        // ============================ MMA issuers ===========================
        // A single thread can issue a tcgen05.mma only every ~100 cycles, far
        // slower than the tensor core retires these small MMAs, so four warps
        // issue: issuer i handles the chunks c = i (mod 4) of every tile, which
        // all use ring buffer i.
        const int issuer = warp - kEpiWarps;
        const uint32_t id64 = idesc_f16_f32(128, 64);
        const uint32_t id16 = idesc_f16_f32(128, 16);
        const uint32_t id32 = idesc_f16_f32(128, 32);
        // descriptor bases (start address in 16-byte units in the low bits)
        const uint64_t dS1 = make_desc(sbase + LY::OffBS1, 1024, 128, 0);    // K-step: +2048 B
        const uint64_t dS2 = make_desc(sbase + LY::OffBS2, 1024, 128, 0);    // K-step: +2048 B
        const uint64_t dS2i = make_desc(sbase + LY::OffBS2i, 1024, 128, 0);
        const uint64_t dS3 = make_desc(sbase + LY::OffBS3, 256, 128, 0);     // per c2: +512 B
        const uint64_t dS3i = make_desc(sbase + LY::OffBS3i, 256, 128, 0);
        // S1' factor: N = 2 kJ1 columns (LBO = kJ1 * 32 B); a 32-column half
        // is +512 B, a K step +kJ1 * 64 B
        const uint64_t dS1i = make_desc(sbase + LY::OffBS1i, LY::kJ1 * 32, 128, 0);
        const uint64_t dA = make_desc(sbase + LY::OffData, 16, 1024, 2);     // tile: +16384 B, K-step: +32 B
        uint32_t g = 0;          // global chunk counter (accumulator buffer g % kDBuf)
        int iter = 0;
        int k_issued = 0;        // filter-row copies issued
        bool ok = true;
        g = issuer;
        for (int64_t unit = first_unit<MODE>(); unit < a.nunits && ok; unit = next_unit<MODE>(unit), ++iter) {
            if (!wait(bar_in, iter & 1)) { ok = false; fail(); break; }
            tc_fence_after();
            if (issuer == 0 && MODE != kModeRows) {      // (rows mode reads its filter rows through L2)
                if (lane == 0) {
                    // the previous tile is finished with the filter buffer (its
                    // epilogue warps arrived on bar_in after all their reads)
                    mbar_expect_tx(bar_k, kKBytes);
                    bulk_copy_g2s(smem + LY::OffK, a.Kh16 + unit_filter_row<MODE>(a, unit) * kM, kKBytes, bar_k);
                }
                ++k_issued;
                __syncwarp();
            }
#pragma unroll 1
            for (int c = issuer; c < LY::Chunks && ok; c += kMmaWarps, g += kMmaWarps) {
                const int stage = chunk_stage(c), k = chunk_index(c);
                const uint32_t b = g % kDBuf;
                // the buffer's previous contents must have been drained ...
                if (g >= kDBuf && !wait(&dfree[b], ((g - kDBuf) / kDBuf) & 1)) { ok = false; fail(); break; }
                // ... and chunks that regroup the data need whole stages
                const int sb = chunk_stage_barrier(c);
                if (sb >= 0 && !wait(&bar_stage[sb], iter & 1)) { ok = false; fail(); break; }
                tc_fence_after();
                if (lane == 0) {
                    // descriptors are loop-invariant bases plus an offset in
                    // 16-byte units added to the start-address field
                    const uint32_t d = tbase + 256 + 64 * b;
                    if (stage == 0) {            // S1: A1 (TMEM) cols j3*kJ1 + j1, j3 = k
#pragma unroll
                        for (int ks = 0; ks < LY::kJ1 / 8; ++ks)
                            mma_ts(d, tbase + k * LY::kJ1 + 8 * ks, dS1 + 128 * ks, id64, ks);
                    } else if (stage == 1 || stage == 4) {   // S2 / S2': smem tile j3 = k
                        const uint64_t db = stage == 1 ? dS2 : dS2i;
                        const uint64_t da = dA + (uint64_t)(k * (kTile >> 4));
#pragma unroll
                        for (int s = 0; s < 4; ++s) mma_ss(d, da + 2 * s, db + 128 * s, id64, s);
                    } else if (stage == 2 || stage == 3) {   // S3 / S3': TMEM cols c2*8 + j3|c3
                        const uint64_t db = (stage == 2 ? dS3 : dS3i) + (uint64_t)(4 * k * 32);
#pragma unroll
                        for (int cl = 0; cl < 4; ++cl) mma_ts(d + cl * 16, tbase + (4 * k + cl) * 8, db + 32 * cl, id16, 0);
                    } else {                     // S1': j3 = 2(k%4) + jl, j1 in [16h, 16h+16), h = k/4 (N = 32)
                        const uint64_t da = dA + (uint64_t)(2 * (k & 3) * (kTile >> 4));
                        const uint64_t db = dS1i + (uint64_t)(32 * (k >> 2));
#pragma unroll
                        for (int jl = 0; jl < 2; ++jl) {
#pragma unroll
                            for (int s = 0; s < 4; ++s)
                                mma_ss(d + jl * 32, da + jl * (kTile >> 4) + 2 * s, db + LY::kJ1 * 4 * s, id32, s);
                        }
                    }
                    tc_commit(&dfull[b]);
                }
                __syncwarp();
                if (c == issuer + 12) {
                    // warm L2 with the next tile's rows (u, w, v of both
                    // sequences of each pair, and the filter spectrum) while
                    // this tile is being transformed: issuer i takes pair i.
                    // Each bulk prefetch occupies the issuing warp for a
                    // while, so they are spread over the four issuers, at
                    // their last S2 chunk; measured against one warp at the
                    // tile start, 3.5% faster overall (and 7% faster than no
                    // prefetch).
                    const void* pf_src = nullptr;
                    uint32_t pf_bytes = (MODE == kModeSplit ? 2 * kN : kN) * sizeof(T);
                    const int64_t nu = next_unit<MODE>(unit);
                    if (MODE != kModeRows && nu < a.nunits && (lane >> 3) == issuer) {
                        const PairInfo Q = pair_info<MODE>(a, nu, issuer);
                        const int which = lane & 7;
                        if (Q.valid) {
                            if (which == 0) pf_src = (const T*)a.u + Q.o0;
                            else if (which == 1 && a.w) pf_src = (const T*)a.w + Q.o0;
                            else if (which == 2 && a.v) pf_src = (const T*)a.v + Q.o0;
                            else if (which == 3 && Q.o1 >= 0) pf_src = (const T*)a.u + Q.o1;
                            else if (which == 4 && Q.o1 >= 0 && a.w) pf_src = (const T*)a.w + Q.o1;
                            else if (which == 5 && Q.o1 >= 0 && a.v) pf_src = (const T*)a.v + Q.o1;
                            else if (which == 6 && issuer == 0) {
                                pf_src = a.Kh16 + unit_filter_row<MODE>(a, nu) * kM;
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
        // the convolution's length and transform length (mask bins)
        // (rows mode: the plan's N, M = R x 8192)
        constexpr int kSeqN = LY::kFull ? 2 * kN : kN, kSeqM = 2 * kSeqN;
        const int64_t nblk = (MODE == kModeRows ? a.N : kSeqN) / 32;

        // w1024^(c1 l) with (c1, l) = (8s + i, lane) in E1 and (lane, 8s + i)
        // in E2' -- the same eight values, kept in registers; wM^(c1 j3) with
        // c1 = lane in E2 and E3' comes from the shared-memory table
        Tw16 tw[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) tw[i] = tw16(__ldg(&a.tw1024[((8 * s + i) * lane) & 1023]));

        // ---- load: x = u*w for t = 256*j1 + 8*l + j3, j1 in [J s, J s + J)
        // with J = kJ1 / 4 (split mode: times w16384^t in the odd tile), into
        // the TMEM A1 columns; then arrive on bar_in.  Loads are issued in
        // batches before any use (absent rows or gates read a present row and
        // are masked afterwards).  A tile's input is loaded while the previous
        // tile's last stage runs (the A columns are free once S3' is done), so
        // its first MMAs can start as soon as the accumulator ring drains.
        // part 0 loads the first half of the j1 batches, part 1 the second
        // half and then signals bar_in; the two halves fill the waits before
        // S2' and before S1' of the previous tile.
        auto load_tile = [&](int64_t lu, int part) {
            const PairInfo LP = pair_info<MODE>(a, lu, q);
            const bool hasL = LP.o1 >= 0;
            const int64_t oo1 = hasL ? LP.o1 : LP.o0;
            const T* pu0 = (const T*)a.u + LP.o0;
            const T* pw0 = a.w ? (const T*)a.w + LP.o0 : pu0;
            const T* pu1 = (const T*)a.u + oo1;
            const T* pw1 = a.w ? (const T*)a.w + oo1 : pu1;
            const bool has_w = a.w != nullptr;
            const bool keep0 = LP.valid, keep1 = hasL;
            constexpr int J = LY::kJ1 / 4;
            constexpr int kHalf = J / 4;      // batches of two j1 per part
#pragma unroll
            for (int jq = 0; jq < kHalf; ++jq) {
                const int jp = part * kHalf + jq;
                uint32_t pk[8][2];
                if constexpr (MODE == kModeRows) {
                    // complex fp16 workspace row, already scaled: eight
                    // consecutive t per j1 (two 16-byte loads)
#pragma unroll
                    for (int jh = 0; jh < 2; ++jh) {
                        const uint4* src = a.work + (LP.o0 + 256 * (J * s + 2 * jp + jh) + 8 * lane) / 4;
                        const uint4 x0 = __ldg(src), x1 = __ldg(src + 1);
                        pk[0][jh] = x0.x; pk[1][jh] = x0.y; pk[2][jh] = x0.z; pk[3][jh] = x0.w;
                        pk[4][jh] = x1.x; pk[5][jh] = x1.y; pk[6][jh] = x1.z; pk[7][jh] = x1.w;
                    }
                } else {
                uint4 ld[2][4];
                if constexpr (LY::kSplit) {
                    // the even tile's rows are read again by the odd tile one
                    // tile later: keep them in L2 until then
                    const uint64_t pol = LP.odd ? l2_evict_first() : l2_evict_last();
#pragma unroll
                    for (int jh = 0; jh < 2; ++jh) {
                        const int64_t t0 = 256 * (J * s + 2 * jp + jh) + 8 * lane;
                        ld[jh][0] = ldg_nc_hint(pu0 + t0, pol);
                        ld[jh][1] = ldg_nc_hint(pw0 + t0, pol);
                        ld[jh][2] = ldg_nc_hint(pu1 + t0, pol);
                        ld[jh][3] = ldg_nc_hint(pw1 + t0, pol);
                    }
                } else {
#pragma unroll
                    for (int jh = 0; jh < 2; ++jh) {
                        const int64_t t0 = 256 * (J * s + 2 * jp + jh) + 8 * lane;
                        ld[jh][0] = __ldg((const uint4*)(pu0 + t0));
                        ld[jh][1] = __ldg((const uint4*)(pw0 + t0));
                        ld[jh][2] = __ldg((const uint4*)(pu1 + t0));
                        ld[jh][3] = __ldg((const uint4*)(pw1 + t0));
                    }
                }
#pragma unroll
                for (int jh = 0; jh < 2; ++jh) {
                    float2 w0 = make_float2(1.f, 0.f);     // w16384^t0 (odd split tile)
                    if constexpr (LY::kSplit) {
                        if (LP.odd) w0 = __ldg(&a.tw16k[256 * (J * s + 2 * jp + jh) + 8 * lane]);
                    }
                    const uint32_t ua[4] = {ld[jh][0].x, ld[jh][0].y, ld[jh][0].z, ld[jh][0].w};
                    const uint32_t wa[4] = {ld[jh][1].x, ld[jh][1].y, ld[jh][1].z, ld[jh][1].w};
                    const uint32_t ub[4] = {ld[jh][2].x, ld[jh][2].y, ld[jh][2].z, ld[jh][2].w};
                    const uint32_t wb[4] = {ld[jh][3].x, ld[jh][3].y, ld[jh][3].z, ld[jh][3].w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float2 xa = IO<T>::unpack2(ua[e]), xb = IO<T>::unpack2(ub[e]);
                        if (has_w) {
                            const float2 g0 = IO<T>::unpack2(wa[e]), g1 = IO<T>::unpack2(wb[e]);
                            xa.x *= g0.x; xa.y *= g0.y; xb.x *= g1.x; xb.y *= g1.y;
                        }
                        if (!keep0) xa = make_float2(0.f, 0.f);
                        if (!keep1) xb = make_float2(0.f, 0.f);
                        if constexpr (LY::kSplit) {
                            if (LP.odd) {
                                // (a + i b)[t] times w16384^t, t = t0 + 2e (+1)
                                const float2 wa0 = cmul(w0, a.w16k_j3[2 * e]), wa1 = cmul(w0, a.w16k_j3[2 * e + 1]);
                                const float2 z0 = cmul(make_float2(xa.x, xb.x), wa0);
                                const float2 z1 = cmul(make_float2(xa.y, xb.y), wa1);
                                xa = make_float2(z0.x, z1.x);
                                xb = make_float2(z0.y, z1.y);
                            }
                        }
                        pk[2 * e][jh] = pack_h2(xa.x, xb.x);
                        pk[2 * e + 1][jh] = pack_h2(xa.y, xb.y);
                    }
                }
                }
#pragma unroll
                for (int j3 = 0; j3 < 8; ++j3)
                    tmem_st2(tbase + lq + j3 * LY::kJ1 + J * s + 2 * jp, pk[j3][0], pk[j3][1]);
            }
            if (part == 1) {
                tc_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_in);
            }
        };

        int iter = 0;
        bool ok = true;
        float nf = 0.f;          // non-finite detector over the outputs (fp16 range)
        if (first_unit<MODE>() < a.nunits) {
            load_tile(first_unit<MODE>(), 0);
            load_tile(first_unit<MODE>(), 1);
        }
        for (int64_t unit = first_unit<MODE>(); unit < a.nunits && ok; unit = next_unit<MODE>(unit), ++iter) {
            const int64_t hch = unit_channel<MODE>(a, unit);

            // (this tile's input was loaded before the loop or during the
            // previous tile's last stage: see load_tile)
            const PairInfo P = pair_info<MODE>(a, unit, q);
            const bool has1 = P.o1 >= 0;

            const __half2* Ks = (const __half2*)(smem + LY::OffK);
            // loaded once per tile and pinned in a register (an opaque move
            // keeps the compiler from re-issuing the global load at each use)
            float kscale = MODE == kModeRows ? 1.f : __ldg(&a.Kscale[hch]);   // (rows: applied by the column pass)
            asm volatile("mov.b32 %0, %0;" : "+f"(kscale));
            const uint8_t* mrow = a.mask ? a.mask + (a.mask_h == 1 ? 0 : hch) * nblk : nullptr;

            // Accumulator chunks are handled in pairs (c, c+1) of one stage:
            // both are waited for and loaded before one TMEM-load wait, and
            // the fences and barrier arrivals are shared.  Each stage has its
            // own loop, so the stage, the ring slots (chunk c of a tile uses
            // buffer c % 4) and the store patterns are fixed at compile time.
            auto begin_pair = [&](int c) -> bool {
                // use number (Chunks/4)*iter + c/4 of the buffer
                const uint32_t par = (uint32_t)(iter * (LY::Chunks / 4) + (c >> 2)) & 1u;
                if (!wait(&dfull[c & 3], par) || !wait(&dfull[(c & 3) + 1], par)) {
                    fail();
                    return false;
                }
                tc_fence_after();
                return true;
            };
            // the pair's accumulators are in registers: hand the buffers back
            auto release = [&](int c) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&dfree[c & 3]);
                    mbar_arrive(&dfree[(c & 3) + 1]);
                }
            };
            // this warp's part of a whole stage is written (TMEM stores waited
            // for, shared-memory stores fenced for the async proxy)
            auto stage_done = [&](int i) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar_stage[i]);
            };
            auto dcol = [&](int c) -> uint32_t { return tbase + lq + 256 + 64 * (c & 3); };

            // E1 (S1 -> S2): lane = l; columns c1 = 8s + i of j3 = k + cc;
            //   twiddle w1024^(c1 l); A2 tile j3, row 32q + c1, K pair 2l.
            // E2' (S2' -> S1'): lane = c1; columns l = 8s + i of j3;
            //   twiddle conj w1024^(c1 l); A6 tile j3, row 32q + l, K pair 2c1.
            // The same eight twiddles and the same store pattern.
            auto e_transpose = [&](int c, int k) {
                uint32_t r[2][16];
                tmem_ld16(dcol(c) + 16 * s, r[0]);
                tmem_ld16(dcol(c + 1) + 16 * s, r[1]);
                tc_wait_ld();
                release(c);
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    uint8_t* tile = smem + LY::OffData + (k + cc) * kTile + (4 * q + s) * 1024;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        *(uint32_t*)(tile + i * 128 + ((4 * lane) ^ (i << 4))) = cmul_h(r[cc][2 * i], r[cc][2 * i + 1], tw[i]);
                    }
                }
                fence_proxy_async_smem();
            };

#pragma unroll 1
            for (int k = 0; k < 8; k += 2) {
                if (!(ok = begin_pair(k))) break;
                e_transpose(k, k);
            }
            // E2: lane = c1; columns c2 = 8s + i of j3 = k, k+1; twiddle
            // wM^(c1 j3); A3 (TMEM) cols c2*8 + j3 (two adjacent columns)
#pragma unroll 1
            for (int k = 0; k < 8 && ok; k += 2) {
                const int c = 8 + k;
                if (!(ok = begin_pair(c))) break;
                uint32_t r[2][16];
                tmem_ld16(dcol(c) + 16 * s, r[0]);
                tmem_ld16(dcol(c + 1) + 16 * s, r[1]);
                const Tw16 t0 = stwM[lane * k], t1 = stwM[lane * (k + 1)];
                tc_wait_ld();
                release(c);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    tmem_st2(tbase + lq + (8 * s + i) * 8 + k, cmul_h(r[0][2 * i], r[0][2 * i + 1], t0),
                             cmul_h(r[1][2 * i], r[1][2 * i + 1], t1));
                tc_wait_st();
            }
            if (ok) stage_done(0);
            // EK: lane = c1; columns c3 of c2 = 4(k+cc) + s; times the filter
            // spectrum row in its fp16 form K/scale (|K/scale| <= 1, so the
            // inverse stages see values no larger than the forward output);
            // the channel scale is applied to y in fp32.  A4 (TMEM) cols
            // c2*8 + c3 (in place)
            if (MODE != kModeRows && ok && !(ok = wait(bar_k, iter & 1))) fail();
#pragma unroll 1
            for (int k = 0; k < 8 && ok; k += 2) {
                const int c = 16 + k;
                // rows mode: this quarter's filter row comes through L2 (or
                // HBM); the loads are issued before the accumulator wait so
                // that their latency overlaps it
                [[maybe_unused]] uint4 kpre[2][2];
                if constexpr (MODE == kModeRows) {
                    const __half2* Kq = a.Kh16 + P.krow * (int64_t)kM;
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        kpre[cc][0] = __ldg((const uint4*)(Kq + k16_index(lane, 4 * (k + cc) + s, 0)));
                        kpre[cc][1] = __ldg((const uint4*)(Kq + k16_index(lane, 4 * (k + cc) + s, 4)));
                    }
                }
                if (!(ok = begin_pair(c))) break;
                uint32_t r[2][16];
                tmem_ld16(dcol(c) + 16 * s, r[0]);
                tmem_ld16(dcol(c + 1) + 16 * s, r[1]);
                tc_wait_ld();
                release(c);
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const int c2 = 4 * (k + cc) + s;
                    uint4 k0, k1;
                    if constexpr (MODE == kModeRows) {
                        k0 = kpre[cc][0];
                        k1 = kpre[cc][1];
                    } else {
                        k0 = *(const uint4*)(Ks + k16_index(lane, c2, 0));
                        k1 = *(const uint4*)(Ks + k16_index(lane, c2, 4));
                    }
                    uint32_t kw[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
                    if (mrow) {
                        // frequency-sparse filter: zero the masked bins (f and
                        // its mirror M - f share one rfft bin)
#pragma unroll
                        for (int c3 = 0; c3 < 8; ++c3) {
                            const int f8 = lane + 32 * c2 + 1024 * c3;
                            int blk;
                            if constexpr (MODE == kModeRows) {
                                // bin c + R f8 of the 2N-point spectrum, c = this
                                // row (krow mod R, R a power of two; 2N <= 2^23)
                                const int f = (int)((uint32_t)P.krow & (uint32_t)(a.R - 1)) + (int)a.R * f8;
                                blk = (f <= (int)a.N ? f : 2 * (int)a.N - f) >> 5;
                            } else {
                                const int f = LY::kSplit ? 2 * f8 + (int)(unit & 1) : f8;   // bin of the full spectrum
                                blk = (f <= kSeqN ? f : kSeqM - f) >> 5;
                            }
                            blk = blk < (int)nblk ? blk : (int)nblk - 1;
                            if (__ldg(&mrow[blk]) == 0) kw[c3] = 0u;
                        }
                    }
                    uint32_t h8[8];
#pragma unroll
                    for (int c3 = 0; c3 < 8; ++c3) {
                        // x K = re(K) (xr, xi) + im(K) (-xi, xr), packed half
                        const float xr = __uint_as_float(r[cc][2 * c3]), xi = __uint_as_float(r[cc][2 * c3 + 1]);
                        const __half2 x = __floats2half2_rn(xr, xi), xs = __floats2half2_rn(-xi, xr);
                        const __half2 kk = u2h(kw[c3]);
                        h8[c3] = h2u(__hfma2(__low2half2(kk), x, __hmul2(__high2half2(kk), xs)));
                    }
                    tmem_st8(tbase + lq + c2 * 8, h8);
                }
                tc_wait_st();
            }
            // E3': lane = c1; columns (c2 = 4(k+cc) + cl, j3 = 2s + jj);
            // twiddle conj wM^(c1 j3); A5 tile j3, row 32q + c1, K pairs of
            // c2 = 4k..4k+7 as two 16-byte stores
#pragma unroll 1
            for (int k = 0; k < 8 && ok; k += 2) {
                const int c = 24 + k;
                if (!(ok = begin_pair(c))) break;
                uint32_t r[2][4][4];
#pragma unroll
                for (int cc = 0; cc < 2; ++cc)
#pragma unroll
                    for (int cl = 0; cl < 4; ++cl) tmem_ld4(dcol(c + cc) + cl * 16 + 4 * s, r[cc][cl]);
                const Tw16 t0 = tw16_conj(stwM[lane * (2 * s)]), t1 = tw16_conj(stwM[lane * (2 * s + 1)]);
                tc_wait_ld();
                release(c);
                const uint32_t m = 32 * q + lane;
#pragma unroll
                for (int jj = 0; jj < 2; ++jj) {
                    uint8_t* tile = smem + LY::OffData + (2 * s + jj) * kTile;
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        uint32_t hq[4];
#pragma unroll
                        for (int cl = 0; cl < 4; ++cl) hq[cl] = cmul_h(r[cc][cl][2 * jj], r[cc][cl][2 * jj + 1], jj ? t1 : t0);
                        const uint32_t off = (m >> 3) * 1024 + (m & 7) * 128 + 16 * (k + cc);
                        *(uint4*)(tile + swz(off)) = make_uint4(hq[0], hq[1], hq[2], hq[3]);
                    }
                }
                fence_proxy_async_smem();
            }
            if (ok) stage_done(1);
            {
                // first half of the next tile's input (the A columns are free
                // now that S3' is done)
                const int64_t nu = next_unit<MODE>(unit);
                if (ok && nu < a.nunits) load_tile(nu, 0);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) tw[i] = tw16_conj(tw[i]);
#pragma unroll 1
            for (int k = 0; k < 8 && ok; k += 2) {
                const int c = 32 + k;
                if (!(ok = begin_pair(c))) break;
                e_transpose(c, k);
            }
            if (ok) stage_done(2);
#pragma unroll
            for (int i = 0; i < 8; ++i) tw[i] = tw16_conj(tw[i]);
            {
                const int64_t nu = next_unit<MODE>(unit);
                if (ok && nu < a.nunits) load_tile(nu, 1);
            }
            // EO: lane = l; chunk 40 + k holds j3 = 2(k%4) + jl (jl = 0, 1) for
            // j1 in [16 (k/4), 16 (k/4) + 16) at columns jl*32 + 2*(j1 % 16).
            // The four chunks of quad Q (40 + 4Q .. 43 + 4Q) hold all eight j3
            // of that j1 half, so a thread gets the eight consecutive
            // t = 256 j1 + 8 l + j3 of each row: one 16-byte store (512
            // contiguous bytes per warp store).  This warp takes
            // j1 = 16Q + 4s + 2 hf + jj in two halves hf (two j1 each, the
            // register budget of one pass).  Plain and window modes:
            // y = s_h v z.  Split mode: the even tile parks z in the CTA's
            // scratch slot, the odd tile writes y = s_h v (z_even + w16384^-t
            // z_odd) / 2.  In a window after the first, positions t < 2048
            // (j1 < 8: warps with s < 2) are not outputs; their gate loads still
            // read inside the sequence and are discarded.
            // (The split parity is re-derived from the unit where it is used:
            // a flag kept across the stages costs a register they need.)
            const bool odd = LY::kSplit && (unit & 1);
            // One output pass per tile, specialised for parking z_even (split
            // mode, even tile) or writing y: a single loop doing either keeps
            // both paths' state live and spills.
            auto output_pass = [&](auto park_tag) {
                constexpr bool PARK = decltype(park_tag)::value;
                const bool emit = !PARK && P.valid && !(P.tail_only && s < 2);
                const bool park = PARK && P.valid;
#pragma unroll 1
                for (int Q = 0; Q < (LY::Chunks - 40) / 4 && ok; ++Q) {
                    const int c0 = 40 + 4 * Q;
#pragma unroll 1
                    for (int hf = 0; hf < 2 && ok; ++hf) {
                        const int jb = 16 * Q + 4 * s + 2 * hf;      // this pass's first j1
                        // output gate values, requested before the accumulator
                        // wait so that their latency overlaps it (an empty pair
                        // reads row 0 of the channel and discards it)
                        uint4 va[2], vb[2];
                        if (!PARK && MODE != kModeRows) {
                            const T* vr = a.v ? (const T*)a.v : (const T*)a.u;   // any readable row if no gate
#pragma unroll
                            for (int jj = 0; jj < 2; ++jj) {
                                const int64_t t0 = 256 * (jb + jj) + 8 * lane;
                                if constexpr (LY::kSplit) {     // streamed once: leave L2 to the reused rows
                                    const uint64_t pol = l2_evict_first();
                                    va[jj] = ldg_nc_hint(vr + P.o0 + t0, pol);
                                    vb[jj] = ldg_nc_hint(vr + (has1 ? P.o1 : P.o0) + t0, pol);
                                } else {
                                    va[jj] = __ldg((const uint4*)(vr + P.o0 + t0));
                                    vb[jj] = __ldg((const uint4*)(vr + (has1 ? P.o1 : P.o0) + t0));
                                }
                            }
                        }
                        if (hf == 0 && (!(ok = begin_pair(c0)) || !(ok = begin_pair(c0 + 2)))) break;
                        // r[cc][jl][2 jj + (re, im)]: chunk c0 + cc, j3 = 2 cc + jl, j1 = jb + jj
                        uint32_t r[4][2][4];
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc)
#pragma unroll
                            for (int jl = 0; jl < 2; ++jl)
                                tmem_ld4(dcol(c0 + cc) + jl * 32 + 8 * s + 4 * hf, r[cc][jl]);
                        tc_wait_ld();
                        if (hf == 1) {
                            release(c0);
                            release(c0 + 2);
                        }
                        if (park) {
                            uint4* slot = a.scratch + ((int64_t)blockIdx.x * 4 + q) * (kM / 4);
#pragma unroll
                            for (int jj = 0; jj < 2; ++jj) {
                                uint32_t hz[8];
#pragma unroll
                                for (int j3 = 0; j3 < 8; ++j3)
                                    hz[j3] = pack_h2(__uint_as_float(r[j3 >> 1][j3 & 1][2 * jj]),
                                                     __uint_as_float(r[j3 >> 1][j3 & 1][2 * jj + 1]));
                                const int64_t t0 = 256 * (jb + jj) + 8 * lane;
                                const uint64_t pol = l2_evict_last();     // read back by the odd tile
                                stg_hint(slot + (t0 >> 2), make_uint4(hz[0], hz[1], hz[2], hz[3]), pol);
                                stg_hint(slot + (t0 >> 2) + 1, make_uint4(hz[4], hz[5], hz[6], hz[7]), pol);
                            }
                        }
                        if (MODE == kModeRows && emit) {
                            // z back into the workspace row as fp16, unscaled
                            // (the inverse column pass applies the row's filter
                            // scale and undoes the unitary pair's 1/8192)
#pragma unroll
                            for (int jj = 0; jj < 2; ++jj) {
                                uint32_t hz[8];
#pragma unroll
                                for (int j3 = 0; j3 < 8; ++j3)
                                    hz[j3] = pack_h2(__uint_as_float(r[j3 >> 1][j3 & 1][2 * jj]),
                                                     __uint_as_float(r[j3 >> 1][j3 & 1][2 * jj + 1]));
                                uint4* dst = a.work + (P.o0 + 256 * (jb + jj) + 8 * lane) / 4;
                                dst[0] = make_uint4(hz[0], hz[1], hz[2], hz[3]);
                                dst[1] = make_uint4(hz[4], hz[5], hz[6], hz[7]);
                            }
                        }
                        if (MODE != kModeRows && emit) {
#pragma unroll
                            for (int jj = 0; jj < 2; ++jj) {
                                const int64_t t0 = 256 * (jb + jj) + 8 * lane;
                                const uint32_t vaw[4] = {va[jj].x, va[jj].y, va[jj].z, va[jj].w};
                                const uint32_t vbw[4] = {vb[jj].x, vb[jj].y, vb[jj].z, vb[jj].w};
                                float2 w0 = make_float2(1.f, 0.f);
                                [[maybe_unused]] const uint4* zslot = nullptr;   // z_even of these t (split, odd tile)
                                if constexpr (LY::kSplit) {
                                    zslot = a.scratch + ((int64_t)blockIdx.x * 4 + q) * (kM / 4) + (t0 >> 2);
                                    w0 = __ldg(&a.tw16k[t0]);
                                }
                                uint32_t oa[4], ob[4];
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    // j3 = 2e (chunk c0 + e, jl 0) and 2e + 1 (jl 1)
                                    float a0 = __uint_as_float(r[e][0][2 * jj]), a1 = __uint_as_float(r[e][1][2 * jj]);
                                    float b0 = __uint_as_float(r[e][0][2 * jj + 1]), b1 = __uint_as_float(r[e][1][2 * jj + 1]);
                                    float sc = kscale;
                                    if constexpr (LY::kSplit) {
                                        // (z_even + conj(w16384^t) z_odd) / 2, t = t0 + 2e (+1)
                                        const float2 w_0 = cmul(w0, a.w16k_j3[2 * e]), w_1 = cmul(w0, a.w16k_j3[2 * e + 1]);
                                        const float2 zo0 = cmulc(make_float2(a0, b0), w_0), zo1 = cmulc(make_float2(a1, b1), w_1);
                                        // z_even of t0 + 2e (+1), loaded where used
                                        const uint2 zp = ldg2_hint(reinterpret_cast<const uint2*>(zslot) + e,
                                                                   l2_evict_first());
                                        const float2 ze0 = __half22float2(u2h(zp.x)), ze1 = __half22float2(u2h(zp.y));
                                        a0 = ze0.x + zo0.x; b0 = ze0.y + zo0.y;
                                        a1 = ze1.x + zo1.x; b1 = ze1.y + zo1.y;
                                        sc *= 0.5f;
                                    }
                                    a0 *= sc; a1 *= sc; b0 *= sc; b1 *= sc;
                                    nonfinite_fold(nf, a0); nonfinite_fold(nf, a1);
                                    nonfinite_fold(nf, b0); nonfinite_fold(nf, b1);
                                    if (a.v) {
                                        const float2 g0 = IO<T>::unpack2(vaw[e]), g1 = IO<T>::unpack2(vbw[e]);
                                        a0 *= g0.x; a1 *= g0.y; b0 *= g1.x; b1 *= g1.y;
                                    }
                                    oa[e] = IO<T>::pack2(a0, a1);
                                    ob[e] = IO<T>::pack2(b0, b1);
                                }
                                if constexpr (LY::kSplit) {
                                    const uint64_t pol = l2_evict_first();
                                    stg_hint((T*)a.y + P.o0 + t0, make_uint4(oa[0], oa[1], oa[2], oa[3]), pol);
                                    if (has1) stg_hint((T*)a.y + P.o1 + t0, make_uint4(ob[0], ob[1], ob[2], ob[3]), pol);
                                } else {
                                    *(uint4*)((T*)a.y + P.o0 + t0) = make_uint4(oa[0], oa[1], oa[2], oa[3]);
                                    if (has1) *(uint4*)((T*)a.y + P.o1 + t0) = make_uint4(ob[0], ob[1], ob[2], ob[3]);
                                }
                            }
                        }
                    }
                }
            };
            if constexpr (LY::kSplit) {
                if (odd) output_pass(std::false_type{});
                else output_pass(std::true_type{});
            } else {
                output_pass(std::false_type{});
            }
        }
        if constexpr (MODE != kModeRows) nonfinite_report(nf, a.status);
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

struct TcResources {
    int mode = kModePlain;
    uint8_t* bimg = nullptr;
    float2* tw1024 = nullptr;
    Tw16* twM16 = nullptr;
    float2* tw16k = nullptr;      // split mode
    uint4* scratch = nullptr;     // split mode: num_sms x 4 x 8192 half2
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

template <int MODE>
std::vector<uint8_t> build_bimage() {
    using LY = Lay<MODE>;
    constexpr int J = LY::kJ1;
    std::vector<uint8_t> img(LY::BImageBytes, 0);
    const double r32 = 1.0 / std::sqrt(32.0), r8 = 1.0 / std::sqrt(8.0);
    auto off = [](int o) { return (size_t)(o - LY::OffBS1); };
    std::vector<std::complex<double>> F;
    // S1: c1 <- j1 (j1 < J: the nonzero inputs)
    F.assign(32 * J, 0);
    for (int c = 0; c < 32; ++c) for (int j = 0; j < J; ++j) F[c * J + j] = wpow((long long)c * j, 32, -1) * r32;
    put_complex_matrix(img, off(LY::OffBS1), 32, J, F);
    // S2: c2 <- l
    F.assign(32 * 32, 0);
    for (int c = 0; c < 32; ++c) for (int j = 0; j < 32; ++j) F[c * 32 + j] = wpow((long long)c * j, 32, -1) * r32;
    put_complex_matrix(img, off(LY::OffBS2), 32, 32, F);
    // S3 (per c2): c3 <- j3 with w8^(c3 j3) w256^(c2 j3);  S3': j3 <- c3, conjugate
    for (int c2 = 0; c2 < 32; ++c2) {
        std::vector<std::complex<double>> G(64), Gi(64);
        for (int c3 = 0; c3 < 8; ++c3)
            for (int j3 = 0; j3 < 8; ++j3) {
                const std::complex<double> gv = wpow((long long)c3 * j3, 8, -1) * wpow((long long)c2 * j3, 256, -1) * r8;
                G[c3 * 8 + j3] = gv;
                Gi[j3 * 8 + c3] = std::conj(gv);
            }
        put_complex_matrix(img, off(LY::OffBS3) + c2 * 512, 8, 8, G);
        put_complex_matrix(img, off(LY::OffBS3i) + c2 * 512, 8, 8, Gi);
    }
    // S2': l <- c2
    F.assign(32 * 32, 0);
    for (int l = 0; l < 32; ++l) for (int c = 0; c < 32; ++c) F[l * 32 + c] = wpow((long long)c * l, 32, +1) * r32;
    put_complex_matrix(img, off(LY::OffBS2i), 32, 32, F);
    // S1': j1 <- c1 (j1 < J: the kept outputs)
    F.assign(J * 32, 0);
    for (int j = 0; j < J; ++j) for (int c = 0; c < 32; ++c) F[j * 32 + c] = wpow((long long)c * j, 32, +1) * r32;
    put_complex_matrix(img, off(LY::OffBS1i), J, 32, F);
    return img;
}

uint16_t half_bits(float x) {
    const __half h = __float2half_rn(x);
    uint16_t b;
    std::memcpy(&b, &h, 2);
    return b;
}
// exp(-2 pi i e / 8192), e < 256, as the packed-half pair (tr, ti), (-ti, tr)
std::vector<Tw16> twiddle_table16() {
    std::vector<Tw16> t(256);
    for (int e = 0; e < 256; ++e) {
        const std::complex<double> z = wpow(e, kM, -1);
        const float tr = (float)z.real(), ti = (float)z.imag();
        t[e].p = (uint32_t)half_bits(tr) | ((uint32_t)half_bits(ti) << 16);
        t[e].q = (uint32_t)half_bits(-ti) | ((uint32_t)half_bits(tr) << 16);
    }
    return t;
}

std::vector<float2> twiddle_table(int n, int count) {
    std::vector<float2> t(count);
    for (int e = 0; e < count; ++e) {
        const std::complex<double> z = wpow(e, n, -1);
        t[e] = make_float2((float)z.real(), (float)z.imag());
    }
    return t;
}

// K_f -> rfft bins [0, N] of each channel.  split = 0: one row of the
// 8192-point spectrum per channel; split = 1: the 16384-point spectrum as
// two rows per channel (even bins, odd bins).
__global__ void tc_export_kernel(const __half2* __restrict__ Kh, const float* __restrict__ scale,
                                 float* __restrict__ out, int64_t H, int split) {
    const int64_t nb = split ? 2 * kN + 1 : kN + 1;
    const int64_t total = H * nb;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t h = i / nb, f = i % nb;
        const int64_t row = split ? 2 * h + (f & 1) : h;
        const int64_t f8 = split ? f >> 1 : f;
        const int c1 = (int)(f8 & 31), c2 = (int)((f8 >> 5) & 31), c3 = (int)(f8 >> 10);
        const float2 z = __half22float2(Kh[row * kM + k16_index(c1, c2, c3)]);
        out[2 * i] = z.x * scale[h];
        out[2 * i + 1] = z.y * scale[h];
    }
}

// Kernel mode of a plan: sequences of 4096 run plain; sequences of 8192 carry
// both the parity split's filter rows (calls with a frequency mask: the mask
// acts on the 16384-point spectrum) and the two-block rows of the planar
// kernel (every other call); longer sequences need windows (filters of at
// most 2049 taps).
int tc_mode(int64_t N, int64_t L) {
    (void)L;
    if (N <= kN) return kModePlain;      // N < 4096: several sequences per transform (tc_planar.cu)
    if (N == 2 * kN) return kModeSplit;
    if (N == 4 * kN) return kModeBlocks4;
    return kModeWindows;
}

}  // namespace

bool tc_supported(int64_t N, int64_t L, int dtype) {
    if (dtype != kF16 && dtype != kBF16) return false;
    if (N <= kN || N == 2 * kN || N == 4 * kN) return true;
    return N > kN && L <= kHop + 1;      // overlap-save windows (N a power of two)
}

int64_t tc_windows(int64_t N) { return N <= kN ? 1 : N / kHop - 1; }
bool tc_overlap_save(int64_t N, int64_t L) { return tc_mode(N, L) == kModeWindows; }
bool tc_full_spectrum(int64_t N, int64_t L) {
    const int m = tc_mode(N, L);
    return m != kModeWindows && m != kModeBlocks4;
}
int64_t tc_tiles_per_pair_group(int64_t N, int64_t L) {
    const int m = tc_mode(N, L);
    return m == kModeWindows ? tc_windows(N) : (m == kModeSplit ? 2 : (m == kModeBlocks4 ? 4 : 1));
}

namespace {

template <int MODE>
cudaError_t set_smem_attributes() {
    cudaError_t e = cudaFuncSetAttribute(tc_fftconv_n4096_kernel<__nv_bfloat16, MODE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Lay<MODE>::SmemBytes);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(tc_fftconv_n4096_kernel<__half, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Lay<MODE>::SmemBytes);
    return e;
}

template <typename V>
cudaError_t upload_vec(V** dst, const std::vector<V>& v) {
    cudaError_t e = cudaMalloc((void**)dst, v.size() * sizeof(V));
    if (e == cudaSuccess) e = cudaMemcpy(*dst, v.data(), v.size() * sizeof(V), cudaMemcpyHostToDevice);
    return e;
}

template <int MODE>
void launch_mode(const Plan& p, const TcArgs& a, int64_t grid, cudaStream_t s) {
    if (p.dtype == kBF16)
        tc_fftconv_n4096_kernel<__nv_bfloat16, MODE><<<(unsigned)grid, kThreads, Lay<MODE>::SmemBytes, s>>>(a);
    else
        tc_fftconv_n4096_kernel<__half, MODE><<<(unsigned)grid, kThreads, Lay<MODE>::SmemBytes, s>>>(a);
}

}  // namespace

cudaError_t tc_plan_init(Plan& p) {
    TcResources* r = new TcResources();
    p.tc = r;
    r->mode = tc_mode(p.N, p.L);
    if (r->mode != kModeSplit) {
        // sequences of 4096 and overlap-save windows run the planar kernel
        // (tc_planar.cu); the SIMT engine computes their 8192-point filter
        // spectrum, so the plan also carries that twiddle table
        p.logTab = 13;
        cudaError_t e = upload_vec(&p.tw, twiddle_table(kM, kM));
        if (e == cudaSuccess) e = tc_planar_init(p);
        return e;
    }
    const std::vector<uint8_t> img = build_bimage<kModeSplit>();
    cudaError_t e = cudaMalloc((void**)&r->bimg, img.size());
    if (e == cudaSuccess) e = cudaMemcpy(r->bimg, img.data(), img.size(), cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = upload_vec(&r->tw1024, twiddle_table(1024, 1024));
    if (e == cudaSuccess) e = upload_vec(&r->twM16, twiddle_table16());
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&r->num_sms, cudaDevAttrMultiProcessorCount, p.device);
    if (e == cudaSuccess && r->mode == kModeSplit) {
        e = upload_vec(&r->tw16k, twiddle_table(2 * kM, kM));
        if (e == cudaSuccess) e = cudaMalloc((void**)&r->scratch, (size_t)r->num_sms * 4 * kM * sizeof(uint32_t));
    }
    // the SIMT engine computes the filter spectrum (8192 points, or 16384 in
    // the split mode), so the plan also carries that twiddle table
    const int64_t mf = r->mode == kModeSplit ? 2 * kM : kM;
    p.logTab = r->mode == kModeSplit ? 14 : 13;
    if (e == cudaSuccess) e = upload_vec(&p.tw, twiddle_table((int)mf, (int)mf));
    if (e == cudaSuccess) e = set_smem_attributes<kModePlain>();
    if (e == cudaSuccess) e = set_smem_attributes<kModeWindows>();
    if (e == cudaSuccess) e = set_smem_attributes<kModeSplit>();
    // unmasked calls run the planar kernel's two-block mode
    if (e == cudaSuccess) e = tc_planar_init(p);
    return e;
}

void tc_plan_free(Plan& p) {
    tc_planar_free(p);
    TcResources* r = (TcResources*)p.tc;
    if (!r) return;
    cudaFree(r->bimg);
    cudaFree(r->tw1024);
    cudaFree(r->twM16);
    cudaFree(r->tw16k);
    cudaFree(r->scratch);
    delete r;
    p.tc = nullptr;
}

static int64_t tc_filter_rows(const Plan& p) { return tc_mode(p.N, p.L) == kModeSplit ? 2 * p.H : p.H; }

// K_f: rows of 8192 complex fp16 (scaled so each channel's largest component
// is 1; the split mode has two rows per channel, even and odd bins), then [H]
// fp32 scales; sequences of 8192 then append the two-block rows
// (tc_planar_two_block_bytes).
static size_t tc_split_bytes(const Plan& p) {
    return (size_t)tc_filter_rows(p) * kKBytes + (((size_t)p.H * 4 + 15) & ~size_t(15));
}
size_t tc_filter_bytes(const Plan& p) {
    if (tc_mode(p.N, p.L) == kModeBlocks4) return tc_planar_two_block_bytes(p);
    return tc_split_bytes(p) + (tc_mode(p.N, p.L) == kModeSplit ? tc_planar_two_block_bytes(p) : 0);
}

cudaError_t tc_precompute(const Plan& p, const void* k, void* Kf, cudaStream_t s) {
    if (tc_mode(p.N, p.L) == kModeBlocks4) return tc_planar_precompute_two_block(p, k, Kf, s);
    if (tc_mode(p.N, p.L) != kModeSplit) return tc_planar_precompute(p, k, Kf, s);
    cudaError_t e = simt_precompute_to_tc_split(p, k, Kf, s);
    if (e == cudaSuccess) e = tc_planar_precompute_two_block(p, k, (uint8_t*)Kf + tc_split_bytes(p), s);
    return e;
}

cudaError_t tc_forward(const Plan& p, const ForwardArgs& fa, cudaStream_t s) {
    const TcResources* r = (const TcResources*)p.tc;
    if (r->mode == kModeBlocks4) return tc_planar_forward(p, fa, kPlanarTwoBlock, s);
    if (r->mode != kModeSplit)
        return tc_planar_forward(p, fa, r->mode == kModeWindows ? kPlanarWindows : kPlanarPlain, s);
    if (!fa.mask) {
        ForwardArgs two = fa;
        two.Kf = (const uint8_t*)fa.Kf + tc_split_bytes(p);
        return tc_planar_forward(p, two, kPlanarTwoBlock, s);
    }
    TcArgs a{};
    a.u = fa.u; a.w = fa.w; a.v = fa.v; a.y = fa.y;
    a.Kh16 = (const __half2*)fa.Kf;
    a.Kscale = (const float*)((const uint8_t*)fa.Kf + (size_t)tc_filter_rows(p) * kKBytes);
    a.mask = fa.mask; a.mask_h = fa.mask_h;
    a.B = fa.B; a.H = p.H;
    a.N = p.N;
    a.nwin = r->mode == kModeWindows ? tc_windows(p.N) : 1;
    a.pb = (fa.B + 1) / 2;
    a.tpc = (a.pb + 3) / 4;
    const int64_t groups = p.H * a.nwin * a.tpc;       // CTA-sized work items
    a.nunits = r->mode == kModeSplit ? 2 * groups : groups;
    a.bimg = (const uint4*)r->bimg;
    a.tw1024 = r->tw1024;
    a.twM16 = r->twM16;
    a.tw16k = r->tw16k;
    a.scratch = r->scratch;
    for (int j = 0; j < 8; ++j) {
        const std::complex<double> z = wpow(j, 2 * kM, -1);
        a.w16k_j3[j] = make_float2((float)z.real(), (float)z.imag());
    }
    a.status = p.status;
    const int64_t grid = groups < r->num_sms ? groups : r->num_sms;
    if (r->mode == kModeSplit) launch_mode<kModeSplit>(p, a, grid, s);
    else if (r->mode == kModeWindows) launch_mode<kModeWindows>(p, a, grid, s);
    else launch_mode<kModePlain>(p, a, grid, s);
    return cudaGetLastError();
}

// Self-test of the bounded-wait path: one warp initialises an mbarrier that
// expects one arrival and waits for its first phase with the same bounded
// wait the convolution kernels use (at most `polls` blocking polls).  With
// `arrive` set, lane 0 arrives first and the wait succeeds; otherwise nothing
// arrives, the wait gives up and the kernel records FFTCONV_ERR_TIMEOUT in the
// status word, exactly as a convolution kernel would.  Nothing is faulted and
// the context stays usable.
__global__ void bounded_wait_selftest_kernel(int* status, uint32_t polls, int arrive) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncwarp();
    if (arrive && threadIdx.x == 0) mbar_arrive(&bar);
    __syncwarp();
    const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bar, 0, &abort_flag, polls));
    if (!ok && threadIdx.x == 0) atomicExch(status, kStatusTimeout);
}

cudaError_t selftest_bounded_wait(const Plan& p, uint32_t polls, int arrive, cudaStream_t s) {
    bounded_wait_selftest_kernel<<<1, 32, 0, s>>>(p.status, polls, arrive);
    return cudaGetLastError();
}

// ------------------------------------------------ staged row engine ---

namespace {

// workspace row (h0 + ch, c) of the staged forward transform of k (permuted
// positions, rfft(k)/M) -> K_f row h * R + c in the tensor-core layout with
// its own scale (one CTA per row)
__global__ void tc_rows_convert_kernel(const float2* __restrict__ work, __half2* __restrict__ Kh,
                                       float* __restrict__ scales, int64_t h0, int64_t R) {
    constexpr int NT = 256;
    __shared__ float red[NT / 32];
    const int64_t row = blockIdx.x;                    // (ch, c) within the chunk
    const int64_t ch = row / R, c = row - ch * R;
    const float2* src = work + row * (int64_t)kM;
    float m = 0.f;
    for (int p = threadIdx.x; p < kM; p += NT) {
        const float2 z = src[p];
        m = fmaxf(m, fmaxf(fabsf(z.x), fabsf(z.y)));
    }
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    m = 0.f;
    for (int i = 0; i < NT / 32; ++i) m = fmaxf(m, red[i]);
    const float sc = m > 0.f ? m : 1.f, inv = 1.f / sc;
    const int64_t krow = (h0 + ch) * R + c;
    for (int p = threadIdx.x; p < kM; p += NT) {
        const int k = (int)perm_to_freq(p, 13);       // the row transform's output order
        const float2 z = src[p];
        Kh[krow * kM + k16_index(k & 31, (k >> 5) & 31, k >> 10)] = __floats2half2_rn(z.x * inv, z.y * inv);
    }
    if (threadIdx.x == 0) scales[krow] = sc;
}

// K_f of a staged tensor-core plan -> rfft bins [0, N]: bin f is row c = f % R,
// position k = f / R; the 1/M is undone
__global__ void tc_rows_export_kernel(const __half2* __restrict__ Kh, const float* __restrict__ scales,
                                      float* __restrict__ out, int64_t H, int64_t N, int64_t R) {
    const int64_t nb = N + 1, total = H * nb;
    const float m = (float)(2 * N);
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t h = i / nb, f = i - h * nb;
        const int64_t c = f % R, k = f / R, krow = h * R + c;
        const float2 z = __half22float2(Kh[krow * kM + k16_index((int)(k & 31), (int)((k >> 5) & 31), (int)(k >> 10))]);
        out[2 * i] = z.x * scales[krow] * m;
        out[2 * i + 1] = z.y * scales[krow] * m;
    }
}

}  // namespace

bool tc_staged_supported(int64_t N, int64_t L, int dtype) {
    return (dtype == kF16 || dtype == kBF16) && N >= 4 * kN && N <= (int64_t(1) << 22) && L > kHop + 1;
}

size_t tc_staged_spectrum_bytes(const Plan& p) { return (size_t)(p.H * (p.M / kM)) * kKBytes; }

size_t tc_staged_filter_bytes(const Plan& p) {
    const int64_t rows = p.H * (p.M / kM);
    return (size_t)rows * kKBytes + (((size_t)rows * 4 + 15) & ~size_t(15));
}

cudaError_t tc_rows_init(Plan& p) {
    TcResources* r = new TcResources();
    p.tc = r;
    r->mode = kModeRows;
    const std::vector<uint8_t> img = build_bimage<kModeRows>();
    cudaError_t e = cudaMalloc((void**)&r->bimg, img.size());
    if (e == cudaSuccess) e = cudaMemcpy(r->bimg, img.data(), img.size(), cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = upload_vec(&r->tw1024, twiddle_table(1024, 1024));
    if (e == cudaSuccess) e = upload_vec(&r->twM16, twiddle_table16());
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&r->num_sms, cudaDevAttrMultiProcessorCount, p.device);
    if (e == cudaSuccess) e = set_smem_attributes<kModeRows>();
    return e;
}

cudaError_t tc_rows_forward(const Plan& p, const ForwardArgs& fa, int64_t pair0, int64_t npairs, cudaStream_t s) {
    const TcResources* r = (const TcResources*)p.tc;
    const int64_t R = p.M / kM;
    TcArgs a{};
    a.Kh16 = (const __half2*)fa.Kf;
    a.Kscale = (const float*)((const uint8_t*)fa.Kf + (size_t)(p.H * R) * kKBytes);
    a.mask = fa.mask; a.mask_h = fa.mask_h;
    a.B = fa.B; a.H = p.H; a.N = p.N;
    a.nwin = 1;
    // workspace units per channel (rows mode divides by it for the channel):
    // the pairs, times the overlap-save windows of each
    a.pb = (fa.B + 1) / 2 * p.nwin;
    a.tpc = 1;
    a.work = (uint4*)p.work; a.R = R; a.pair0 = pair0;
    a.nunits = npairs * (R / 4);
    a.bimg = (const uint4*)r->bimg;
    a.tw1024 = r->tw1024;
    a.twM16 = r->twM16;
    a.status = p.status;
    const int64_t grid = a.nunits < r->num_sms ? a.nunits : r->num_sms;
    launch_mode<kModeRows>(p, a, grid, s);
    return cudaGetLastError();
}

cudaError_t tc_rows_convert(const Plan& p, int64_t h0, int64_t nch, void* Kf, cudaStream_t s) {
    const int64_t R = p.M / kM;
    tc_rows_convert_kernel<<<(unsigned)(nch * R), 256, 0, s>>>(
        p.work, (__half2*)Kf, (float*)((uint8_t*)Kf + (size_t)(p.H * R) * kKBytes), h0, R);
    return cudaGetLastError();
}

cudaError_t tc_rows_export(const Plan& p, const void* Kf, float* out, cudaStream_t s) {
    const int64_t R = p.M / kM, total = p.H * (p.N + 1);
    int blocks = (int)((total + 255) / 256);
    if (blocks > 65535) blocks = 65535;
    tc_rows_export_kernel<<<blocks, 256, 0, s>>>((const __half2*)Kf,
                                                 (const float*)((const uint8_t*)Kf + (size_t)(p.H * R) * kKBytes), out,
                                                 p.H, p.N, R);
    return cudaGetLastError();
}

cudaError_t tc_export_rfft(const Plan& p, const void* Kf, float* out, cudaStream_t s) {
    const int split = tc_mode(p.N, p.L) == kModeSplit ? 1 : 0;
    if (!split) return tc_planar_export(p, Kf, out, s);
    const int64_t total = p.H * (p.N + 1);
    int blocks = (int)((total + 255) / 256);
    if (blocks > 65535) blocks = 65535;
    tc_export_kernel<<<blocks, 256, 0, s>>>((const __half2*)Kf,
                                            (const float*)((const uint8_t*)Kf + (size_t)tc_filter_rows(p) * kKBytes),
                                            out, p.H, split);
    return cudaGetLastError();
}

}  // namespace fftconv
