// internal.h -- plan structure and kernel launchers shared by the C ABI
// implementation (api.cu) and the kernel translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace fftconv {

enum Path : int { kPathSimtFused = 1, kPathSimtStaged = 2, kPathTcFused = 3, kPathTcStaged = 4 };
enum DType : int { kF32 = 0, kF16 = 1, kBF16 = 2 };

// Staged path factorization M = R * C (log2 of C for log2(M) = logM): rows
// of C = 1024 points, or longer where that keeps R <= 256, and C <= 2^14
// (the row kernel's limit).  Measured on B200 this balances the column and
// row passes far better than the longest rows: N = 32768 runs 1.8x faster as
// 64 x 1024 than as 4 x 16384, N = 2^20 5% faster as 256 x 8192 than as
// 128 x 16384.  Every staged plan and the static-scratch entry point use it,
// so they share the K_f layout [H][R][C].
inline int staged_log_cols(int logM) {
    int lc = logM - 8 > 10 ? logM - 8 : 10;
    if (lc > logM - 1) lc = logM - 1;
    if (lc > 14) lc = 14;
    return lc;
}

struct Plan {
    int64_t N = 0, H = 0, L = 0, M = 0;
    int logM = 0;
    int dtype = 0;
    int order = 0;
    int path = 0;
    int device = 0;
    size_t filter_bytes = 0;

    // fp32 twiddle table exp(-2 pi i e / Ltab), e < Ltab (fused: Ltab = M;
    // staged: Ltab = C).
    float2* tw = nullptr;
    int logTab = 0;
    // exp(-2 pi i e / 2N), e < 2N: the transform table of the backward pass's
    // filter gradient (tensor-core plans with N <= 4096)
    float2* twgrad = nullptr;

    // staged path: M = R * C, two-level table for exp(-2 pi i e / M)
    int logR = 0, logC = 0;
    int twSplit = 0;            // bits of the low table
    float2* twLo = nullptr;     // exp(-2 pi i e / M), e < 2^twSplit
    float2* twHi = nullptr;     // exp(-2 pi i (e << twSplit) / M)
    float2* work = nullptr;     // [chunkPairs][R][C] complex fp32 (fp16 on the tensor-core staged path)
    // tensor-core staged path, overlap-save windows (nwin > 1): transforms of
    // M = 2 winHop points, window w of a sequence reads inputs
    // [(w-1) winHop, (w+1) winHop) (zero before 0) and writes outputs
    // [w winHop, (w+1) winHop); the workspace units are (pair, window)
    int64_t winHop = 0, nwin = 1;
    int64_t chunkPairs = 0;
    size_t workBytes = 0;

    // tensor-core path resources (owned by the tc translation units:
    // tc_kernels.cu for the parity split and the staged row pass,
    // tc_planar.cu for sequences of 4096 and overlap-save windows)
    void* tc = nullptr;
    void* tcp = nullptr;

    int* status = nullptr;      // device status word (timeouts)

    // host-buffer entry point: copy streams and chunk events, created on
    // first use (fftconv_forward_host)
    static constexpr int kHostChunks = 8;
    cudaStream_t copy_in = nullptr, copy_out = nullptr;
    cudaEvent_t ev_start = nullptr, ev_out = nullptr;
    cudaEvent_t ev_in[kHostChunks] = {}, ev_comp[kHostChunks] = {};
};

struct ForwardArgs {
    const void* u;
    const void* w;
    const void* v;
    void* y;
    const void* Kf;
    const uint8_t* mask;
    int64_t mask_h;
    int64_t B;
};

// Thread-local detail string returned by fftconv_last_error (api.cu).
void set_last_error(const char* msg);

// SIMT fp32 path (simt_kernels.cu)
cudaError_t simt_fused_forward(const Plan& p, const ForwardArgs& a, cudaStream_t s);
cudaError_t simt_fused_precompute(const Plan& p, const void* k, void* Kf, cudaStream_t s);
cudaError_t simt_staged_forward(const Plan& p, const ForwardArgs& a, cudaStream_t s);
cudaError_t simt_staged_precompute(const Plan& p, const void* k, void* Kf, cudaStream_t s);
cudaError_t simt_export_rfft(const Plan& p, const void* Kf, float* out, cudaStream_t s);
bool simt_fused_supported(int logM);

// tensor-core path (tc_kernels.cu)
bool tc_supported(int64_t N, int64_t L, int dtype);
int64_t tc_windows(int64_t N);   // overlap-save windows per sequence (1: one transform)
bool tc_overlap_save(int64_t N, int64_t L);   // the plan runs overlap-save windows
bool tc_full_spectrum(int64_t N, int64_t L);  // the plan stores the 2N-point filter spectrum
int64_t tc_tiles_per_pair_group(int64_t N, int64_t L);   // tiles per (channel, 4 pairs)
cudaError_t tc_plan_init(Plan& p);
void tc_plan_free(Plan& p);
size_t tc_filter_bytes(const Plan& p);
cudaError_t tc_precompute(const Plan& p, const void* k, void* Kf, cudaStream_t s);
cudaError_t tc_forward(const Plan& p, const ForwardArgs& a, cudaStream_t s);
cudaError_t tc_export_rfft(const Plan& p, const void* Kf, float* out, cudaStream_t s);
cudaError_t selftest_bounded_wait(const Plan& p, uint32_t polls, int arrive, cudaStream_t s);

// tensor-core fused kernel with planar complex data (tc_planar.cu):
// sequences of at most 4096 (plain), of 8192 and 16384 as two and four blocks
// of 4096 (kPlanarTwoBlock: the filter rows G_0 .. G_{P-1} of
// tc_planar_precompute_two_block), and overlap-save windows
enum { kPlanarPlain = 0, kPlanarWindows = 1, kPlanarTwoBlock = 2, kPlanarMonarch = 3 };
cudaError_t tc_planar_init(Plan& p);
void tc_planar_free(Plan& p);
cudaError_t tc_planar_precompute(const Plan& p, const void* k, void* Kf, cudaStream_t s);
size_t tc_planar_two_block_bytes(const Plan& p);
cudaError_t tc_planar_precompute_two_block(const Plan& p, const void* k, void* Kf, cudaStream_t s);
cudaError_t tc_planar_forward(const Plan& p, const ForwardArgs& a, int mode, cudaStream_t s);
// N = 4096 with a Monarch-aligned frequency mask: bit c2 of keep_c2 keeps the
// spectrum bins f with (f >> 5) & 31 == c2 (f = c1 + 32 c2 + 1024 c3); the
// stages of masked c2 are skipped
cudaError_t tc_planar_forward_monarch(const Plan& p, const ForwardArgs& a, uint32_t keep_c2, cudaStream_t s);
cudaError_t tc_planar_export(const Plan& p, const void* Kf, float* out, cudaStream_t s);
// backward pass (N <= 4096): the correlation launch of the planar kernel and
// the filter gradient on fp32 lanes (simt_kernels.cu)
cudaError_t tc_planar_correlate(const Plan& p, const ForwardArgs& a, void* y2, const void* v2, cudaStream_t s);
cudaError_t simt_filter_grad(const Plan& p, const void* u, const void* w, const void* v, const void* dy, int64_t B,
                             float* dk, cudaStream_t s);

// staged path with the tensor-core row pass (rows of C = 8192): the column
// passes are the SIMT ones (simt_kernels.cu), the row pass and the filter
// layout are the tensor-core kernel's (tc_kernels.cu)
constexpr int kTcRowLogC = 13;
bool tc_staged_supported(int64_t N, int64_t L, int dtype);
size_t tc_staged_filter_bytes(const Plan& p);
size_t tc_staged_spectrum_bytes(const Plan& p);   // the fp16 rows; the [H * R] fp32 scales follow
cudaError_t tc_rows_init(Plan& p);
cudaError_t tc_rows_forward(const Plan& p, const ForwardArgs& fa, int64_t pair0, int64_t npairs, cudaStream_t s);
cudaError_t tc_rows_convert(const Plan& p, int64_t h0, int64_t nch, void* Kf, cudaStream_t s);
cudaError_t tc_rows_export(const Plan& p, const void* Kf, float* out, cudaStream_t s);
cudaError_t tc_staged_forward(const Plan& p, const ForwardArgs& a, cudaStream_t s);
cudaError_t tc_staged_precompute(const Plan& p, const void* k, void* Kf, cudaStream_t s);

}  // namespace fftconv
