// noalloc.cu -- fftconv_forward_noalloc: the staged convolution with its
// scratch memory in a fixed, statically allocated device array instead of a
// plan workspace, for callers that may not allocate device memory at all.
//
// Who needs this: code embedded in a host framework that owns every byte of
// device memory through its own pool and forbids direct cudaMalloc, and
// latency-critical paths that cannot pay for cudaMalloc's implicit device
// synchronisation.  Such callers cannot create a plan (plans allocate their
// tables and workspace), so this entry point needs none: the staged passes
// read their twiddle tables and write their intermediate spectra into
// file-scope __device__ arrays that exist for as long as the library is
// loaded, on every GPU that loads it.
//
// Limits and sharing: the scratch array holds kScratchElems complex fp32
// values (16 MiB), enough for one sequence pair of transform length
// M = 2N <= 2^21, i.e. N <= 2^20; larger N is rejected.  Every call uses the
// same arrays, and each call overwrites what the previous one left there (no
// value needs to start at zero: every pass writes before it reads), so calls
// whose execution overlaps on the GPU -- on different streams or from
// different host threads -- race and must be serialised by the caller.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <mutex>

#include "../../include/fftconv.h"
#include "internal.h"

namespace fftconv {
namespace {

constexpr int kMaxLogM = 21;                                  // M <= 2^21
constexpr int64_t kScratchElems = int64_t(1) << kMaxLogM;     // 16 MiB of float2
constexpr int kMaxLogC = 14;
constexpr int kMaxDevices = 64;

// The scratch workspace and the twiddle tables of the staged passes.
static __device__ __align__(256) float2 g_scratch[kScratchElems];
static __device__ __align__(256) float2 g_twC[int64_t(1) << kMaxLogC];
static __device__ __align__(256) float2 g_twLo[int64_t(1) << ((kMaxLogM + 1) / 2)];
static __device__ __align__(256) float2 g_twHi[int64_t(1) << ((kMaxLogM + 1) / 2)];

// Device addresses of the static arrays in the calling thread's current
// context.  They are looked up on every call (a host-side query that
// allocates nothing once the module is loaded): a cached address would go
// stale after cudaDeviceReset or under a context other than the one it was
// taken in, and the passes would then write through it.
struct DeviceSymbols {
    float2* scratch = nullptr;
    float2* twC = nullptr;
    float2* twLo = nullptr;
    float2* twHi = nullptr;
};

// Which twiddle tables the static arrays hold, per device: the transform
// length they were filled for and the context that filled them (a context id
// from the driver is unique for the life of the process).  A call refills
// them only when either differs.
struct ResidentTables {
    unsigned long long ctx_id = 0;
    int logM = 0;
    float2* twC = nullptr;
};
ResidentTables g_resident[kMaxDevices];
std::mutex g_resident_mutex;

int noalloc_fail(int status, const char* fmt, ...) {
    char buf[400];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    set_last_error(buf);
    return status;
}

// exp(-2 pi i e / L) evaluated in double precision on the device.
__global__ void fill_twiddles(float2* twC, int64_t C, float2* lo, int64_t nlo, float2* hi, int64_t nhi, int64_t M,
                              int split) {
    const int64_t total = C + nlo + nhi;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        double sn, cs;
        if (i < C) {
            sincospi(2.0 * (double)i / (double)C, &sn, &cs);
            twC[i] = make_float2((float)cs, (float)-sn);
        } else if (i < C + nlo) {
            const int64_t e = i - C;
            sincospi(2.0 * (double)e / (double)M, &sn, &cs);
            lo[e] = make_float2((float)cs, (float)-sn);
        } else {
            const int64_t e = i - C - nlo;
            sincospi(2.0 * (double)((e << split) % M) / (double)M, &sn, &cs);
            hi[e] = make_float2((float)cs, (float)-sn);
        }
    }
}

// Resolve the device addresses of the static arrays for the current context
// (host code cannot use the array names as device pointers).
int device_symbols(DeviceSymbols* s, int* dev) {
    cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess) return noalloc_fail(FFTCONV_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (*dev < 0 || *dev >= kMaxDevices) return noalloc_fail(FFTCONV_ERR_UNSUPPORTED, "device index %d", *dev);
    e = cudaGetSymbolAddress((void**)&s->scratch, g_scratch);
    if (e == cudaSuccess) e = cudaGetSymbolAddress((void**)&s->twC, g_twC);
    if (e == cudaSuccess) e = cudaGetSymbolAddress((void**)&s->twLo, g_twLo);
    if (e == cudaSuccess) e = cudaGetSymbolAddress((void**)&s->twHi, g_twHi);
    if (e != cudaSuccess) return noalloc_fail(FFTCONV_ERR_CUDA, "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    return FFTCONV_OK;
}

// Unique id of the calling thread's current context, through the driver
// entry points the runtime exposes (no link-time dependency on the driver
// library).  Returns false if the driver cannot say: the tables are then
// refilled on every call.
bool current_context_id(unsigned long long* id) {
    using GetCurrent = int (*)(void**);
    using GetId = int (*)(void*, unsigned long long*);
    static GetCurrent get_current = nullptr;
    static GetId get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q1 = cudaDriverEntryPointSymbolNotFound, q2 = q1;
        void* f1 = nullptr;
        void* f2 = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f1, 12000, cudaEnableDefault, &q1) == cudaSuccess &&
            cudaGetDriverEntryPointByVersion("cuCtxGetId", &f2, 12000, cudaEnableDefault, &q2) == cudaSuccess &&
            q1 == cudaDriverEntryPointSuccess && q2 == cudaDriverEntryPointSuccess) {
            get_current = (GetCurrent)f1;
            get_id = (GetId)f2;
        }
    });
    if (!get_current || !get_id) return false;
    void* ctx = nullptr;
    if (get_current(&ctx) != 0 || !ctx) return false;
    return get_id(ctx, id) == 0 && *id != 0;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
    if (!a || !b) return false;
    const uintptr_t a0 = (uintptr_t)a, b0 = (uintptr_t)b;
    return a0 < b0 + nb && b0 < a0 + na;
}

}  // namespace
}  // namespace fftconv

using namespace fftconv;

extern "C" int fftconv_forward_noalloc(const void* u, const void* K_f, void* y, int64_t B, int64_t H, int64_t N,
                                       fftconv_dtype_t dtype, const void* w, const void* v,
                                       const uint8_t* block_mask, int64_t mask_h, fftconv_stream_t stream) {
    set_last_error("");
    if (dtype != FFTCONV_F32 && dtype != FFTCONV_F16 && dtype != FFTCONV_BF16)
        return noalloc_fail(FFTCONV_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (B < 0 || H <= 0 || N <= 0) return noalloc_fail(FFTCONV_ERR_INVALID_ARG, "B, H, N out of range");
    if ((N & (N - 1)) != 0 || N < 256)
        return noalloc_fail(FFTCONV_ERR_UNSUPPORTED, "N=%lld must be a power of two >= 256", (long long)N);
    if (2 * N > kScratchElems)
        return noalloc_fail(FFTCONV_ERR_UNSUPPORTED,
                            "N=%lld exceeds the static scratch: at most N=%lld (2N complex fp32 values in %lld bytes)",
                            (long long)N, (long long)(kScratchElems / 2), (long long)(kScratchElems * 8));
    if (B == 0) return FFTCONV_OK;
    if (!u || !K_f || !y) return noalloc_fail(FFTCONV_ERR_INVALID_ARG, "u, K_f and y must be non-NULL");
    if (!aligned16(u) || !aligned16(K_f) || !aligned16(y) || !aligned16(w) || !aligned16(v))
        return noalloc_fail(FFTCONV_ERR_ALIGNMENT, "u, K_f, y, w, v must be 16-byte aligned");
    if (block_mask && mask_h != 1 && mask_h != H)
        return noalloc_fail(FFTCONV_ERR_INVALID_ARG, "mask_h must be 1 or H");
    const size_t bytes = (size_t)B * (size_t)H * (size_t)N * (dtype == FFTCONV_F32 ? 4 : 2);
    // K_f is the order-4 layout: H rows of 2N complex fp32 values
    const size_t kf_bytes = (size_t)H * (size_t)(2 * N) * sizeof(float2);
    if (overlap(y, bytes, u, bytes) || overlap(y, bytes, w, bytes) || overlap(y, bytes, v, bytes) ||
        overlap(y, bytes, K_f, kf_bytes))
        return noalloc_fail(FFTCONV_ERR_INVALID_ARG, "y overlaps an input");

    DeviceSymbols sym;
    int dev = 0;
    int rc = device_symbols(&sym, &dev);
    if (rc != FFTCONV_OK) return rc;

    // A plan-shaped description on the stack pointing at the static arrays;
    // the staged passes themselves are the ones every staged plan runs.
    Plan p;
    p.N = N; p.H = H; p.L = N; p.M = 2 * N;
    int logM = 0;
    while ((int64_t(1) << logM) < p.M) ++logM;
    p.logM = logM;
    p.dtype = (int)dtype;
    p.path = kPathSimtStaged;
    p.logC = staged_log_cols(logM);     // the K_f layout of every staged plan
    p.logR = logM - p.logC;
    p.logTab = p.logC;
    p.twSplit = (logM + 1) / 2;
    p.tw = sym.twC;
    p.twLo = sym.twLo;
    p.twHi = sym.twHi;
    p.work = sym.scratch;
    p.chunkPairs = kScratchElems / p.M;
    p.workBytes = (size_t)kScratchElems * sizeof(float2);

    cudaStream_t s = (cudaStream_t)stream;
    const int64_t C = int64_t(1) << p.logC;
    const int64_t nlo = int64_t(1) << p.twSplit, nhi = p.M >> p.twSplit;
    {
        // refill the twiddle tables only when N or the context changed since
        // the last fill on this device (the fill is ordered on `s` before the
        // passes; earlier calls' passes read tables of the same N)
        unsigned long long ctx = 0;
        const bool known = current_context_id(&ctx);
        std::lock_guard<std::mutex> lock(g_resident_mutex);
        ResidentTables& r = g_resident[dev];
        if (!known || r.ctx_id != ctx || r.logM != logM || r.twC != p.tw) {
            fill_twiddles<<<64, 256, 0, s>>>(p.tw, C, p.twLo, nlo, p.twHi, nhi, p.M, p.twSplit);
            cudaError_t e = cudaGetLastError();
            if (e != cudaSuccess) {
                r = ResidentTables{};
                return noalloc_fail(FFTCONV_ERR_CUDA, "twiddle fill: %s", cudaGetErrorString(e));
            }
            r.ctx_id = known ? ctx : 0;
            r.logM = known ? logM : 0;
            r.twC = p.tw;
        }
    }
    cudaError_t e;
    ForwardArgs a{u, w, v, y, K_f, block_mask, block_mask ? mask_h : 0, B};
    e = simt_staged_forward(p, a, s);
    if (e != cudaSuccess) return noalloc_fail(FFTCONV_ERR_CUDA, "staged passes: %s", cudaGetErrorString(e));
    return FFTCONV_OK;
}
