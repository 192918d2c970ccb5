// api.cu -- the C ABI (include/fftconv.h): plan creation, argument
// validation, host-side fp64 twiddle tables and dispatch to the kernels.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "../../include/fftconv.h"
#include "internal.h"

using namespace fftconv;

namespace {

thread_local std::string g_last_error;

int fail(int status, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return status;
}

int cuda_fail(cudaError_t e, const char* what) {
    return fail(FFTCONV_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int ilog2(int64_t v) {
    int l = 0;
    while ((int64_t(1) << l) < v) ++l;
    return l;
}

size_t dtype_size(int dt) { return dt == kF32 ? 4 : 2; }

// exp(-2 pi i e / L) for e < count (scaled by `mult`: exp(-2 pi i e*mult / L)),
// evaluated in double with the angle reduced exactly, then rounded to fp32.
std::vector<float2> host_twiddles(int64_t L, int64_t count, int64_t mult) {
    std::vector<float2> t((size_t)count);
    const double two_pi = 6.283185307179586476925286766559;
    for (int64_t e = 0; e < count; ++e) {
        const int64_t r = (e * mult) % L;
        const double a = two_pi * (double)r / (double)L;
        t[(size_t)e] = make_float2((float)std::cos(a), (float)-std::sin(a));
    }
    return t;
}

cudaError_t upload(float2** dst, const std::vector<float2>& v) {
    cudaError_t e = cudaMalloc((void**)dst, v.size() * sizeof(float2));
    if (e != cudaSuccess) return e;
    return cudaMemcpy(*dst, v.data(), v.size() * sizeof(float2), cudaMemcpyHostToDevice);
}

void free_plan(Plan* p) {
    if (!p) return;
    int cur = 0;
    cudaGetDevice(&cur);
    cudaSetDevice(p->device);
    if (p->tc) tc_plan_free(*p);
    cudaFree(p->tw);
    cudaFree(p->twgrad);
    cudaFree(p->twLo);
    cudaFree(p->twHi);
    cudaFree(p->work);
    cudaFree(p->status);
    if (p->copy_in) cudaStreamDestroy(p->copy_in);
    if (p->copy_out) cudaStreamDestroy(p->copy_out);
    if (p->ev_start) cudaEventDestroy(p->ev_start);
    if (p->ev_out) cudaEventDestroy(p->ev_out);
    for (int i = 0; i < Plan::kHostChunks; ++i) {
        if (p->ev_in[i]) cudaEventDestroy(p->ev_in[i]);
        if (p->ev_comp[i]) cudaEventDestroy(p->ev_comp[i]);
    }
    cudaSetDevice(cur);
    delete p;
}

bool ranges_overlap(const void* a, size_t na, const void* b, size_t nb) {
    if (!a || !b || !na || !nb) return false;
    const uintptr_t a0 = (uintptr_t)a, b0 = (uintptr_t)b;
    return a0 < b0 + nb && b0 < a0 + na;
}

}  // namespace

namespace fftconv {
void set_last_error(const char* msg) { g_last_error = msg; }
}  // namespace fftconv

struct fftconv_plan_s {
    Plan p;
};

extern "C" {

const char* fftconv_version(void) { return "fftconv-b200 0.1"; }

const char* fftconv_status_string(int status) {
    switch (status) {
        case FFTCONV_OK: return "ok";
        case FFTCONV_ERR_INVALID_ARG: return "invalid argument";
        case FFTCONV_ERR_UNSUPPORTED: return "unsupported configuration";
        case FFTCONV_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
        case FFTCONV_ERR_CUDA: return "CUDA error";
        case FFTCONV_ERR_OOM: return "out of device memory";
        case FFTCONV_ERR_TIMEOUT: return "device wait timed out";
        case FFTCONV_ERR_RANGE: return "non-finite result (fp16 intermediate out of range)";
        default: return "unknown status";
    }
}

const char* fftconv_last_error(void) { return g_last_error.c_str(); }

int fftconv_plan_create_ex(fftconv_plan_t* out, int64_t N, int64_t H, fftconv_dtype_t dtype,
                           int order, int64_t L) {
    g_last_error.clear();
    if (!out) return fail(FFTCONV_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (N <= 0 || H <= 0) return fail(FFTCONV_ERR_INVALID_ARG, "N=%lld and H=%lld must be positive",
                                      (long long)N, (long long)H);
    if (dtype != FFTCONV_F32 && dtype != FFTCONV_F16 && dtype != FFTCONV_BF16)
        return fail(FFTCONV_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (L <= 0 || L > N) return fail(FFTCONV_ERR_INVALID_ARG, "filter length L=%lld not in [1, N]", (long long)L);
    if ((N & (N - 1)) != 0) return fail(FFTCONV_ERR_UNSUPPORTED, "N=%lld is not a power of two", (long long)N);
    if (N < 256 || N > (int64_t(1) << 22))
        return fail(FFTCONV_ERR_UNSUPPORTED, "N=%lld outside [256, 2^22]", (long long)N);
    if (order < 0 || order > 5) return fail(FFTCONV_ERR_UNSUPPORTED, "order %d not in {0,1,2,3,4,5}", order);
    if (H > (int64_t(1) << 24)) return fail(FFTCONV_ERR_UNSUPPORTED, "H=%lld too large", (long long)H);

    Plan* p = new (std::nothrow) Plan();
    if (!p) return fail(FFTCONV_ERR_OOM, "host allocation failed");
    p->N = N; p->H = H; p->L = L; p->M = 2 * N; p->logM = ilog2(2 * N);
    p->dtype = (int)dtype; p->order = order;
    cudaGetDevice(&p->device);

    const bool tc_ok = tc_supported(N, L, (int)dtype);
    const bool tc_staged_ok = tc_staged_supported(N, L, (int)dtype);
    if (order == 5) {
        if (!tc_staged_ok) {
            delete p;
            return fail(FFTCONV_ERR_UNSUPPORTED,
                        "order 5 needs fp16/bf16, 16384 <= N <= 2^22 and L > 2049 (N=%lld, L=%lld)",
                        (long long)N, (long long)L);
        }
        p->path = kPathTcStaged;
    } else if (order == 0 && !tc_ok && tc_staged_ok) {
        p->path = kPathTcStaged;
    } else if (order == 4 || (order == 0 && !tc_ok && !simt_fused_supported(p->logM))) {
        p->path = kPathSimtStaged;
    } else if (order == 1) {
        if (!simt_fused_supported(p->logM)) { delete p; return fail(FFTCONV_ERR_UNSUPPORTED, "order 1 needs N <= 8192"); }
        p->path = kPathSimtFused;
    } else if (tc_ok) {
        p->path = kPathTcFused;
    } else if (simt_fused_supported(p->logM)) {
        p->path = kPathSimtFused;
    } else {
        delete p;
        return fail(FFTCONV_ERR_UNSUPPORTED,
                    "order %d asks for a fused on-chip transform; none holds N=%lld with L=%lld "
                    "(fused kernels: N <= 16384 with 16-bit data, N <= 8192 in fp32, or L <= 2049 with 16-bit "
                    "data); use order 0, 4 or 5",
                    order, (long long)N, (long long)L);
    }

    cudaError_t e = cudaMalloc((void**)&p->status, sizeof(int));
    if (e == cudaSuccess) e = cudaMemset(p->status, 0, sizeof(int));
    if (e != cudaSuccess) { free_plan(p); return e == cudaErrorMemoryAllocation ? fail(FFTCONV_ERR_OOM, "status word") : cuda_fail(e, "plan status"); }

    if (p->path == kPathSimtFused) {
        p->logTab = p->logM;
        e = upload(&p->tw, host_twiddles(p->M, p->M, 1));
        p->filter_bytes = (size_t)H * (size_t)p->M * sizeof(float2);
    } else if (p->path == kPathSimtStaged || p->path == kPathTcStaged) {
        // Automatic tensor-core staged plans with a filter much shorter than
        // the sequence run overlap-save windows: hop Lw = the smallest power
        // of two >= max(L, 16384), one 2 Lw-point transform per window,
        // N / Lw windows per sequence (the same number of transform points as
        // one 2N-point transform, in shorter columns).  The filter spectrum
        // then has 2 Lw points, so such plans take no block mask and export
        // no 2N-point spectrum; order 5 keeps the full transform.
        if (p->path == kPathTcStaged && order == 0) {
            int64_t lw = 16384;
            while (lw < L) lw *= 2;
            if (2 * lw <= N) {
                p->winHop = lw;
                p->nwin = N / lw;
                p->M = 2 * lw;
                p->logM = ilog2(p->M);
            }
        }
        // (the tensor-core row pass takes rows of 8192)
        p->logC = p->path == kPathTcStaged ? kTcRowLogC : staged_log_cols(p->logM);
        p->logR = p->logM - p->logC;
        p->logTab = p->logC;
        const int64_t C = int64_t(1) << p->logC;
        e = upload(&p->tw, host_twiddles(C, C, 1));
        p->twSplit = (p->logM + 1) / 2;
        if (e == cudaSuccess) e = upload(&p->twLo, host_twiddles(p->M, int64_t(1) << p->twSplit, 1));
        if (e == cudaSuccess)
            e = upload(&p->twHi, host_twiddles(p->M, p->M >> p->twSplit, int64_t(1) << p->twSplit));
        // workspace: the SIMT passes take a chunk of pairs of about 64 MB
        // (L2-sized), at least one.  The tensor-core row pass keeps the
        // workspace in fp16 and takes chunks of 512 MB (at least two pairs, so
        // that the fp32 filter precompute fits one channel): its launches then
        // run many tiles per SM, which measured faster on B200 than L2-sized
        // chunks (N = 32768: 0.84 against 0.99 ms per call in fp32).
        const bool ws16 = p->path == kPathTcStaged;
        const size_t per_pair = (size_t)p->M * (ws16 ? 2 * sizeof(uint16_t) : sizeof(float2));
        p->chunkPairs = (int64_t)((size_t(ws16 ? 512 : 64) << 20) / per_pair);
        if (p->chunkPairs < (ws16 ? 2 : 1)) p->chunkPairs = ws16 ? 2 : 1;
        p->workBytes = per_pair * (size_t)p->chunkPairs;
        if (e == cudaSuccess) e = cudaMalloc((void**)&p->work, p->workBytes);
        p->filter_bytes = (size_t)H * (size_t)p->M * sizeof(float2);
        if (p->path == kPathTcStaged) {
            if (e == cudaSuccess) e = tc_rows_init(*p);
            p->filter_bytes = tc_staged_filter_bytes(*p);
        }
    } else {
        e = tc_plan_init(*p);
        p->filter_bytes = tc_filter_bytes(*p);
        // the backward pass's filter gradient transforms length 2N on fp32 lanes
        if (e == cudaSuccess && N <= 8192) e = upload(&p->twgrad, host_twiddles(p->M, p->M, 1));
    }
    if (e != cudaSuccess) {
        free_plan(p);
        if (e == cudaErrorMemoryAllocation) return fail(FFTCONV_ERR_OOM, "plan tables/workspace");
        return cuda_fail(e, "plan tables");
    }
    fftconv_plan_s* h = new (std::nothrow) fftconv_plan_s();
    if (!h) { free_plan(p); return fail(FFTCONV_ERR_OOM, "host allocation failed"); }
    h->p = *p;
    delete p;   // shallow copy moved into the handle (device pointers now owned by h)
    *out = h;
    return FFTCONV_OK;
}

int fftconv_plan_create(fftconv_plan_t* out, int64_t N, int64_t H, fftconv_dtype_t dtype, int order) {
    return fftconv_plan_create_ex(out, N, H, dtype, order, N);
}

int fftconv_plan_destroy(fftconv_plan_t plan) {
    g_last_error.clear();
    if (!plan) return FFTCONV_OK;
    cudaDeviceSynchronize();
    Plan* p = new (std::nothrow) Plan(plan->p);
    if (p) free_plan(p);
    delete plan;
    return FFTCONV_OK;
}

size_t fftconv_filter_bytes(fftconv_plan_t plan) { return plan ? plan->p.filter_bytes : 0; }

size_t fftconv_workspace_bytes(fftconv_plan_t plan) { return plan ? plan->p.workBytes : 0; }

int fftconv_plan_path(fftconv_plan_t plan) {
    if (!plan) return fail(FFTCONV_ERR_INVALID_ARG, "plan is NULL");
    return plan->p.path;
}

int fftconv_filter_precompute(fftconv_plan_t plan, const void* k, void* K_f, fftconv_stream_t stream) {
    g_last_error.clear();
    if (!plan || !k || !K_f) return fail(FFTCONV_ERR_INVALID_ARG, "plan, k and K_f must be non-NULL");
    if (!aligned16(k) || !aligned16(K_f)) return fail(FFTCONV_ERR_ALIGNMENT, "k or K_f not 16-byte aligned");
    const Plan& p = plan->p;
    if (ranges_overlap(k, (size_t)(p.H * p.L) * dtype_size(p.dtype), K_f, p.filter_bytes))
        return fail(FFTCONV_ERR_INVALID_ARG, "k and K_f overlap");
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    switch (p.path) {
        case kPathSimtFused: e = simt_fused_precompute(p, k, K_f, s); break;
        case kPathSimtStaged: e = simt_staged_precompute(p, k, K_f, s); break;
        case kPathTcStaged: e = tc_staged_precompute(p, k, K_f, s); break;
        default: e = tc_precompute(p, k, K_f, s); break;
    }
    if (e != cudaSuccess) return cuda_fail(e, "filter precompute launch");
    return FFTCONV_OK;
}

static int validate_forward(const Plan& p, const void* u, const void* K_f, void* y, int64_t B,
                            int64_t H, int64_t N, const void* w, const void* v, const uint8_t* mask,
                            int64_t mask_h) {
    if (B < 0) return fail(FFTCONV_ERR_INVALID_ARG, "B=%lld is negative", (long long)B);
    if (H != p.H || N != p.N)
        return fail(FFTCONV_ERR_INVALID_ARG, "H=%lld N=%lld do not match the plan (H=%lld N=%lld)",
                    (long long)H, (long long)N, (long long)p.H, (long long)p.N);
    if (B == 0) return FFTCONV_OK;
    if (!u || !K_f || !y) return fail(FFTCONV_ERR_INVALID_ARG, "u, K_f and y must be non-NULL");
    if (!aligned16(u) || !aligned16(K_f) || !aligned16(y) || !aligned16(w) || !aligned16(v))
        return fail(FFTCONV_ERR_ALIGNMENT, "u, K_f, y, w and v must be 16-byte aligned");
    if (mask && mask_h != 1 && mask_h != H)
        return fail(FFTCONV_ERR_INVALID_ARG, "mask_h=%lld must be 1 or H=%lld", (long long)mask_h, (long long)H);
    if (mask && N < 32) return fail(FFTCONV_ERR_UNSUPPORTED, "block mask needs N >= 32");
    if (p.path == kPathTcFused &&
        (double)H * (double)tc_tiles_per_pair_group(p.N, p.L) * (double)(((B + 1) / 2 + 3) / 4) >= 2147483648.0)
        return fail(FFTCONV_ERR_UNSUPPORTED, "too many tiles for one launch");
    if (mask && p.path == kPathTcFused && p.N < 4096)
        return fail(FFTCONV_ERR_UNSUPPORTED,
                    "block masks act on the 2N-point spectrum; this tensor-core plan (N=%lld) packs %lld "
                    "sequences into one 8192-point transform: create the plan with order 1 or 4 for masks",
                    (long long)p.N, (long long)(4096 / p.N));
    if (mask && ((p.path == kPathTcFused && !tc_full_spectrum(p.N, p.L)) || p.nwin > 1))
        return fail(FFTCONV_ERR_UNSUPPORTED,
                    "block masks act on the 2N-point spectrum; this plan (N=%lld, L=%lld: overlap-save "
                    "windows or blocks of 4096) has none: create the plan with order 1 or 4 (or 5 for "
                    "N >= 16384, L > 2049)",
                    (long long)p.N, (long long)p.L);
    if (B > (int64_t(1) << 30) / 1) {
        if ((double)B * (double)H > 4.0e9) return fail(FFTCONV_ERR_UNSUPPORTED, "B*H too large");
    }
    const size_t bytes = (size_t)B * (size_t)H * (size_t)N * dtype_size(p.dtype);
    if (ranges_overlap(y, bytes, u, bytes) || ranges_overlap(y, bytes, w, bytes) ||
        ranges_overlap(y, bytes, v, bytes) || ranges_overlap(y, bytes, K_f, p.filter_bytes))
        return fail(FFTCONV_ERR_INVALID_ARG, "y overlaps an input");
    if ((double)H * (double)((B + 1) / 2) > 2147483647.0)
        return fail(FFTCONV_ERR_UNSUPPORTED, "too many sequence pairs for one launch");
    return FFTCONV_OK;
}

static int run_forward(const Plan& p, const ForwardArgs& a, cudaStream_t s) {
    cudaError_t e;
    switch (p.path) {
        case kPathSimtFused: e = simt_fused_forward(p, a, s); break;
        case kPathSimtStaged: e = simt_staged_forward(p, a, s); break;
        case kPathTcStaged: e = tc_staged_forward(p, a, s); break;
        default: e = tc_forward(p, a, s); break;
    }
    if (e != cudaSuccess) return cuda_fail(e, "forward launch");
    return FFTCONV_OK;
}

int fftconv_forward(fftconv_plan_t plan, const void* u, const void* K_f, void* y, int64_t B, int64_t H,
                    int64_t N, const void* w, const void* v, const uint8_t* block_mask, int64_t mask_h,
                    fftconv_stream_t stream) {
    g_last_error.clear();
    if (!plan) return fail(FFTCONV_ERR_INVALID_ARG, "plan is NULL");
    const Plan& p = plan->p;
    int rc = validate_forward(p, u, K_f, y, B, H, N, w, v, block_mask, mask_h);
    if (rc != FFTCONV_OK || B == 0) return rc;
    ForwardArgs a{u, w, v, y, K_f, block_mask, block_mask ? mask_h : 0, B};
    return run_forward(p, a, (cudaStream_t)stream);
}

int fftconv_forward_monarch(fftconv_plan_t plan, const void* u, const void* K_f, void* y, int64_t B, int64_t H,
                            int64_t N, const void* w, const void* v, uint32_t keep_c2, fftconv_stream_t stream) {
    g_last_error.clear();
    if (!plan) return fail(FFTCONV_ERR_INVALID_ARG, "plan is NULL");
    const Plan& p = plan->p;
    if (p.path != kPathTcFused || p.N != 4096)
        return fail(FFTCONV_ERR_UNSUPPORTED,
                    "Monarch-aligned masks act on the 8192-point spectrum of a tensor-core plan with N = 4096 "
                    "(this plan: N=%lld, path %d)", (long long)p.N, (int)p.path);
    int rc = validate_forward(p, u, K_f, y, B, H, N, w, v, nullptr, 0);
    if (rc != FFTCONV_OK || B == 0) return rc;
    cudaError_t e;
    if (keep_c2 == 0) {
        e = cudaMemsetAsync(y, 0, (size_t)B * (size_t)H * (size_t)N * dtype_size(p.dtype), (cudaStream_t)stream);
    } else {
        ForwardArgs a{u, w, v, y, K_f, nullptr, 0, B};
        e = tc_planar_forward_monarch(p, a, keep_c2, (cudaStream_t)stream);
    }
    if (e != cudaSuccess) return cuda_fail(e, "forward launch");
    return FFTCONV_OK;
}

static size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

}  // extern "C"

// Copy streams and events of the host-buffer entry point, created once per
// plan on the plan's device (non-blocking streams, events without timing).
static int host_resources(Plan& p) {
    if (p.copy_in) return FFTCONV_OK;
    int cur = 0;
    cudaGetDevice(&cur);
    cudaSetDevice(p.device);
    cudaError_t e = cudaStreamCreateWithFlags(&p.copy_in, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&p.copy_out, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p.ev_start, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p.ev_out, cudaEventDisableTiming);
    for (int i = 0; i < Plan::kHostChunks && e == cudaSuccess; ++i) {
        e = cudaEventCreateWithFlags(&p.ev_in[i], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p.ev_comp[i], cudaEventDisableTiming);
    }
    cudaSetDevice(cur);
    if (e != cudaSuccess) return cuda_fail(e, "host-buffer streams");
    return FFTCONV_OK;
}

extern "C" {

size_t fftconv_forward_host_staging_bytes(fftconv_plan_t plan, int64_t B, int has_w, int has_v, int has_mask,
                                          int64_t mask_h) {
    if (!plan || B < 0) return 0;
    const Plan& p = plan->p;
    const size_t t = round256((size_t)B * (size_t)p.H * (size_t)p.N * dtype_size(p.dtype));
    size_t total = 2 * t;                          // u, y
    if (has_w) total += t;
    if (has_v) total += t;
    if (has_mask) total += round256((size_t)(mask_h > 0 ? mask_h : 1) * (size_t)(p.N / 32));
    return total;
}

int fftconv_forward_host(fftconv_plan_t plan, const void* u_host, const void* K_f, void* y_host, int64_t B,
                         int64_t H, int64_t N, const void* w_host, const void* v_host, const uint8_t* mask_host,
                         int64_t mask_h, void* staging, size_t staging_bytes, fftconv_stream_t stream) {
    g_last_error.clear();
    if (!plan) return fail(FFTCONV_ERR_INVALID_ARG, "plan is NULL");
    const Plan& p = plan->p;
    if (B < 0 || H != p.H || N != p.N) return validate_forward(p, u_host, K_f, y_host, B, H, N, nullptr, nullptr,
                                                               nullptr, 1);
    if (B == 0) return FFTCONV_OK;
    if (!u_host || !y_host || !K_f || !staging)
        return fail(FFTCONV_ERR_INVALID_ARG, "u_host, y_host, K_f and staging must be non-NULL");
    if ((reinterpret_cast<uintptr_t>(staging) & 255u) != 0)
        return fail(FFTCONV_ERR_ALIGNMENT, "staging must be 256-byte aligned");
    const size_t need = fftconv_forward_host_staging_bytes(plan, B, w_host != nullptr, v_host != nullptr,
                                                           mask_host != nullptr, mask_h);
    if (staging_bytes < need)
        return fail(FFTCONV_ERR_INVALID_ARG, "staging has %zu bytes, %zu needed", staging_bytes, need);
    const size_t bytes = (size_t)B * (size_t)p.H * (size_t)p.N * dtype_size(p.dtype);
    const size_t t = round256(bytes);
    char* base = (char*)staging;
    void* du = base; base += t;
    void* dy = base; base += t;
    void* dw = nullptr; void* dv = nullptr; uint8_t* dm = nullptr;
    if (w_host) { dw = base; base += t; }
    if (v_host) { dv = base; base += t; }
    const size_t mbytes = mask_host ? (size_t)mask_h * (size_t)(p.N / 32) : 0;
    if (mask_host) { dm = (uint8_t*)base; }
    cudaStream_t s = (cudaStream_t)stream;
    int rc = validate_forward(p, du, K_f, dy, B, H, N, dw, dv, dm, mask_h);
    if (rc != FFTCONV_OK) return rc;
    rc = host_resources(plan->p);
    if (rc != FFTCONV_OK) return rc;

    // Pipelined over chunks of batch rows: chunk i's uploads run on the copy-in
    // stream, its forward pass on `stream`, its download on the copy-out
    // stream, so uploads, compute and downloads of different chunks overlap
    // (the two copy directions use separate engines).  `stream` orders the
    // whole call: the copies start after its earlier work, and its later work
    // waits for the last download.
    const size_t row = (size_t)p.H * (size_t)p.N * dtype_size(p.dtype);
    int64_t rows = (B + Plan::kHostChunks - 1) / Plan::kHostChunks;
    rows += rows & 1;                                // whole pairs of rows
    const int nchunks = (int)((B + rows - 1) / rows);
    Plan& q = plan->p;
    cudaError_t e = cudaEventRecord(q.ev_start, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(q.copy_in, q.ev_start, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(q.copy_out, q.ev_start, 0);
    if (e == cudaSuccess && mask_host) e = cudaMemcpyAsync(dm, mask_host, mbytes, cudaMemcpyHostToDevice, q.copy_in);
    for (int i = 0; i < nchunks && e == cudaSuccess; ++i) {
        const int64_t r0 = i * rows, nr = (B - r0 < rows) ? B - r0 : rows;
        const size_t off = (size_t)r0 * row, nb = (size_t)nr * row;
        e = cudaMemcpyAsync((char*)du + off, (const char*)u_host + off, nb, cudaMemcpyHostToDevice, q.copy_in);
        if (e == cudaSuccess && w_host)
            e = cudaMemcpyAsync((char*)dw + off, (const char*)w_host + off, nb, cudaMemcpyHostToDevice, q.copy_in);
        if (e == cudaSuccess && v_host)
            e = cudaMemcpyAsync((char*)dv + off, (const char*)v_host + off, nb, cudaMemcpyHostToDevice, q.copy_in);
        if (e == cudaSuccess) e = cudaEventRecord(q.ev_in[i], q.copy_in);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(s, q.ev_in[i], 0);
        if (e != cudaSuccess) break;
        ForwardArgs a{(const char*)du + off, dw ? (const char*)dw + off : nullptr,
                      dv ? (const char*)dv + off : nullptr, (char*)dy + off, K_f, dm, mask_host ? mask_h : 0, nr};
        rc = run_forward(p, a, s);
        if (rc != FFTCONV_OK) return rc;
        e = cudaEventRecord(q.ev_comp[i], s);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(q.copy_out, q.ev_comp[i], 0);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync((char*)y_host + off, (const char*)dy + off, nb, cudaMemcpyDeviceToHost, q.copy_out);
    }
    if (e == cudaSuccess) e = cudaEventRecord(q.ev_out, q.copy_out);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, q.ev_out, 0);
    if (e != cudaSuccess) return cuda_fail(e, "host-buffer pipeline");
    return FFTCONV_OK;
}

int fftconv_backward(fftconv_plan_t plan, const void* u, const void* K_f, const void* dy, int64_t B, int64_t H,
                     int64_t N, const void* w, const void* v, void* du, void* dw, void* dv, float* dk,
                     fftconv_stream_t stream) {
    g_last_error.clear();
    if (!plan) return fail(FFTCONV_ERR_INVALID_ARG, "plan is NULL");
    const Plan& p = plan->p;
    if (p.path != kPathTcFused || p.N > 8192)
        return fail(FFTCONV_ERR_UNSUPPORTED,
                    "the backward pass runs on fp16/bf16 tensor-core plans with N <= 8192 (this plan: %s, N=%lld)",
                    p.path == kPathTcFused ? "tensor-core" : "not tensor-core", (long long)p.N);
    int rc = validate_forward(p, u, K_f, du, B, H, N, w, v, nullptr, 0);
    if (rc != FFTCONV_OK) return rc;
    if (B == 0) {
        if (dk) {
            cudaError_t e = cudaMemsetAsync(dk, 0, sizeof(float) * (size_t)(p.H * p.L), (cudaStream_t)stream);
            if (e != cudaSuccess) return cuda_fail(e, "dk clear");
        }
        return FFTCONV_OK;
    }
    if (!dy || !du) return fail(FFTCONV_ERR_INVALID_ARG, "dy and du must be non-NULL");
    if (dw && !w) return fail(FFTCONV_ERR_INVALID_ARG, "dw needs the gate w");
    if (dv && !v) return fail(FFTCONV_ERR_INVALID_ARG, "dv needs the gate v");
    if (!aligned16(dy) || !aligned16(du) || !aligned16(dw) || !aligned16(dv) || !aligned16(dk))
        return fail(FFTCONV_ERR_ALIGNMENT, "dy, du, dw, dv and dk must be 16-byte aligned");
    const size_t bytes = (size_t)B * (size_t)H * (size_t)N * dtype_size(p.dtype);
    const void* ins[5] = {u, w, v, dy, K_f};
    const size_t in_bytes[5] = {bytes, bytes, bytes, bytes, p.filter_bytes};
    void* outs[4] = {du, dw, dv, dk};
    const size_t out_bytes[4] = {bytes, bytes, bytes, sizeof(float) * (size_t)(p.H * p.L)};
    for (int i = 0; i < 4; ++i) {
        for (int j = 0; j < 5; ++j)
            if (ranges_overlap(outs[i], out_bytes[i], ins[j], in_bytes[j]))
                return fail(FFTCONV_ERR_INVALID_ARG, "an output of the backward pass overlaps an input");
        for (int j = i + 1; j < 4; ++j)
            if (ranges_overlap(outs[i], out_bytes[i], outs[j], out_bytes[j]))
                return fail(FFTCONV_ERR_INVALID_ARG, "two outputs of the backward pass overlap");
    }
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaSuccess;
    // dv = dy * conv(u * w, k): the forward pass with dy as the output gate
    if (dv) {
        ForwardArgs a{u, w, dy, dv, K_f, nullptr, 0, B};
        e = tc_forward(p, a, s);
    }
    // du = w * corr(dy * v, k), dw = u * corr(dy * v, k) (N = 8192: on the
    // two-block filter rows, the last part of K_f)
    if (e == cudaSuccess) {
        const void* Kc = p.N == 8192 ? (const void*)((const uint8_t*)K_f + p.filter_bytes - tc_planar_two_block_bytes(p))
                                     : K_f;
        ForwardArgs a{dy, v, w, du, Kc, nullptr, 0, B};
        e = tc_planar_correlate(p, a, dw, u, s);
    }
    // dk = sum_b corr(dy * v, u * w)[:L]
    if (e == cudaSuccess && dk) e = simt_filter_grad(p, u, w, v, dy, B, dk, s);
    if (e != cudaSuccess) return cuda_fail(e, "backward launch");
    return FFTCONV_OK;
}

int fftconv_filter_to_rfft(fftconv_plan_t plan, const void* K_f, float* out, fftconv_stream_t stream) {
    g_last_error.clear();
    if (!plan || !K_f || !out) return fail(FFTCONV_ERR_INVALID_ARG, "plan, K_f and out must be non-NULL");
    if (!aligned16(K_f) || ((uintptr_t)out & 7u)) return fail(FFTCONV_ERR_ALIGNMENT, "K_f/out misaligned");
    const Plan& p = plan->p;
    if (p.path == kPathTcFused && !tc_full_spectrum(p.N, p.L))
        return fail(FFTCONV_ERR_UNSUPPORTED,
                    "this plan (overlap-save windows or blocks of 4096) stores 8192-point spectra of k, "
                    "not the 2N-point one");
    if (p.nwin > 1)
        return fail(FFTCONV_ERR_UNSUPPORTED,
                    "this overlap-save plan stores the %lld-point spectrum of k, not the 2N-point one",
                    (long long)p.M);
    cudaError_t e = p.path == kPathTcFused    ? tc_export_rfft(p, K_f, out, (cudaStream_t)stream)
                    : p.path == kPathTcStaged ? tc_rows_export(p, K_f, out, (cudaStream_t)stream)
                                              : simt_export_rfft(p, K_f, out, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "export launch");
    return FFTCONV_OK;
}

int fftconv_selftest_bounded_wait(fftconv_plan_t plan, int64_t polls, int arrive, fftconv_stream_t stream) {
    g_last_error.clear();
    if (!plan) return fail(FFTCONV_ERR_INVALID_ARG, "plan is NULL");
    if (polls < 1 || polls > (int64_t(1) << 20))
        return fail(FFTCONV_ERR_INVALID_ARG, "polls=%lld outside [1, 2^20]", (long long)polls);
    cudaError_t e = selftest_bounded_wait(plan->p, (uint32_t)polls, arrive ? 1 : 0, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
    return FFTCONV_OK;
}

int fftconv_device_status(fftconv_plan_t plan, fftconv_stream_t stream) {
    g_last_error.clear();
    if (!plan) return fail(FFTCONV_ERR_INVALID_ARG, "plan is NULL");
    cudaStream_t s = (cudaStream_t)stream;
    int host = 0;
    cudaError_t e = cudaMemcpyAsync(&host, plan->p.status, sizeof(int), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "status read");
    if (host != 0) {
        int zero = 0;
        cudaMemcpy(plan->p.status, &zero, sizeof(int), cudaMemcpyHostToDevice);
        return fail(host, host == FFTCONV_ERR_RANGE
                              ? "a forward call produced non-finite values: an fp16 intermediate overflowed "
                                "(or an input held inf/NaN)"
                              : "a bounded device wait timed out");
    }
    return FFTCONV_OK;
}

}  // extern "C"
