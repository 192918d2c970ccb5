/*
 * fftconv.h -- C ABI of the B200 (sm_100a) exact causal long-convolution
 * library.
 *
 * Operation (page "FlashFFTConv: Efficient Convolutions for Long Sequences
 * with Tensor Cores", summary paragraph, "Approach" and "Key results"): for
 * every batch row b and channel h,
 *
 *     y[b,h,t] = v[b,h,t] * sum_{s=0}^{min(t, L-1)} k[h,s] * u[b,h,t-s] * w[b,h,t-s]
 *
 * for 0 <= t < N, computed as irfft(rfft(u*w, 2N) * K_f, 2N)[:N] with
 * K_f = rfft(k zero-padded to 2N).  The gates w and v are optional ("gated
 * convolution", Key results); a filter shorter than the sequence (L < N) is
 * the "partial convolution" and a block mask on K_f the "frequency-sparse
 * convolution" (Approach; measured-effects table, 75% / 79% sparsity rows).
 * The length-2N transform is evaluated as a product of small DFT factors (a
 * Monarch decomposition, Approach) inside the library's kernels.
 *
 * Conventions shared by every entry point:
 *   - Every data pointer is a DEVICE pointer unless its name ends in _host.
 *     The caller owns and allocates every buffer passed in; the library owns
 *     only what a plan allocates (its tables and its workspace).
 *   - Tensors are row-major with the sequence index fastest: u, w, v, y are
 *     [B, H, N]; k is [H, L].  Their element type is the plan dtype.
 *   - Device pointers must be 16-byte aligned.
 *   - All calls return an fftconv_status_t (0 = success).  On failure nothing
 *     has been launched and fftconv_last_error() describes the cause
 *     (thread-local).  Nothing throws across the ABI.
 *   - Calls taking a cudaStream_t are asynchronous on that stream, allocate
 *     no memory and do not synchronise (except where noted).
 */
#ifndef FFTCONV_H_
#define FFTCONV_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FFTCONV_API __attribute__((visibility("default")))
#else
#define FFTCONV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Opaque stream handle; identical to cudaStream_t (NULL = legacy default). */
typedef struct CUstream_st* fftconv_stream_t;

typedef struct fftconv_plan_s* fftconv_plan_t;

typedef enum {
    FFTCONV_F32 = 0,   /* float                    */
    FFTCONV_F16 = 1,   /* IEEE binary16 (__half)   */
    FFTCONV_BF16 = 2   /* bfloat16 (__nv_bfloat16) */
} fftconv_dtype_t;

typedef enum {
    FFTCONV_OK = 0,
    FFTCONV_ERR_INVALID_ARG = -1,   /* null/negative/mismatched argument      */
    FFTCONV_ERR_UNSUPPORTED = -2,   /* valid but not implemented (e.g. N=3000) */
    FFTCONV_ERR_ALIGNMENT = -3,     /* pointer not 16-byte aligned            */
    FFTCONV_ERR_CUDA = -4,          /* a CUDA runtime call or launch failed   */
    FFTCONV_ERR_OOM = -5,           /* plan allocation failed                 */
    FFTCONV_ERR_TIMEOUT = -6,       /* a bounded device wait gave up          */
    FFTCONV_ERR_RANGE = -7          /* non-finite result: an fp16 intermediate
                                       of a 16-bit tensor-core plan overflowed
                                       (or an input held inf/NaN); see below  */
} fftconv_status_t;

/* Range of the 16-bit tensor-core paths (FFTCONV_PATH_TC_FUSED and
 * FFTCONV_PATH_TC_STAGED).  Their transform intermediates are fp16 (largest
 * finite value 65504); the fp32 paths (orders 1 and 4) keep fp32 throughout.
 *   - Fused kernel (N <= 4096; N = 8192 and 16384 as two and four blocks
 *     of 4096 or, N = 8192 with a block mask, split by bin parity;
 *     overlap-save windows): each unitary stage can grow a value by at most
 *     the number of its inputs over the square root of its length, so with
 *     max|u*w| <= 90 no intermediate can overflow whatever the data and the
 *     filter.  Above that it depends on the data: a constant (DC) input
 *     overflows the forward transform near max|u*w| = 1450, zero-mean random
 *     data stays finite far beyond.
 *   - Staged tensor-core path (order 5 from N = 16384; N >= 32768 with
 *     L > 2049): no data-independent bound is useful; inputs with a large
 *     mean overflow near max|u*w| = 10^3 for R = 2N/8192 = 256 rows per
 *     column.
 * An overflow is never silent: the kernels that write y check the
 * convolution values (before the output gate v; the fused tensor-core kernel
 * checks at least, per pair of rows, the outputs at one position j1 of every
 * residue (l, j3) of t = 256 j1 + 8 l + j3, which every fp16 overflow of its
 * transform reaches) and, if one is inf or NaN, set the plan's status word
 * to FFTCONV_ERR_RANGE, which fftconv_device_status returns (and resets).
 * y then holds the non-finite values; rerun such inputs with an fp32 plan
 * (order 4) or rescale u. */

/* Kernel family a plan uses (fftconv_plan_path). */
typedef enum {
    FFTCONV_PATH_SIMT_FUSED = 1,    /* fp32 FFT in shared memory, one kernel  */
    FFTCONV_PATH_SIMT_STAGED = 2,   /* fp32, column/row passes via workspace  */
    FFTCONV_PATH_TC_FUSED = 3,      /* tcgen05 tensor-core Monarch, one kernel */
    FFTCONV_PATH_TC_STAGED = 4      /* staged, tensor-core row pass of 8192    */
} fftconv_path_t;

/* Create a plan for sequences of length N (a power of two, 256 <= N <= 2^22)
 * and H channels with full-length filters (L = N).
 *
 * `order` is the Monarch order of the decomposition, the number of DFT-factor
 * levels the length-2N transform is split into ("Approach": order-p Monarch
 * decomposition), read as a request for where the intermediate lives:
 *   0     automatic (the fastest kernel this library has for the plan);
 *   2, 3  fused: one kernel, the transform stays on chip (no intermediate in
 *         device memory).  This library's fused kernels split every transform
 *         they hold into three levels, so 2 and 3 are the same request.  They
 *         exist for N <= 16384 (tensor cores for fp16/bf16 at N = 256 ..
 *         16384: N = 8192 and 16384 as two and four blocks of 4096 in one
 *         tile, N = 8192 with a block mask as the 16384-point spectrum split
 *         by bin parity; fp32 lanes up to 8192 otherwise) and, with filters
 *         of at most 2049 taps, for longer N as overlap-save windows of one
 *         fused transform each.  A four-block plan (N = 16384) stores
 *         8192-point filter rows: it rejects block masks and
 *         fftconv_filter_to_rfft (FFTCONV_ERR_UNSUPPORTED; order 5 serves
 *         them).  Orders 2 and 3 at N > 16384 with L > 2049 return
 *         FFTCONV_ERR_UNSUPPORTED: no fused kernel holds that transform on
 *         chip; orders 0, 4 and 5 serve it;
 *   4     staged: one intermediate pass through a plan-owned workspace in
 *         device memory (column passes, a row pass, inverse column passes),
 *         fp32 lanes throughout, any N.
 * Two further values select an engine inside those families:
 *   1     fused on fp32 lanes (N <= 8192), whatever the dtype;
 *   5     staged, with the row pass on the tensor cores (fp16/bf16,
 *         16384 <= N <= 2^22, L > 2049).  Order 0 chooses it for N >= 32768,
 *         as overlap-save windows of 2 x hop points when the filter is at most
 *         half the sequence (hop = the power of two >= max(L, 16384)); such a
 *         windowed plan rejects block masks and fftconv_filter_to_rfft with
 *         FFTCONV_ERR_UNSUPPORTED, order 5 keeps the full transform.
 * Other values are FFTCONV_ERR_UNSUPPORTED.  fftconv_plan_path reports the
 * kernel family chosen.  Synchronous: allocates the plan's device tables (a
 * few hundred KB) and, on the staged paths, its workspace (about 64 MB for
 * order 4, 512 MB for the tensor-core staged path; fftconv_workspace_bytes) on
 * the current device.  *out receives the plan, or NULL on failure. */
FFTCONV_API int fftconv_plan_create(fftconv_plan_t* out, int64_t N, int64_t H,
                        fftconv_dtype_t dtype, int order);

/* As fftconv_plan_create with a filter of length L (1 <= L <= N): the
 * partial convolution, defined as the convolution with k zero-padded to N
 * (FlashFFTConv: Efficient Convolutions for Long Sequences with Tensor Cores,
 * summary and "Approach": partial convolutions).
 * With a 16-bit dtype, N >= 32768 and L <= 2049, orders 0, 2 and 3 choose the
 * tensor-core path as overlap-save: windows of 4096 inputs with hop 2048, each
 * one 8192-point transform, N/2048 - 1 windows per sequence.  Such a plan
 * stores the 8192-point filter spectrum, so fftconv_forward rejects a
 * block_mask and fftconv_filter_to_rfft is unsupported on it
 * (FFTCONV_ERR_UNSUPPORTED); orders 1 and 4 keep the 2N-point spectrum. */
FFTCONV_API int fftconv_plan_create_ex(fftconv_plan_t* out, int64_t N, int64_t H,
                           fftconv_dtype_t dtype, int order, int64_t L);

/* Release a plan and its device memory (synchronises the device first).
 * NULL is accepted. */
FFTCONV_API int fftconv_plan_destroy(fftconv_plan_t plan);

/* Bytes of the opaque transformed filter K_f for this plan (0 for NULL). */
FFTCONV_API size_t fftconv_filter_bytes(fftconv_plan_t plan);

/* Bytes of the plan's own device workspace (0 on the fused paths). */
FFTCONV_API size_t fftconv_workspace_bytes(fftconv_plan_t plan);

/* The kernel family this plan dispatches to (an fftconv_path_t), or <0. */
FFTCONV_API int fftconv_plan_path(fftconv_plan_t plan);

/* K_f <- rfft(k zero-padded to 2N) in the plan's internal (digit-permuted)
 * layout with the 1/(2N) normalisation folded in.  k: [H, L] device, plan
 * dtype.  K_f: device, fftconv_filter_bytes(plan) bytes, written completely.
 * Run once per filter; the result is reused by every forward call. */
FFTCONV_API int fftconv_filter_precompute(fftconv_plan_t plan, const void* k, void* K_f,
                              fftconv_stream_t stream);

/* y <- causal convolution of u (gated by w and v) with the filter K_f.
 *   u, y       : [B, H, N] device, plan dtype.  y must not overlap u, w or v.
 *   K_f        : from fftconv_filter_precompute on this plan.
 *   B, H, N    : B >= 0; H and N must equal the plan's.  B == 0 is a no-op.
 *   w, v       : [B, H, N] device or NULL (absent gate = all ones).
 *   block_mask : NULL, or [mask_h, N/32] device bytes; block m covers rfft
 *                bins [32m, 32m+32) of each channel's filter (the last block
 *                also holds the Nyquist bin N); 0 zeroes those bins (and their
 *                Hermitian mirrors), anything else keeps them.
 *   mask_h     : 1 (one mask row for all channels) or H; ignored when
 *                block_mask is NULL.  A block_mask on an overlap-save plan
 *                (see fftconv_plan_create_ex) is FFTCONV_ERR_UNSUPPORTED.
 * Asynchronous on `stream`; allocates nothing.  Calls on the staged path
 * share the plan's workspace and must be serialised on one stream. */
FFTCONV_API int fftconv_forward(fftconv_plan_t plan, const void* u, const void* K_f, void* y,
                    int64_t B, int64_t H, int64_t N, const void* w, const void* v,
                    const uint8_t* block_mask, int64_t mask_h,
                    fftconv_stream_t stream);

/* fftconv_forward with a Monarch-aligned frequency mask (FlashFFTConv:
 * Efficient Convolutions for Long Sequences with Tensor Cores, "Approach":
 * frequency-sparse convolutions skip blocks of the Monarch matrix products;
 * "Key results": up to 79% frequency sparsity).  For tensor-core plans with
 * N = 4096 (fftconv_plan_path == FFTCONV_PATH_TC_FUSED): the 2N = 8192-point
 * filter spectrum index is written f = c1 + 32 c2 + 1024 c3 (c1, c2 < 32,
 * c3 < 8), the digits of the kernel's order-3 decomposition; bit c2 of
 * keep_c2 keeps the bins with that middle digit.  A bin f is used only when
 * the c2 of f and the c2 of its mirror (8192 - f) mod 8192 are both kept, so
 * the masked spectrum stays Hermitian and y real (keep sets closed under
 * c2 -> 31 - c2 lose only the bins f = 0 mod 32 at their edges).  The work of
 * a masked c2 is skipped, not zeroed: its forward and inverse 8-point stage
 * products (tcgen05 MMAs) and their epilogue work, and every K step of the
 * 32-point inverse stage whose eight c2 are all masked.
 *   keep_c2 : 0xffffffff is the unmasked call; 0 gives y = 0.
 * Other arguments as fftconv_forward (no block_mask).  Other plans:
 * FFTCONV_ERR_UNSUPPORTED.  Asynchronous on `stream`; allocates nothing. */
FFTCONV_API int fftconv_forward_monarch(fftconv_plan_t plan, const void* u, const void* K_f, void* y,
                            int64_t B, int64_t H, int64_t N, const void* w, const void* v,
                            uint32_t keep_c2, fftconv_stream_t stream);

/* Gradients of y = v * conv(u * w, k) for the incoming gradient dy, for
 * training (FlashFFTConv: Efficient Convolutions for Long Sequences with Tensor
 * Cores, "Key results": the convolution inside trained models; the page gives
 * no backward, so these are the plain adjoints of the forward definition).
 * With g = dy * v and the correlation c[t] = sum_{s<L, t+s<N} g[t+s] k[s]:
 *     du = w * c,   dw = u * c,   dv = dy * conv(u * w, k),
 *     dk[h, s] = sum_b sum_t g_b[t] (u*w)_b[t-s]   for s < L.
 *   u, w, v, dy   : [B, H, N] device, plan dtype (w, v may be NULL: ones).
 *   K_f           : from fftconv_filter_precompute on this plan.
 *   du            : [B, H, N] device, plan dtype, required.
 *   dw, dv        : [B, H, N] device or NULL (not computed); dw needs w and
 *                   dv needs v.
 *   dk            : [H, L] fp32 device or NULL; overwritten with the sum over
 *                   the batch (the call clears it first).
 * Outputs must not overlap each other or any input.  Supported on fp16/bf16
 * tensor-core plans with N <= 8192 (fftconv_plan_path ==
 * FFTCONV_PATH_TC_FUSED); other plans return FFTCONV_ERR_UNSUPPORTED.  du and
 * dw come from one launch of the fused tensor-core kernel with the product by
 * conj(K_f) (correlation; at N = 8192 as two blocks of 4096, block 0 adding
 * block 1's spectrum times conj(G_1)) and two gated outputs, dv from the forward kernel
 * with dy as the output gate, dk from fp32 transforms of dy*v and u*w per
 * (channel, batch chunk).  Asynchronous on `stream`; allocates nothing.  The
 * fp16 range note above applies to du, dw, dv (FFTCONV_ERR_RANGE). */
FFTCONV_API int fftconv_backward(fftconv_plan_t plan, const void* u, const void* K_f, const void* dy,
                                 int64_t B, int64_t H, int64_t N, const void* w, const void* v,
                                 void* du, void* dw, void* dv, float* dk, fftconv_stream_t stream);

/* Device bytes fftconv_forward_host needs as staging for B rows with the
 * given gates and mask present (nonzero = present). */
FFTCONV_API size_t fftconv_forward_host_staging_bytes(fftconv_plan_t plan, int64_t B, int has_w,
                                          int has_v, int has_mask, int64_t mask_h);

/* fftconv_forward on HOST buffers: copies u_host (and w_host, v_host,
 * mask_host) into the caller's device staging buffer, runs the forward pass
 * and copies y back into y_host.  The work is pipelined over up to 8 chunks of
 * batch rows: uploads run on a plan-owned copy stream, each chunk's forward
 * pass on `stream`, downloads on a second plan-owned copy stream, so the two
 * copy directions and the compute overlap.  The call as a whole is ordered on
 * `stream` (it starts after the stream's earlier work; later work on the
 * stream sees y_host written) and returns without waiting (page-locked host
 * memory keeps the copies asynchronous; pageable memory works but blocks).
 * Calls on one plan share its copy streams and must be issued from one host
 * thread in order.  K_f stays a device pointer.  staging: device, at least
 * fftconv_forward_host_staging_bytes(...) bytes, 256-byte aligned. */
FFTCONV_API int fftconv_forward_host(fftconv_plan_t plan, const void* u_host, const void* K_f,
                         void* y_host, int64_t B, int64_t H, int64_t N,
                         const void* w_host, const void* v_host,
                         const uint8_t* mask_host, int64_t mask_h, void* staging,
                         size_t staging_bytes, fftconv_stream_t stream);

/* fftconv_forward without a plan and without allocating: for callers that
 * may not call cudaMalloc at all (code inside a host framework whose memory
 * pool owns every byte of device memory, or latency-critical paths that
 * cannot pay for cudaMalloc's implicit synchronisation).  It runs the staged
 * passes of an order-4 plan, with their intermediate spectra and twiddle
 * tables in the library's own statically allocated device arrays (16 MiB of
 * scratch, held on every GPU that loads the library until the process exits).
 * The FlashFFTConv page has no counterpart for this entry point.
 *   u, y, w, v, block_mask, mask_h, B: as for fftconv_forward (device memory,
 *     16-byte aligned; w, v, block_mask may be NULL).
 *   K_f : the filter transform that fftconv_filter_precompute wrote for an
 *     order-4 plan with the same N, H and dtype (made once, by code that may
 *     allocate, e.g. when the filter is loaded).  It is read as that layout,
 *     H x 2N complex fp32 values: a K_f from a plan of any other order is both
 *     the wrong layout and too short, so the call would read past its end.
 *   N   : power of two, 256 <= N <= 2^20 (2N complex fp32 values must fit the
 *     scratch); larger N returns FFTCONV_ERR_UNSUPPORTED with the limit in
 *     fftconv_last_error().
 * Calls no cudaMalloc/cudaFree and allocates nothing else.  Every call looks up
 * the device addresses of the static arrays in the calling thread's current
 * context (cudaGetSymbolAddress); the first call on a device may load the
 * library's device code there, so make that first call before any stream
 * capture.  The passes' twiddle tables live in the static arrays too and are
 * refilled only when N or the context differs from the previous call on that
 * device.  All calls share these arrays and each call overwrites the scratch,
 * so calls whose execution overlaps on the GPU (other streams, other host
 * threads) race; serialise them (a call also relies on the tables an earlier
 * call of the same N filled having been written). */
FFTCONV_API int fftconv_forward_noalloc(const void* u, const void* K_f, void* y, int64_t B, int64_t H,
                                        int64_t N, fftconv_dtype_t dtype, const void* w, const void* v,
                                        const uint8_t* block_mask, int64_t mask_h,
                                        fftconv_stream_t stream);

/* Test hook: export K_f in natural order as out[h, f, 0..1] = (Re, Im) of
 * rfft(k)[f] for f in [0, N] (normalisation undone), fp32, device.
 * FFTCONV_ERR_UNSUPPORTED on an overlap-save plan (see fftconv_plan_create_ex). */
FFTCONV_API int fftconv_filter_to_rfft(fftconv_plan_t plan, const void* K_f, float* out,
                           fftconv_stream_t stream);

/* Synchronise `stream` and return the plan's device status word:
 * FFTCONV_OK, FFTCONV_ERR_TIMEOUT if a bounded device-side wait gave up, or
 * FFTCONV_ERR_RANGE if a 16-bit tensor-core forward produced non-finite
 * values (see the range note above), since the last call (the word is reset
 * to OK by this call). */
FFTCONV_API int fftconv_device_status(fftconv_plan_t plan, fftconv_stream_t stream);

/* Self-test of the device-side failure path (the pages describe none; this
 * exists so the bounded waits can be tested without faulting a GPU).  Launches
 * one warp on `stream` that waits on an on-chip barrier with the convolution
 * kernels' bounded wait, giving up after `polls` (1 <= polls <= 2^20) blocking
 * polls.  arrive != 0: the barrier is signalled first and the wait succeeds;
 * arrive == 0: nothing signals it, the wait gives up and the plan's status
 * word becomes FFTCONV_ERR_TIMEOUT (read and reset by fftconv_device_status).
 * Asynchronous; allocates nothing; the context stays usable. */
FFTCONV_API int fftconv_selftest_bounded_wait(fftconv_plan_t plan, int64_t polls, int arrive,
                                  fftconv_stream_t stream);

/* Static description of a status code. */
FFTCONV_API const char* fftconv_status_string(int status);

/* Detail of the last failure on the calling thread ("" if none). */
FFTCONV_API const char* fftconv_last_error(void);

/* Library version string. */
FFTCONV_API const char* fftconv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FFTCONV_H_ */
