// tc_kernels.cu -- tcgen05 tensor-core fused path (placeholder until the
// kernel lands: reports itself unsupported so plans fall back to SIMT).
#include "internal.h"

namespace fftconv {

bool tc_supported(int64_t, int64_t, int) { return false; }
cudaError_t tc_plan_init(Plan&) { return cudaErrorNotSupported; }
void tc_plan_free(Plan&) {}
size_t tc_filter_bytes(const Plan&) { return 0; }
cudaError_t tc_precompute(const Plan&, const void*, void*, cudaStream_t) { return cudaErrorNotSupported; }
cudaError_t tc_forward(const Plan&, const ForwardArgs&, cudaStream_t) { return cudaErrorNotSupported; }
cudaError_t tc_export_rfft(const Plan&, const void*, float*, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace fftconv
