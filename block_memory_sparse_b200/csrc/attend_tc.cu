// Placeholder: tensor-core attention path (replaced by the tcgen05 kernel).
#include "common.cuh"
#include "kernels.h"
namespace infllm {
bool attend_tc_supported(const Dev&) { return false; }
cudaError_t launch_attend_tc(const Dev&, int64_t, int, int, int64_t, void*, cudaStream_t, const void*) {
    return cudaErrorNotSupported;
}
}  // namespace infllm
