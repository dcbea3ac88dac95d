// Grouped GEMM with fine-grained FP8 operands (placeholder until the tcgen05
// FP8 kernel lands).
#include "common.cuh"

namespace moe {

cudaError_t launch_grouped_gemm_fp8(const void*, const float*, const void*, const float*,
                                    const int32_t*, int, int, int, int, bool, void*, float*, int,
                                    int32_t*, cudaStream_t, const char** why) {
  *why = "FP8 grouped GEMM is not available in this build";
  return cudaErrorNotSupported;
}

}  // namespace moe
