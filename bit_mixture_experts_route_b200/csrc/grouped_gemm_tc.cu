// Grouped NF4 GEMM, prefill path (tcgen05 tensor cores, TMEM accumulators).
// Not yet available in this build: the dispatcher routes every size to the
// GEMV kernel.
#include "common.cuh"

namespace moe_launch {

bool grouped_gemm_tc_supported(int, int, moe_epilogue_t) { return false; }

cudaError_t grouped_gemm_tc(const void*, moe_dtype_t, int, const int32_t*, int, const uint8_t*,
                            const float*, const int32_t*, int, int, int, int, moe_epilogue_t,
                            void*, moe_dtype_t, int32_t*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace moe_launch
