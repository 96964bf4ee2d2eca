// Tensor-core grouped GEMMs (tcgen05 / TMEM / TMA) -- not built yet: the
// launchers report "not supported" so callers see MOE_ERR_UNSUPPORTED.
#include "common.cuh"
#include "launch.h"

namespace moe {

int tc_block_m() { return 128; }

cudaError_t launch_router_logits_tc(const void*, const void*, const float*, int, int, int, float*,
                                    int*, cudaStream_t) {
  return cudaErrorNotSupported;
}
cudaError_t launch_swiglu_tc(const void*, const uint32_t*, const int32_t*, const int32_t*, int,
                             const moe_experts&, void*, int*, cudaStream_t) {
  return cudaErrorNotSupported;
}
cudaError_t launch_down_tc(const void*, const int32_t*, const int32_t*, int, const moe_experts&,
                           void*, int*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace moe
