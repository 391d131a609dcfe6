// tc_gemm.cu -- tensor-core grouped GEMMs (not built yet: the streaming kernels serve).
#include "tc_gemm.h"

namespace moe {

bool tc_supported(const moe_shape&) { return false; }

cudaError_t launch_tc_gate_up(const moe_shape&, const Layout&, char*, const uint16_t*,
                              const int32_t*, const moe_weights&, cudaStream_t) {
  return cudaErrorNotSupported;
}

cudaError_t launch_tc_down(const moe_shape&, const Layout&, char*, const int32_t*, const float*,
                           const float*, const moe_weights&, float*, float*, float*,
                           cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace moe
