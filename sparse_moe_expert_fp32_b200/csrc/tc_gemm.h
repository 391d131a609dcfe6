// tc_gemm.h -- tensor-core (tcgen05/TMEM, TMA-fed) grouped SwiGLU GEMMs and router GEMM.
#pragma once

#include "moe_internal.h"

namespace moe {

// Can the tensor-core kernels run this shape? (I, Is multiples of 128, H of 256, sm_100.)
bool tc_supported(const moe_shape& s);

// Tensor-core router logits (fp32 router matrix split exactly into three bf16 pieces).
bool tc_router_supported(const moe_shape& s);
cudaError_t launch_tc_router(const moe_shape& s, const Layout& L, char* ws, const uint16_t* x,
                             const float* wr, float* logits, cudaStream_t st);

cudaError_t launch_tc_gate_up(const moe_shape& s, const Layout& L, char* ws, const uint16_t* x,
                              const int32_t* sorted_token, const moe_weights& w, cudaStream_t st);
cudaError_t launch_tc_down(const moe_shape& s, const Layout& L, char* ws,
                           const int32_t* sorted_token, const float* sorted_w, const float* sgate,
                           const moe_weights& w, float* y, float* y_shared, float* out,
                           cudaStream_t st);

}  // namespace moe
