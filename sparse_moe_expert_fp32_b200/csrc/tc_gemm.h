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
                              const int32_t* sorted_token, const moe_weights& w, int h_f16,
                              cudaStream_t st);
cudaError_t launch_tc_down(const moe_shape& s, const Layout& L, char* ws,
                           const int32_t* sorted_token, const float* sorted_w, const float* sgate,
                           const moe_weights& w, float* y, float* y_shared, float* out,
                           cudaStream_t st);

// Token rows in dispatch order (xs[p] = x[sorted_token[p]]) for the gate|up GEMMs' TMA boxes.
cudaError_t launch_gather_rows(const moe_shape& s, const Layout& L, char* ws, const uint16_t* x,
                               const int32_t* sorted_token, cudaStream_t st);

// The same grouped GEMMs on CTA pairs (tcgen05.mma.cta_group::2, M = 256): each SM holds
// half of a token tile, and the down GEMM takes the hi and lo halves of h in one MMA.
// For batches with many tokens per expert (prefill).
cudaError_t launch_tc2_gate_up(const moe_shape& s, const Layout& L, char* ws, const uint16_t* x,
                               const int32_t* sorted_token, const moe_weights& w, int h_f16,
                               cudaStream_t st);
cudaError_t launch_tc2_down(const moe_shape& s, const Layout& L, char* ws,
                            const int32_t* sorted_token, const float* sorted_w, const float* sgate,
                            const moe_weights& w, float* y, float* y_shared, float* out,
                            cudaStream_t st);
// The down GEMM on fp16 operands (w.w_down_f16, w.ws_down_f16 and h' = fp16(h 2^-8) in plane
// 0 of h, written by a gate|up launch with h_f16 = 1): 256-row tiles, one MMA per K step.
cudaError_t launch_tc2_down_f16(const moe_shape& s, const Layout& L, char* ws,
                                const int32_t* sorted_token, const float* sorted_w,
                                const float* sgate, const moe_weights& w, float* y,
                                float* y_shared, float* out, cudaStream_t st);

// The same grouped GEMMs with the routed experts' weights in FP8 (E4M3 codes, one fp32 scale
// per weight row; the shared expert stays bf16): one CTA per tile, E4M3 MMAs on the codes
// against E4M3 pieces of the token operand (two for x, four for h; the down launcher splits
// h first). Any batch size on tensor-core shapes; the down GEMM always combines into `out`.
bool tc8_supported(const moe_shape& s);
cudaError_t launch_tc8_gate_up(const moe_shape& s, const Layout& L, char* ws, const uint16_t* x,
                               const int32_t* sorted_token, const moe_weights& w,
                               const moe_fp8_experts& q, cudaStream_t st);
cudaError_t launch_tc8_down(const moe_shape& s, const Layout& L, char* ws,
                            const int32_t* sorted_token, const float* sorted_w, const float* sgate,
                            const moe_weights& w, const moe_fp8_experts& q, float* out,
                            cudaStream_t st);

}  // namespace moe
