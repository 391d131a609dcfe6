// router.cu -- stages 1-2 of the layer: "Router [T, 512]" and "Top 10 + normalize"
// (Qwen3.8-Flash-Next architecture study, MoE section: routing uses an FP32 softmax and
// normalises the selected router probabilities; the shared expert has its own sigmoid
// output gate).
//
//   router_logits_stream_kernel : logits = x . Wr^T on CUDA cores, fp32 accumulation
//                                 (small batches; larger ones use the tensor-core router
//                                 in tc_gemm.cu).
//   router_topk_kernel          : one warp per token: top-k with lowest-index ties,
//                                 renormalised softmax weights, 10th/11th gap,
//                                 shared-expert gate sigmoid(w_shared . x).
#include <float.h>

#include "device_common.cuh"
#include "moe_internal.h"
#include "tc_gemm.h"

namespace moe {
namespace {

constexpr int kRouterWarps = 8;
constexpr int kRowsPerWarp = 8;  // router rows (experts) per warp
constexpr int kTokPerWarp = 4;   // tokens per warp

// logits[t][e] = sum_h x[t][h] * wr[e][h]. A warp computes 8 experts x 4 tokens; lanes
// stride over h in chunks of 4 elements; the 32 partial sums are combined with one
// transpose-reduction. Grid: (ceil(E/64), ceil(T/4)).
__global__ void __launch_bounds__(kRouterWarps * 32)
router_logits_stream_kernel(const uint16_t* __restrict__ x, const float* __restrict__ wr,
                            float* __restrict__ logits, int T, int H, int E) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int e0 = (blockIdx.x * kRouterWarps + warp) * kRowsPerWarp;
  const int t0 = blockIdx.y * kTokPerWarp;
  if (e0 >= E) return;

  float acc[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) acc[i] = 0.f;

  const int nchunk = H / 4;
  for (int c = lane; c < nchunk; c += 32) {
    float xv[kTokPerWarp][4];
#pragma unroll
    for (int q = 0; q < kTokPerWarp; ++q) {
      const int t = t0 + q;
      if (t < T) {
        uint2 u = __ldg(reinterpret_cast<const uint2*>(x + (size_t)t * H + 4 * c));
        xv[q][0] = bf16lo(u.x); xv[q][1] = bf16hi(u.x);
        xv[q][2] = bf16lo(u.y); xv[q][3] = bf16hi(u.y);
      } else {
        xv[q][0] = xv[q][1] = xv[q][2] = xv[q][3] = 0.f;
      }
    }
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
      const int e = e0 + r;
      float4 w = make_float4(0.f, 0.f, 0.f, 0.f);
      if (e < E) w = __ldg(reinterpret_cast<const float4*>(wr + (size_t)e * H + 4 * c));
#pragma unroll
      for (int q = 0; q < kTokPerWarp; ++q) {
        float a = acc[r * 4 + q];
        a = fmaf(w.x, xv[q][0], a);
        a = fmaf(w.y, xv[q][1], a);
        a = fmaf(w.z, xv[q][2], a);
        a = fmaf(w.w, xv[q][3], a);
        acc[r * 4 + q] = a;
      }
    }
  }
  const float s = warp_transpose_sum32(acc, lane);
  const int e = e0 + lane / 4;
  const int t = t0 + lane % 4;
  if (e < E && t < T) logits[(size_t)t * E + e] = s;
}

// One warp per token. Lane l holds logits of experts l, l+32, ...; VPL = values per lane.
template <int VPL>
__global__ void __launch_bounds__(256)
router_topk_kernel(const float* __restrict__ logits, const float* __restrict__ bias,
                   const uint16_t* __restrict__ x, const uint16_t* __restrict__ wsg, int T, int H,
                   int E, int k, int32_t* __restrict__ ids, float* __restrict__ w,
                   float* __restrict__ sgate, float* __restrict__ gap,
                   float* __restrict__ out_zero) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;

  float v[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = lane + 32 * i;
    float l = -FLT_MAX;
    if (e < E) {
      l = logits[(size_t)t * E + e];
      if (bias) l += bias[e];
    }
    v[i] = l;
  }

  uint32_t taken = 0;
  int my_id = 0;
  float my_val = 0.f;
  float next_val = -FLT_MAX;  // (k+1)-th largest
  const int rounds = (k < E) ? k + 1 : k;
  for (int r = 0; r < rounds; ++r) {
    float bv = -FLT_MAX;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !((taken >> i) & 1u) && (v[i] > bv || (v[i] == bv && e < bi))) {
        bv = v[i];
        bi = e;
      }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (bi < E && (bi & 31) == lane) taken |= 1u << (bi >> 5);
    if (r < k) {
      if (lane == r) {
        my_id = bi;
        my_val = bv;
      }
    } else {
      next_val = bv;
    }
  }

  // renormalised softmax over the selected logits: the full-softmax denominator cancels
  const float vmax = __shfl_sync(0xffffffffu, my_val, 0);
  const float ex = (lane < k) ? expf(my_val - vmax) : 0.f;
  const float den = warp_sum(ex);
  if (lane < k) {
    ids[(size_t)t * k + lane] = my_id;
    w[(size_t)t * k + lane] = ex / den;
  }
  const float kth = __shfl_sync(0xffffffffu, my_val, k - 1);
  if (gap && lane == 0) gap[t] = (k < E) ? kth - next_val : __int_as_float(0x7f800000);

  // shared-expert gate: sigmoid(w_shared . x[t])
  float g = 0.f;
  const uint16_t* xr = x + (size_t)t * H;
  for (int c = lane; c < H / 8; c += 32) {
    const uint4 xa = ld_v4(xr + 8 * c);
    const uint4 wa = ld_v4(wsg + 8 * c);
    float xf[8];
    unpack8(xa, xf);
    g = dot8_acc(wa, xf, g);
  }
  g = warp_sum(g);
  if (lane == 0) sgate[t] = 1.f / (1.f + expf(-g));

  if (out_zero) {
    float4* o = reinterpret_cast<float4*>(out_zero + (size_t)t * H);
    for (int c = lane; c < H / 4; c += 32) o[c] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

}  // namespace

cudaError_t launch_router_logits_stream(const moe_shape& s, const uint16_t* x, const float* wr,
                                        float* logits, cudaStream_t st) {
  LaunchScope scope(MOE_K_ROUTER_LOGITS, st);
  dim3 grid((s.E + kRouterWarps * kRowsPerWarp - 1) / (kRouterWarps * kRowsPerWarp),
            (s.T + kTokPerWarp - 1) / kTokPerWarp);
  router_logits_stream_kernel<<<grid, kRouterWarps * 32, 0, st>>>(x, wr, logits, s.T, s.H, s.E);
  return cudaGetLastError();
}

// Token count from which the tensor-core router (a GEMM over the exact three-piece split
// of the router matrix) replaces the CUDA-core one.
constexpr int kTcRouterMinTokens = 512;

cudaError_t launch_router_logits(const moe_shape& s, const Layout& L, char* ws, const uint16_t* x,
                                 const float* wr, float* logits, cudaStream_t st) {
  if (s.T >= kTcRouterMinTokens && tc_router_supported(s))
    return launch_tc_router(s, L, ws, x, wr, logits, st);
  return launch_router_logits_stream(s, x, wr, logits, st);
}

cudaError_t launch_router_topk(const moe_shape& s, const float* logits, const float* bias,
                               const uint16_t* x, const uint16_t* wsg, int32_t* ids, float* w,
                               float* sgate, float* gap, float* out_zero, cudaStream_t st) {
  LaunchScope scope(MOE_K_ROUTER_TOPK, st);
  const int warps = 8;
  dim3 grid((s.T + warps - 1) / warps);
  const int vpl = (s.E + 31) / 32;
#define MOE_TOPK_CASE(N)                                                                     \
  router_topk_kernel<N><<<grid, warps * 32, 0, st>>>(logits, bias, x, wsg, s.T, s.H, s.E, s.k, \
                                                     ids, w, sgate, gap, out_zero)
  if (vpl <= 1) MOE_TOPK_CASE(1);
  else if (vpl <= 2) MOE_TOPK_CASE(2);
  else if (vpl <= 4) MOE_TOPK_CASE(4);
  else if (vpl <= 8) MOE_TOPK_CASE(8);
  else if (vpl <= 16) MOE_TOPK_CASE(16);
  else MOE_TOPK_CASE(32);
#undef MOE_TOPK_CASE
  return cudaGetLastError();
}

}  // namespace moe
