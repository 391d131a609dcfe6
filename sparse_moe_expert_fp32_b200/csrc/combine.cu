// combine.cu -- stage 5, "Weighted combine + gated shared expert" (Qwen3.8-Flash-Next
// architecture study, MoE section, layer formula
// MoE(x) = sum_{e in top-k} p_e expert_e(x) + sigmoid(w_shared x) shared(x)),
// plus the bounded wait used by the failure-detection check.
#include "device_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

// out[t, :] = sum_j w[t,j] * y[assign_row[t,j], :] + sg[t] * y_shared[t, :], in that order.
// One CTA per token, float4 over the hidden dimension (coalesced rows of y).
__global__ void __launch_bounds__(256)
combine_kernel(const float* __restrict__ y, const float* __restrict__ y_shared,
               const int32_t* __restrict__ assign_row, const float* __restrict__ topk_w,
               const float* __restrict__ sgate, float* __restrict__ out, int H, int k, int R) {
  const int t = blockIdx.x;
  __shared__ int rows[kMaxK];
  __shared__ float wts[kMaxK];
  if (threadIdx.x < k) {
    rows[threadIdx.x] = assign_row[(size_t)t * k + threadIdx.x];
    wts[threadIdx.x] = topk_w[(size_t)t * k + threadIdx.x];
  }
  __syncthreads();
  const float sg = sgate[t];
  for (int c = threadIdx.x; c < H / 4; c += blockDim.x) {
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
      if ((unsigned)rows[j] >= (unsigned)R) continue;  // not a packed row: contributes nothing
      const float4 v = __ldg(reinterpret_cast<const float4*>(y + (size_t)rows[j] * H) + c);
      const float wj = wts[j];
      a.x = fmaf(wj, v.x, a.x);
      a.y = fmaf(wj, v.y, a.y);
      a.z = fmaf(wj, v.z, a.z);
      a.w = fmaf(wj, v.w, a.w);
    }
    const float4 s = __ldg(reinterpret_cast<const float4*>(y_shared + (size_t)t * H) + c);
    a.x = fmaf(sg, s.x, a.x);
    a.y = fmaf(sg, s.y, a.y);
    a.z = fmaf(sg, s.z, a.z);
    a.w = fmaf(sg, s.w, a.w);
    reinterpret_cast<float4*>(out + (size_t)t * H)[c] = a;
  }
}

// Waits for *flag != 0 at most timeout_ns; on expiry records the timeout flag and returns.
__global__ void wait_flag_kernel(const int32_t* flag, uint64_t timeout_ns, uint32_t* status) {
  if (threadIdx.x != 0) return;
  const volatile int32_t* f = flag;
  const uint64_t t0 = globaltimer_ns();
  while (*f == 0) {
    if (globaltimer_ns() - t0 > timeout_ns) {
      set_flag(status, kFlagTimeout);
      return;
    }
    __nanosleep(256);
  }
}

}  // namespace

cudaError_t launch_combine(const moe_shape& s, const float* y, const float* y_shared,
                           const int32_t* assign_row, const float* topk_w, const float* sgate,
                           float* out, cudaStream_t st) {
  LaunchScope scope(MOE_K_COMBINE, st);
  combine_kernel<<<s.T, 256, 0, st>>>(y, y_shared, assign_row, topk_w, sgate, out, s.H, s.k,
                                      s.T * s.k);
  return cudaGetLastError();
}

cudaError_t launch_wait_flag(const int32_t* flag, uint64_t timeout_ns, uint32_t* status,
                             cudaStream_t st) {
  LaunchScope scope(MOE_K_OTHER, st);
  wait_flag_kernel<<<1, 32, 0, st>>>(flag, timeout_ns, status);
  return cudaGetLastError();
}

}  // namespace moe
