// down_f16.cu -- weight pre-pass for the down projection's fp16 operands (stage 4, the down
// half of expert(x) = W_down(SiLU(W_gate x) * W_up x); Qwen3.8-Flash-Next architecture
// study, MoE section).
//
// The down GEMM can take h as one fp16 value per element instead of the bf16 pair
// (hi, lo). The tensor core's f16 MMA needs both operands in one format, so W_down is
// re-encoded once, at load time, as W' = fp16(W * 2^8); the gate|up epilogue then stores
// h' = fp16(h * 2^-8), and W' h' = W h with no rescaling in the epilogue. A bf16 value w
// with 2^-25 <= |w| < 256 (or w = 0) has at most 8 significant bits and an exponent that
// fp16 holds after the 2^8 shift, so the re-encoding is exact there; smaller magnitudes
// round to the nearest multiple of 2^-32 (an error of at most 2^-33), larger ones saturate
// at 65504 * 2^-8 and raise the range flag. One thread per 8 weights, 16-byte accesses.
#include <cuda_fp16.h>

#include <algorithm>

#include "device_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

__device__ __forceinline__ uint16_t to_f16_x256(uint16_t b, bool& saturated) {
  float f = __uint_as_float((uint32_t)b << 16) * 256.0f;  // exact (a power of two)
  if (fabsf(f) > 65504.0f) {  // includes inf; NaN passes through as NaN
    f = copysignf(65504.0f, f);
    saturated = true;
  }
  return __half_as_ushort(__float2half_rn(f));
}

__global__ void __launch_bounds__(256)
down_to_f16_kernel(const uint16_t* __restrict__ w, size_t n8, uint16_t* __restrict__ out,
                   uint32_t* __restrict__ status) {
  bool saturated = false;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8;
       i += (size_t)gridDim.x * blockDim.x) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(w) + i);
    const uint32_t in[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint16_t lo = to_f16_x256((uint16_t)(in[q] & 0xFFFFu), saturated);
      const uint16_t hi = to_f16_x256((uint16_t)(in[q] >> 16), saturated);
      o[q] = (uint32_t)lo | ((uint32_t)hi << 16);
    }
    reinterpret_cast<uint4*>(out)[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  if (__any_sync(0xffffffffu, saturated) && (threadIdx.x & 31) == 0) set_flag(status, kFlagRange);
}

}  // namespace

cudaError_t launch_down_to_f16(const uint16_t* w, size_t n, uint16_t* out, uint32_t* status,
                               int sms, cudaStream_t st) {
  LaunchScope scope(MOE_K_OTHER, st);
  const size_t n8 = n / 8;
  const size_t blocks = std::min<size_t>((n8 + 255) / 256, (size_t)sms * 8);
  down_to_f16_kernel<<<(unsigned)std::max<size_t>(blocks, 1), 256, 0, st>>>(w, n8, out, status);
  return cudaGetLastError();
}

}  // namespace moe
