// fp8_quant.cu -- the FP8 expert pre-pass: bf16 routed-expert banks -> E4M3 codes with one
// fp32 scale per weight row ("Qwen3.8, weights in hand: 98% of a 2.4T model is routed
// experts", section "What FP8 actually quantizes": the routed experts are the part stored
// in FP8; the format and its scaling are this library's reading, stated in include/moe.h).
//
//   scale = amax_row / 448           (IEEE fp32 division; 0 for an all-zero row)
//   code  = E4M3 RNE of (w / scale)  (IEEE fp32 division; saturating at +-448)
//
// One warp per weight row; 16-byte loads of bf16 and 16-byte stores of codes. Run once at
// load time; HBM-bound (reads 2 bytes and writes 1 byte per weight).
#include <cuda_fp8.h>

#include "device_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t u16) { return __uint_as_float(u16 << 16); }

__device__ __forceinline__ uint32_t pack4_e4m3(float a, float b, float c, float d, float inv_ok,
                                               float scale) {
  // inv_ok == 0: a zero row, every code 0 (no division by a zero scale)
  uint32_t r = 0;
  const float v[4] = {a, b, c, d};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float q = inv_ok != 0.f ? __fdiv_rn(v[i], scale) : 0.f;
    r |= (uint32_t)__nv_cvt_float_to_fp8(q, __NV_SATFINITE, __NV_E4M3) << (8 * i);
  }
  return r;
}

// rows of n bf16 (n a multiple of 16) -> codes [rows][n], scales [rows]
__global__ void __launch_bounds__(256)
quantize_rows_kernel(const uint16_t* __restrict__ w, size_t rows, int n, uint8_t* __restrict__ q,
                     float* __restrict__ scale) {
  const int lane = threadIdx.x & 31;
  const size_t nwarps = ((size_t)gridDim.x * blockDim.x) >> 5;
  for (size_t row = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; row < rows;
       row += nwarps) {
    const uint16_t* src = w + row * (size_t)n;
    float amax = 0.f;
    for (int c = lane * 8; c < n; c += 256) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + c));
      const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        amax = fmaxf(amax, fabsf(bf16_bits_to_f32(u[i] & 0xFFFFu)));
        amax = fmaxf(amax, fabsf(bf16_bits_to_f32(u[i] >> 16)));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float sc = amax > 0.f ? __fdiv_rn(amax, 448.f) : 0.f;
    if (lane == 0) scale[row] = sc;
    const float ok = sc > 0.f ? 1.f : 0.f;
    uint8_t* dst = q + row * (size_t)n;
    for (int c = lane * 16; c < n; c += 512) {
      const uint4 v0 = __ldg(reinterpret_cast<const uint4*>(src + c));
      const uint4 v1 = __ldg(reinterpret_cast<const uint4*>(src + c + 8));
      const uint32_t u[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
      uint32_t o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        o[i] = pack4_e4m3(bf16_bits_to_f32(u[2 * i] & 0xFFFFu), bf16_bits_to_f32(u[2 * i] >> 16),
                          bf16_bits_to_f32(u[2 * i + 1] & 0xFFFFu),
                          bf16_bits_to_f32(u[2 * i + 1] >> 16), ok, sc);
      *reinterpret_cast<uint4*>(dst + c) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

}  // namespace

cudaError_t launch_quantize_fp8_rows(const uint16_t* w, size_t rows, int n, uint8_t* q,
                                     float* scale, int sms, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  const size_t blocks = (rows + 7) / 8;
  LaunchScope scope(MOE_K_OTHER, st);
  quantize_rows_kernel<<<(int)(blocks < (size_t)sms * 8 ? blocks : (size_t)sms * 8), 256, 0, st>>>(
      w, rows, n, q, scale);
  return cudaGetLastError();
}

}  // namespace moe
