/*
 * synth_cuda.cu -- device half of the seeded input generator (see synth_def.h).
 * Fills device buffers with exactly the bits the host half produces, so that the
 * large weight banks (up to 51.5 GB) are made in place on the GPU while the host
 * regenerates only the slices it needs. Inputs only; no step of the MoE layer.
 */
#include <cuda_runtime.h>
#include <stdint.h>

#include "synth_def.h"

namespace {

__global__ void fill_kernel(void* __restrict__ out, uint64_t n, uint64_t key, float sigma,
                            uint64_t index_offset, int bf16, const uint8_t* __restrict__ zero_mask,
                            uint64_t I, uint64_t H) {
  uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t t = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; t < n; t += stride) {
    uint64_t idx = index_offset + t;
    float v;
    bool zeroed = false;
    if (zero_mask) {
      uint64_t row = idx / H;
      uint64_t e = row / (2 * I);
      uint64_t ch = (row % (2 * I)) % I;
      zeroed = zero_mask[e * I + ch] != 0;
    }
    if (zeroed) {
      v = 0.0f;
    } else {
      v = __fmul_rn(synth_std(key, idx), sigma);
    }
    if (bf16)
      static_cast<uint16_t*>(out)[t] = synth_bf16_rne(v);
    else
      static_cast<float*>(out)[t] = v;
  }
}

int launch(void* out, uint64_t n, uint64_t seed, uint32_t tid, float sigma, uint64_t index_offset,
           int bf16, const uint8_t* zero_mask, uint64_t I, uint64_t H, void* stream) {
  if (n == 0) return 0;
  if (!out) return (int)cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  uint64_t blocks = (n + 255) / 256;
  uint64_t cap = (uint64_t)sms * 16;
  if (blocks > cap) blocks = cap;
  fill_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(
      out, n, synth_key(seed, tid), sigma, index_offset, bf16, zero_mask, I, H);
  return (int)cudaGetLastError();
}

}  // namespace

extern "C" {

/* Device buffer of n bf16 elements = elements [index_offset, +n) of tensor tid. */
int synth_cuda_fill_bf16(void* out, uint64_t n, uint64_t seed, uint32_t tid, float sigma,
                         uint64_t index_offset, void* stream) {
  return launch(out, n, seed, tid, sigma, index_offset, 1, nullptr, 1, 1, stream);
}

/* Device buffer of n fp32 elements = elements [index_offset, +n) of tensor tid. */
int synth_cuda_fill_f32(void* out, uint64_t n, uint64_t seed, uint32_t tid, float sigma,
                        uint64_t index_offset, void* stream) {
  return launch(out, n, seed, tid, sigma, index_offset, 0, nullptr, 1, 1, stream);
}

/* Routed gate|up bank [E][2I][H] bf16 with optional device zero mask [E][I]. */
int synth_cuda_fill_gate_up_bf16(void* out, uint64_t E, uint64_t I, uint64_t H, uint64_t seed,
                                 uint32_t tid, float sigma, const uint8_t* zero_mask_dev,
                                 void* stream) {
  return launch(out, E * 2 * I * H, seed, tid, sigma, 0, 1, zero_mask_dev, I, H, stream);
}

}  // extern "C"
