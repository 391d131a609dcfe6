// device_common.cuh -- small device helpers used by several kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ uint16_t f32_to_bf16_rn(float f) {
  __nv_bfloat16 b = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&b);
}

// 16-byte load of data that is read once (weights): bypass L1 allocation.
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint4 ld_v4(const void* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

// Unpack 8 bf16 (one uint4) into floats.
__device__ __forceinline__ void unpack8(const uint4& v, float* f) {
  f[0] = bf16lo(v.x); f[1] = bf16hi(v.x);
  f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
  f[4] = bf16lo(v.z); f[5] = bf16hi(v.z);
  f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
}

// dot of 8 bf16 weights with 8 floats, accumulated into acc
__device__ __forceinline__ float dot8_acc(const uint4& w, const float* x, float acc) {
  acc = fmaf(bf16lo(w.x), x[0], acc); acc = fmaf(bf16hi(w.x), x[1], acc);
  acc = fmaf(bf16lo(w.y), x[2], acc); acc = fmaf(bf16hi(w.y), x[3], acc);
  acc = fmaf(bf16lo(w.z), x[4], acc); acc = fmaf(bf16hi(w.z), x[5], acc);
  acc = fmaf(bf16lo(w.w), x[6], acc); acc = fmaf(bf16hi(w.w), x[7], acc);
  return acc;
}

// Sum each of the 32 per-lane values across the warp; lane l returns the total of
// value index l. 31 shuffles (recursive halving) instead of 32 full reductions.
__device__ __forceinline__ float warp_transpose_sum32(float (&a)[32], int lane) {
#pragma unroll
  for (int half = 16; half >= 1; half >>= 1) {
    const bool upper = (lane & half) != 0;
#pragma unroll
    for (int j = 0; j < half; ++j) {
      float send = upper ? a[j] : a[j + half];
      float keep = upper ? a[j + half] : a[j];
      a[j] = keep + __shfl_xor_sync(0xffffffffu, send, half);
    }
  }
  return a[0];
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void set_flag(uint32_t* status, uint32_t bit) {
  if (status) atomicOr(status, bit);
}

constexpr int kScanThreads = 1024;

// Block-wide exclusive scan of one value per thread; blockDim.x must be kScanThreads (32
// warps). Returns this thread's exclusive prefix; *total receives the block's sum.
__device__ inline int block_exclusive_scan(int v, int* smem_warp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) smem_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int s = smem_warp[lane];
    int si = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, si, o);
      if (lane >= o) si += n;
    }
    smem_warp[lane] = si - s;  // exclusive warp prefix
    if (lane == 31) smem_warp[32] = si;
  }
  __syncthreads();
  const int r = smem_warp[warp] + incl - v;
  *total = smem_warp[32];
  __syncthreads();
  return r;
}

// N block-wide exclusive scans at once (one value of each per thread, one set of barriers);
// blockDim.x must be kScanThreads. smem_warp holds 33 * N ints.
template <int N>
__device__ inline void block_exclusive_scan_n(const int (&v)[N], int (&prefix)[N],
                                              int (&total)[N], int* smem_warp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl[N];
#pragma unroll
  for (int j = 0; j < N; ++j) {
    incl[j] = v[j];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, incl[j], o);
      if (lane >= o) incl[j] += n;
    }
    if (lane == 31) smem_warp[j * 33 + warp] = incl[j];
  }
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int j = 0; j < N; ++j) {
      const int s = smem_warp[j * 33 + lane];
      int si = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, si, o);
        if (lane >= o) si += n;
      }
      smem_warp[j * 33 + lane] = si - s;  // exclusive warp prefix
      if (lane == 31) smem_warp[j * 33 + 32] = si;
    }
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < N; ++j) {
    prefix[j] = smem_warp[j * 33 + warp] + incl[j] - v[j];
    total[j] = smem_warp[j * 33 + 32];
  }
  __syncthreads();
}


}  // namespace moe
