// tc_common.cuh -- pieces shared by the tensor-core kernels (tc_gemm.cu: one CTA per tile;
// tc2_gemm.cu: CTA pairs): kernel arguments, the grouped-GEMM tile decoding, bounded
// mbarrier waits, and tensor-map encoding on the host. Internal to libmoe_b200.so.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>

#include <mutex>

#include "device_common.cuh"
#include "moe_internal.h"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // a pipeline wait longer than this is a fault
constexpr uint64_t kDrainLimitNs = 200000000ull;  // waits while leaving after an abort

struct TcArgs {
  const int* plan;
  int E, H, I, Is, T, k, ldh;
  size_t h_plane;
  const int32_t* sorted_token;
  const float* sorted_w;
  const float* sgate;
  uint16_t* h;
  float* y;
  float* y_shared;
  float* out;
  uint32_t* status;
  float* logits;      // router: [T][E]
  int ntiles;         // router: tile count (no plan)
  int* counter;       // next tile to hand out (zeroed before the launch)
  int* counter_next;  // gate|up: the down kernel's counter, zeroed here for its launch
  int h_f16;          // gate|up: store h as fp16(h * 2^-8) in plane 0 (fp16 down operands)
};

struct Tile {
  int g, m, p0, nvalid, N;
};

// Tile -> (group, M tile, packed rows). Groups own consecutive tile ranges
// [tp[g], tp[g+1]); a group of more than max_tile rows is split into near-equal chunks
// whose tiles are adjacent.
__device__ __forceinline__ Tile decode_tile(const int* row0, const int* tp, int E, int tile,
                                            int max_tile) {
  int lo = 0, hi = E + 1;  // tp[lo] <= tile < tp[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (tp[mid] <= tile) lo = mid;
    else hi = mid;
  }
  Tile t;
  t.g = lo;
  const int n = row0[lo + 1] - row0[lo];
  const int nch = (n + max_tile - 1) / max_tile;
  const int cs = (((n + nch - 1) / nch) + 15) & ~15;
  const int local = tile - tp[lo];
  t.m = local / nch;
  const int c = local - t.m * nch;
  const int start = c * cs;
  t.nvalid = min(cs, n - start);
  t.N = (t.nvalid + 15) & ~15;
  t.p0 = row0[lo] + start;
  return t;
}

// Bounded wait on an mbarrier phase; false if it ran out (flag recorded) or another role
// already gave up. The fast path is one non-blocking test (a blocking try_wait costs ~170
// cycles even on a completed phase, idle time for the tensor core when the MMA-issuing
// thread pays it); the waiting loop is out of line so that the issue loops stay short.
template <class State>
__device__ __noinline__ bool wait_phase_slow(uint64_t* bar, uint32_t parity, State& S,
                                             uint32_t* status) {
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t spin = 1;; ++spin) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((spin & 31) == 0) {
      if (S.abort) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        S.abort = 1;
        set_flag(status, kFlagTimeout);
        return false;
      }
    }
  }
}

template <class State>
__device__ __forceinline__ bool wait_phase(uint64_t* bar, uint32_t parity, State& S,
                                           uint32_t* status) {
  if (ptx::mbar_test_wait(bar, parity)) return true;
  return wait_phase_slow(bar, parity, S, status);
}

// Short bounded wait used while leaving after an abort.
__device__ __forceinline__ void drain_phase(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!ptx::mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kDrainLimitNs) return;
  }
}

// h = SiLU(gate) * up for the down GEMM: the bf16 pair (hi = bf16(h) at h[at], lo =
// bf16(h - hi) at h[plane + at], about 16 significant bits) or, when the down operands are
// fp16, h' = fp16(h * 2^-8) at h[at] (11 significant bits down to |h| = 2^-6; W' = W * 2^8
// makes W' h' = W h). A value beyond fp16's range saturates and raises the range flag.
__device__ __forceinline__ void store_h(uint16_t* h, size_t plane, size_t at, float hv, int f16,
                                        uint32_t* status) {
  if (f16) {
    float v = hv * 0.00390625f;  // 2^-8, exact
    if (fabsf(v) > 65504.f) {
      v = copysignf(65504.f, v);
      set_flag(status, kFlagRange);
    }
    h[at] = __half_as_ushort(__float2half_rn(v));
  } else {
    const uint16_t hi = f32_to_bf16_rn(hv);
    h[at] = hi;
    h[plane + at] = f32_to_bf16_rn(hv - bf16lo(hi));
  }
}

__device__ __forceinline__ int token_of_row(const TcArgs& a, int p, int R) {
  if (p >= R) return p - R;
  const int t = a.sorted_token[p];
  if ((unsigned)t >= (unsigned)a.T) {
    set_flag(a.status, kFlagBounds);
    return 0;
  }
  return t;
}

// ---------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D tensor of 2-byte elements [outer][inner] (inner contiguous; bf16 unless `dt` says
// fp16), box [box_outer][box_inner] with the swizzle matching box_inner (64 elements:
// 128-byte swizzle, 32: 64-byte swizzle).
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
              uint32_t box_inner, uint32_t box_outer,
              CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * sizeof(uint16_t)};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw =
      box_inner == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// n-D tensor of 2-byte elements (bf16 unless `dt` says fp16): dims innermost first,
// strides (bytes) of dims 1..n-1, box per dim; the 128-byte swizzle (64-element rows).
bool make_map_nd(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
                 const uint64_t* strides, const uint32_t* box,
                 CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  auto fn = encode_fn();
  if (!fn || rank < 2 || rank > 5) return false;
  cuuint64_t d[5], st[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
    if (i + 1 < rank) st[i] = strides[i];
  }
  return fn(m, dt, (cuuint32_t)rank, const_cast<void*>(base), d, st, bx, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

TcArgs base_args(const moe_shape& s, const Layout& L, char* ws) {
  TcArgs a{};
  a.plan = reinterpret_cast<const int*>(ws + L.plan);
  a.E = s.E;
  a.H = s.H;
  a.I = s.I;
  a.Is = s.Is;
  a.T = s.T;
  a.k = s.k;
  a.ldh = L.ldh;
  a.h_plane = L.h_plane;
  a.h = reinterpret_cast<uint16_t*>(ws + L.h);
  a.status = reinterpret_cast<uint32_t*>(ws + L.status);
  return a;
}

}  // namespace
}  // namespace moe
