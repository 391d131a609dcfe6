// router.cu -- stages 1-2 of the layer: "Router [T, 512]" and "Top 10 + normalize"
// (Qwen3.8-Flash-Next architecture study, MoE section: routing uses an FP32 softmax and
// normalises the selected router probabilities; the shared expert has its own sigmoid
// output gate).
//
//   router_logits_small_kernel  : logits = x . Wr^T on CUDA cores for small batches, as
//                                 eight partial sums over hidden-dimension slices; larger
//                                 batches use the tensor-core router in tc_gemm.cu.
//   router_topk_kernel          : two warps per token: one takes the top-k with
//                                 lowest-index ties, the renormalised softmax weights and
//                                 the 10th/11th gap, the other the shared-expert gate
//                                 sigmoid(w_shared . x) and the zeroing of the token's
//                                 output row.
#include <float.h>

#include <mutex>

#include "device_common.cuh"
#include "moe_internal.h"
#include "tc_gemm.h"

namespace moe {
namespace {

// Small batches (T < 512): partial logits over kRouterSplits slices of the hidden
// dimension, part[s][t][e] = sum_{h in slice s} x[t][h] * wr[e][h], fp32 FMAs in h order. A
// CTA computes 32 tokens x 64 experts of one slice: x and wr chunks of 320 hidden positions
// (the whole slice at hidden 2560; 120 KB) are staged in shared memory (both transposed: x
// as [h][token], wr as [h][expert]). All of a chunk's global loads are issued at once, into
// registers, so their latency is paid once per chunk; the next chunk's loads are in flight
// while the current one is multiplied. Each thread accumulates 2 tokens x 4 experts: an
// 8-byte and a 16-byte
// shared-memory load (one wavefront each per warp) feed 8 FMAs, so the FMA pipe, not shared
// memory, sets the pace. The top-k kernel adds the slices in order s = 0 .. kRouterSplits-1,
// so the logits are the same on every run. Grid (ceil(E/64), kRouterSplits, ceil(T/32)):
// 128 CTAs at E = 512, T = 64; wr is read once per token block.
constexpr int kSplits = kRouterSplits;
constexpr int kSmallTok = 32;
constexpr int kSmallExp = 64;
constexpr int kSmallKc = 320;
constexpr int kSmallThreads = 256;
constexpr int kSmallXLoads = kSmallTok * (kSmallKc / 8) / kSmallThreads;  // uint4 per thread
constexpr int kSmallWLoads = kSmallExp * (kSmallKc / 4) / kSmallThreads;  // float4 per thread
constexpr size_t kSmallSmem = (size_t)kSmallKc * (kSmallTok + kSmallExp) * sizeof(float);
static_assert(kSmallXLoads * kSmallThreads * 8 == kSmallTok * kSmallKc, "x chunk split");
static_assert(kSplits % 4 == 0, "the top-k kernel adds the slices two or four at a time");
static_assert(kSmallWLoads * kSmallThreads * 4 == kSmallExp * kSmallKc, "wr chunk split");

__global__ void __launch_bounds__(kSmallThreads)
router_logits_small_kernel(const uint16_t* __restrict__ x, const float* __restrict__ wr,
                           float* __restrict__ part, int T, int H, int E, int nslices) {
  extern __shared__ float4 dsm[];
  float* xs_all = reinterpret_cast<float*>(dsm);  // [Kc][Tok]
  float* ws_all = xs_all + kSmallKc * kSmallTok;  // [Kc][Exp]
  const int e0 = blockIdx.x * kSmallExp;
  const int t0 = blockIdx.z * kSmallTok;
  const int slice = H / nslices;  // a multiple of 8 (H is a multiple of 64)
  const int kbeg = blockIdx.y * slice, kend = kbeg + slice;
  const int tid = threadIdx.x;
  const int tg = tid & 15;  // tokens 2 tg, 2 tg + 1
  const int eg = tid >> 4;  // experts 4 eg .. 4 eg + 3
  float acc[2][4] = {};
  uint4 xr[kSmallXLoads];
  float4 wv[kSmallWLoads];

  // global -> registers for the chunk at k0 (zeros outside the tensor)
  auto load = [&](int k0) {
    const int kn = min(kSmallKc, kend - k0);
#pragma unroll
    for (int q = 0; q < kSmallXLoads; ++q) {
      const int i = tid + q * kSmallThreads;
      const int r = i % kSmallTok, c = i / kSmallTok;  // consecutive threads: consecutive tokens
      xr[q] = make_uint4(0u, 0u, 0u, 0u);
      if (8 * c < kn && t0 + r < T) xr[q] = ld_v4(x + (size_t)(t0 + r) * H + k0 + 8 * c);
    }
#pragma unroll
    for (int q = 0; q < kSmallWLoads; ++q) {
      const int i = tid + q * kSmallThreads;
      const int e = i % kSmallExp, c = i / kSmallExp;  // consecutive threads: consecutive experts
      wv[q] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (4 * c < kn && e0 + e < E)
        wv[q] = __ldg(reinterpret_cast<const float4*>(wr + (size_t)(e0 + e) * H + k0) + c);
    }
  };
  // registers -> shared memory
  auto store = [&]() {
    float* xs = xs_all;
    float* ws = ws_all;
#pragma unroll
    for (int q = 0; q < kSmallXLoads; ++q) {
      const int i = tid + q * kSmallThreads;
      const int r = i % kSmallTok, c = i / kSmallTok;
      float f[8];
      unpack8(xr[q], f);
#pragma unroll
      for (int j = 0; j < 8; ++j) xs[(8 * c + j) * kSmallTok + r] = f[j];
    }
#pragma unroll
    for (int q = 0; q < kSmallWLoads; ++q) {
      const int i = tid + q * kSmallThreads;
      const int e = i % kSmallExp, c = i / kSmallExp;
      ws[(4 * c + 0) * kSmallExp + e] = wv[q].x;
      ws[(4 * c + 1) * kSmallExp + e] = wv[q].y;
      ws[(4 * c + 2) * kSmallExp + e] = wv[q].z;
      ws[(4 * c + 3) * kSmallExp + e] = wv[q].w;
    }
  };

  load(kbeg);
  store();
  __syncthreads();
  for (int k0 = kbeg; k0 < kend; k0 += kSmallKc) {
    const bool more = k0 + kSmallKc < kend;
    if (more) load(k0 + kSmallKc);
    const int kn = min(kSmallKc, kend - k0);  // a multiple of 8
    const float2* xs = reinterpret_cast<const float2*>(xs_all) + tg;
    const float4* ws = reinterpret_cast<const float4*>(ws_all) + eg;
    for (int kk = 0; kk < kn; kk += 8) {
      float2 x2[8];
      float4 wv4[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        x2[u] = xs[(kk + u) * (kSmallTok / 2)];
        wv4[u] = ws[(kk + u) * (kSmallExp / 4)];
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {  // h order within each accumulator
        const float xa[2] = {x2[u].x, x2[u].y};
        const float wa[4] = {wv4[u].x, wv4[u].y, wv4[u].z, wv4[u].w};
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(xa[i], wa[j], acc[i][j]);
      }
    }
    if (more) {
      __syncthreads();  // every thread is done reading this chunk
      store();
      __syncthreads();
    }
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int t = t0 + 2 * tg + i;
    if (t >= T) break;
    float* row = part + ((size_t)blockIdx.y * T + t) * E;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = e0 + 4 * eg + j;
      if (e < E) row[e] = acc[i][j];
    }
  }
}

// x[t] . wr[e] in fp32 FMAs (each lane takes every 32nd chunk of 8 elements, four chunks
// in flight, then a warp sum); every lane gets the result.
__device__ __forceinline__ void fma_chunk(const uint4& xa, const float4& a, const float4& b,
                                          float& acc) {
  float xf[8];
  unpack8(xa, xf);
  acc = fmaf(a.x, xf[0], acc); acc = fmaf(a.y, xf[1], acc);
  acc = fmaf(a.z, xf[2], acc); acc = fmaf(a.w, xf[3], acc);
  acc = fmaf(b.x, xf[4], acc); acc = fmaf(b.y, xf[5], acc);
  acc = fmaf(b.z, xf[6], acc); acc = fmaf(b.w, xf[7], acc);
}

__device__ __forceinline__ float exact_logit(const uint16_t* xr, const float* wrow, int H, int lane) {
  const float4* w4 = reinterpret_cast<const float4*>(wrow);
  const int n8 = H / 8;
  float acc = 0.f;
  int c = lane;
  for (; c + 96 < n8; c += 128) {
    uint4 xa[4];
    float4 a[4], b[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int cc = c + 32 * u;
      xa[u] = ld_v4(xr + 8 * cc);
      a[u] = __ldg(w4 + 2 * cc);
      b[u] = __ldg(w4 + 2 * cc + 1);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) fma_chunk(xa[u], a[u], b[u], acc);
  }
  for (; c < n8; c += 32) fma_chunk(ld_v4(xr + 8 * c), __ldg(w4 + 2 * c), __ldg(w4 + 2 * c + 1), acc);
  return warp_sum(acc);
}

// Top-(k+1) by (value desc, index asc) over the lane-held values; lanes r < k receive the
// r-th (id, value), every lane the (k+1)-th value.
template <int VPL>
__device__ __forceinline__ void select_topk(const float (&v)[VPL], int E, int k, int lane,
                                            int& my_id, float& my_val, float& next_val) {
  uint32_t taken = 0;
  my_id = 0;
  my_val = 0.f;
  next_val = -FLT_MAX;
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
}

// Two warps per token (warp 2j: selection, warp 2j+1: shared gate and output row), so the
// two latency chains run side by side. Lane l holds logits of experts l, l+32, ...;
// VPL = values per lane, NS = partial-sum slices (a compile-time count, so that all
// VPL * NS loads of a lane are in flight together).
// `logits` holds `nslices` partial sums [nslices][T][E], added in slice order.
// With `wr` set (logits from the tensor-core router, whose accumulation is not exact fp32),
// a token whose k-th / (k+1)-th gap is below `band` has every expert whose logit lies within
// `band` of the k-th recomputed as an exact fp32 dot product, and the selection is redone on
// those values: the choice then matches fp32 arithmetic except at true near-ties.
template <int VPL, int NS>
__global__ void __launch_bounds__(256)
router_topk_kernel(const float* __restrict__ logits, const float* __restrict__ bias,
                   const uint16_t* __restrict__ x, const uint16_t* __restrict__ wsg,
                   const float* __restrict__ wr, float band, int T, int H, int E, int k,
                   int32_t* __restrict__ ids, float* __restrict__ w, float* __restrict__ sgate,
                   float* __restrict__ gap, float* __restrict__ out_zero) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 6) + (threadIdx.x >> 6);
  if (t >= T) return;

  if ((threadIdx.x >> 5) & 1) {
    // shared-expert gate: sigmoid(w_shared . x[t])
    float g = 0.f;
    const uint16_t* xr = x + (size_t)t * H;
#pragma unroll 4
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
    return;
  }

  // slices added in order, a group of SG slices in flight at a time (SG * VPL loads)
  constexpr int SG = NS < 4 ? NS : (VPL >= 32 ? 2 : 4);
  float v[VPL];
#pragma unroll
  for (int g = 0; g < NS; g += SG) {
    float part[SG][VPL];
#pragma unroll
    for (int sl = 0; sl < SG; ++sl)
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const int e = lane + 32 * i;
        part[sl][i] = e < E ? logits[((size_t)(g + sl) * T + t) * E + e] : 0.f;
      }
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      float l = g == 0 ? part[0][i] : v[i] + part[0][i];
#pragma unroll
      for (int sl = 1; sl < SG; ++sl) l += part[sl][i];
      v[i] = l;
    }
  }
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = lane + 32 * i;
    if (e < E) {
      if (bias) v[i] += bias[e];
    } else {
      v[i] = -FLT_MAX;
    }
  }

  int my_id;
  float my_val, next_val;
  select_topk<VPL>(v, E, k, lane, my_id, my_val, next_val);
  if (wr && k < E) {
    const float kth = __shfl_sync(0xffffffffu, my_val, k - 1);
    if (kth - next_val < band) {
      const uint16_t* xr = x + (size_t)t * H;
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const int e_l = lane + 32 * i;
        uint32_t m = __ballot_sync(0xffffffffu, e_l < E && fabsf(v[i] - kth) <= band);
        while (m) {
          const int src = __ffs(m) - 1;
          m &= m - 1;
          const int e = src + 32 * i;
          float l = exact_logit(xr, wr + (size_t)e * H, H, lane);
          if (bias) l += bias[e];
          if (lane == src) v[i] = l;
        }
      }
      select_topk<VPL>(v, E, k, lane, my_id, my_val, next_val);
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
}

}  // namespace

// Token count from which the tensor-core router (a GEMM over the exact three-piece split
// of the router matrix) replaces the CUDA-core one.
constexpr int kTcRouterMinTokens = 512;
// Half-width of the band of tensor-core logits that is recomputed exactly around the k-th:
// about 4.7x the largest deviation of those logits from fp32 dot products measured on B200
// (3.2e-4 at hidden 8192).
constexpr float kRefineBand = 1.5e-3f;

int router_slices(const moe_shape& s) { return s.T < kTcRouterMinTokens ? kSplits : 1; }

cudaError_t launch_router_logits(const moe_shape& s, const Layout& L, char* ws, const uint16_t* x,
                                 const float* wr, float* logits, cudaStream_t st) {
  const int nslices = router_slices(s);
  if (nslices == 1 && tc_router_supported(s)) return launch_tc_router(s, L, ws, x, wr, logits, st);
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(router_logits_small_kernel,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmallSmem);
  });
  if (attr_err != cudaSuccess) return attr_err;
  LaunchScope scope(MOE_K_ROUTER_LOGITS, st);
  dim3 grid((s.E + kSmallExp - 1) / kSmallExp, nslices, (s.T + kSmallTok - 1) / kSmallTok);
  router_logits_small_kernel<<<grid, kSmallThreads, kSmallSmem, st>>>(x, wr, logits, s.T, s.H,
                                                                      s.E, nslices);
  return cudaGetLastError();
}

cudaError_t launch_router_topk(const moe_shape& s, const float* logits, const float* wr,
                               const float* bias, const uint16_t* x, const uint16_t* wsg,
                               int32_t* ids, float* w,
                               float* sgate, float* gap, float* out_zero, cudaStream_t st) {
  LaunchScope scope(MOE_K_ROUTER_TOPK, st);
  const int nslices = router_slices(s);
  const bool tc_logits = nslices == 1 && tc_router_supported(s);
  // two warps per token; one token per CTA for small batches so that they spread over SMs
  const int tpb = s.T < kTcRouterMinTokens ? 1 : 4;
  const int warps = 2 * tpb;
  dim3 grid((s.T + tpb - 1) / tpb);
  const int vpl = (s.E + 31) / 32;
#define MOE_TOPK_CASE(N)                                                                     \
  do {                                                                                       \
    if (nslices == kSplits)                                                                  \
      router_topk_kernel<N, kSplits><<<grid, warps * 32, 0, st>>>(                             \
          logits, bias, x, wsg, nullptr, kRefineBand, s.T, s.H, s.E, s.k, ids, w, sgate, gap,  \
          out_zero);                                                                         \
    else                                                                                     \
      router_topk_kernel<N, 1><<<grid, warps * 32, 0, st>>>(                                   \
          logits, bias, x, wsg, tc_logits ? wr : nullptr, kRefineBand, s.T, s.H, s.E, s.k, ids, \
          w, sgate, gap, out_zero);                                                          \
  } while (0)
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
