// permute.cu -- stage 3 of the layer, "Dispatch R tokens" (Qwen3.8-Flash-Next
// architecture study, MoE pipeline diagram; R = kT token-expert assignments, section
// "Follow the kernels, one layer at a time").
//
// A stable counting sort of the T*k assignments by expert in three kernels:
//   dispatch_mask_kernel    one CTA per block of 256 tokens: a 256-bit token mask per
//                           expert (atomicOr in shared memory) and its popcount;
//   dispatch_scan_kernel    one CTA: per-expert totals, exclusive scan -> offsets, the
//                           first packed row of every (block, expert), and the grouped
//                           GEMM plan (active groups, tile prefixes);
//   dispatch_scatter_kernel the packed row of assignment (t, j) is the block's base for
//                           its expert plus the number of earlier tokens of the block in
//                           the same mask -- token-ascending inside each expert, and the
//                           same on every run.
// With T <= 256 (one token block, e.g. decode) dispatch_small_kernel does all three steps in
// one CTA with the masks in shared memory; the result is the same.
// An expert id outside [0, E) is skipped and raises the bounds flag in the status word.
#include <mutex>

#include "device_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

__global__ void __launch_bounds__(kPermBlock)
dispatch_mask_kernel(const int32_t* __restrict__ ids, int T, int E, int k,
                     uint32_t* __restrict__ blk_mask, int32_t* __restrict__ blk_count,
                     uint32_t* __restrict__ status) {
  extern __shared__ uint32_t mask[];  // [E][8]
  const int b = blockIdx.x;
  for (int i = threadIdx.x; i < E * 8; i += blockDim.x) mask[i] = 0;
  __syncthreads();
  const int i = threadIdx.x;
  const int t = b * kPermBlock + i;
  if (t < T) {
    for (int j = 0; j < k; ++j) {
      const int e = ids[(size_t)t * k + j];
      if (e < 0 || e >= E) {
        set_flag(status, kFlagBounds);
        continue;
      }
      atomicOr(&mask[e * 8 + (i >> 5)], 1u << (i & 31));
    }
  }
  __syncthreads();
  uint32_t* gm = blk_mask + (size_t)b * E * 8;
  for (int q = threadIdx.x; q < E * 8; q += blockDim.x) gm[q] = mask[q];
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int c = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) c += __popc(mask[e * 8 + w]);
    blk_count[(size_t)b * E + e] = c;
  }
}

// Group sizes n_g (g < E routed, g == E shared = T) -> plan. Called by all threads of a
// kScanThreads CTA; thread g handles group g (E + 1 <= 1025: thread 0 also takes E).
__device__ void build_plan(const int* n_of, int E, int H, int I, int Is, int T, int k,
                           PlanView pv) {
  // thread g takes group g (g <= E); with E == 1024 the last thread also takes group E
  const int g = threadIdx.x;
  int n0 = 0, n1 = 0, has1 = 0;
  if (g <= E && g < kScanThreads) n0 = n_of[g];
  if (g == kScanThreads - 1 && E == kScanThreads) { n1 = n_of[E]; has1 = 1; }
  const int a0 = (g <= E && g < kScanThreads && n0 > 0) ? 1 : 0;
  const int a1 = (has1 && n1 > 0) ? 1 : 0;

  auto inter = [&](int grp) { return grp < E ? I : Is; };
  const int uc = tc_gate_up_chunk(T, k, E);
  const int c0 = tc_nchunks(n0, uc), c1 = tc_nchunks(n1, uc);
  const int d0 = tc_nchunks(n0, kTcChunkDown), d1 = tc_nchunks(n1, kTcChunkDown);
  const int f0 = tc_nchunks(n0, kTcChunkDownF16), f1 = tc_nchunks(n1, kTcChunkDownF16);
  const int q0 = tc_nchunks(n0, kTcChunkGateUp8), q1 = tc_nchunks(n1, kTcChunkGateUp8);
  const int e0 = tc_nchunks(n0, kTcChunkDown8), e1 = tc_nchunks(n1, kTcChunkDown8);
  const int t1a = (g <= E) ? c0 * (inter(g) / 128) : 0;
  const int t1b = has1 ? c1 * (Is / 128) : 0;
  const int t2a = (g <= E) ? d0 * (H / 256) : 0;
  const int t2b = has1 ? d1 * (H / 256) : 0;
  const int t3a = (g <= E) ? f0 * (H / 256) : 0;
  const int t3b = has1 ? f1 * (H / 256) : 0;
  const int t4a = (g <= E) ? q0 * (inter(g) / 128) : 0;
  const int t4b = has1 ? q1 * (Is / 128) : 0;
  const int t5a = (g <= E) ? e0 * (H / 256) : 0;
  const int t5b = has1 ? e1 * (H / 256) : 0;
  const int r0a = (g <= E) ? n0 : 0, r0b = has1 ? n1 : 0;
  // the active groups, the five tile prefixes and the row prefix in one pass
  __shared__ int scan7[33 * 7];
  const int vals[7] = {a0 + a1,   t1a + t1b, t2a + t2b, t3a + t3b,
                       t4a + t4b, t5a + t5b, r0a + r0b};
  int pre[7], tot[7];
  block_exclusive_scan_n<7>(vals, pre, tot, scan7);
  const int pos = pre[0];
  if (a0) pv.active[pos] = g;
  if (a1) pv.active[pos + a0] = E;
  if (threadIdx.x == 0) *pv.n_active = tot[0];
  const int p1 = pre[1], p2 = pre[2], p3 = pre[3], p4 = pre[4], p5 = pre[5], pr = pre[6];
  const int tot1 = tot[1], tot2 = tot[2], tot3 = tot[3], tot4 = tot[4], tot5 = tot[5],
            totr = tot[6];
  if (g <= E) {
    pv.tp1[g] = p1;
    pv.tp2[g] = p2;
    pv.tp3[g] = p3;
    pv.tp4[g] = p4;
    pv.tp5[g] = p5;
    pv.row0[g] = pr;
  }
  if (has1) {
    pv.tp1[E] = p1 + t1a;
    pv.tp2[E] = p2 + t2a;
    pv.tp3[E] = p3 + t3a;
    pv.tp4[E] = p4 + t4a;
    pv.tp5[E] = p5 + t5a;
    pv.row0[E] = pr + r0a;
  }
  if (threadIdx.x == 0) {
    pv.tp1[E + 1] = tot1;
    pv.tp2[E + 1] = tot2;
    pv.tp3[E + 1] = tot3;
    pv.tp4[E + 1] = tot4;
    pv.tp5[E + 1] = tot5;
    pv.row0[E + 1] = totr;
  }
}

__global__ void __launch_bounds__(kScanThreads)
dispatch_scan_kernel(const int32_t* blk_count, int nblk, int T, int E, int k, int H,
                     int I, int Is, int32_t* blk_base, int32_t* __restrict__ offsets,
                     int* __restrict__ plan_base) {
  __shared__ int smem[33];
  __shared__ int n_of[kMaxE + 1];
  const int e = threadIdx.x;
  int total = 0;
  if (e < E) {
    for (int b = 0; b < nblk; ++b) {
      const int c = blk_count[(size_t)b * E + e];
      blk_base[(size_t)b * E + e] = total;
      total += c;
    }
  }
  int R;
  const int off = block_exclusive_scan(e < E ? total : 0, smem, &R);
  if (e < E) {
    offsets[e] = off;
    for (int b = 0; b < nblk; ++b) blk_base[(size_t)b * E + e] += off;
    n_of[e] = total;
  }
  if (threadIdx.x == 0) {
    offsets[E] = R;
    n_of[E] = T;
  }
  __syncthreads();
  build_plan(n_of, E, H, I, Is, T, k, plan_view(plan_base, E));
}

__global__ void __launch_bounds__(kPermBlock)
dispatch_scatter_kernel(const int32_t* __restrict__ ids, const float* __restrict__ topk_w, int T,
                        int E, int k, const uint32_t* __restrict__ blk_mask,
                        const int32_t* __restrict__ blk_base, int32_t* __restrict__ sorted_token,
                        float* __restrict__ sorted_w, int32_t* __restrict__ assign_row) {
  const int b = blockIdx.x;
  const int i = threadIdx.x;
  const int t = b * kPermBlock + i;
  if (t >= T) return;
  const uint32_t* gm = blk_mask + (size_t)b * E * 8;
  const int word = i >> 5;
  const uint32_t below = (1u << (i & 31)) - 1u;
  for (int j = 0; j < k; ++j) {
    const int e = ids[(size_t)t * k + j];
    if (e < 0 || e >= E) continue;
    const uint32_t* m = gm + e * 8;
    int rank = __popc(m[word] & below);
    for (int w = 0; w < word; ++w) rank += __popc(m[w]);
    const int p = blk_base[(size_t)b * E + e] + rank;
    sorted_token[p] = t;
    if (sorted_w) sorted_w[p] = topk_w[(size_t)t * k + j];
    assign_row[(size_t)t * k + j] = p;
  }
}

// The three steps above for T <= kPermBlock in one CTA of kScanThreads threads: thread
// i < T marks token i in the shared-memory masks, thread e < E counts and scans expert e
// (offsets, plan), then token i places its k assignments.
__global__ void __launch_bounds__(kScanThreads)
dispatch_small_kernel(const int32_t* __restrict__ ids, const float* __restrict__ topk_w, int T,
                      int E, int k, int H, int I, int Is, int32_t* __restrict__ offsets,
                      int* __restrict__ plan_base, int32_t* __restrict__ sorted_token,
                      float* __restrict__ sorted_w, int32_t* __restrict__ assign_row,
                      uint32_t* __restrict__ status) {
  extern __shared__ uint32_t mask[];  // [E][8]
  __shared__ int smem[33];
  __shared__ int n_of[kMaxE + 1];
  __shared__ int base[kMaxE];
  const int i = threadIdx.x;
  // token i's first kPre expert ids and routing weights, loaded before anything waits on
  // them (one round trip instead of one per assignment); later ones, if k > kPre, in the loops
  constexpr int kPre = 12;
  int my_ids[kPre];
  float my_w[kPre];
#pragma unroll
  for (int j = 0; j < kPre; ++j) {
    const bool have = i < T && j < k;
    my_ids[j] = have ? ids[(size_t)i * k + j] : -1;
    my_w[j] = (have && topk_w) ? topk_w[(size_t)i * k + j] : 0.f;
  }
  for (int q = threadIdx.x; q < E * 8; q += blockDim.x) mask[q] = 0;
  __syncthreads();
  if (i < T) {
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      if (j >= k) break;
      const int e = j < kPre ? my_ids[j] : ids[(size_t)i * k + j];
      if (e < 0 || e >= E) {
        set_flag(status, kFlagBounds);
        continue;
      }
      atomicOr(&mask[e * 8 + (i >> 5)], 1u << (i & 31));
    }
  }
  __syncthreads();
  const int e = threadIdx.x;
  int total = 0;
  if (e < E) {
#pragma unroll
    for (int w = 0; w < 8; ++w) total += __popc(mask[e * 8 + w]);
  }
  int R;
  const int off = block_exclusive_scan(e < E ? total : 0, smem, &R);
  if (e < E) {
    offsets[e] = off;
    base[e] = off;
    n_of[e] = total;
  }
  if (threadIdx.x == 0) {
    offsets[E] = R;
    n_of[E] = T;
  }
  __syncthreads();
  build_plan(n_of, E, H, I, Is, T, k, plan_view(plan_base, E));
  if (i < T) {
    const int word = i >> 5;
    const uint32_t below = (1u << (i & 31)) - 1u;
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      if (j >= k) break;
      const int ee = j < kPre ? my_ids[j] : ids[(size_t)i * k + j];
      if (ee < 0 || ee >= E) continue;
      const uint32_t* m = mask + ee * 8;
      int rank = __popc(m[word] & below);
      for (int w = 0; w < word; ++w) rank += __popc(m[w]);
      const int p = base[ee] + rank;
      sorted_token[p] = i;
      if (sorted_w) sorted_w[p] = j < kPre ? my_w[j] : topk_w[(size_t)i * k + j];
      assign_row[(size_t)i * k + j] = p;
    }
  }
}

// Plan from caller-supplied offsets. Offsets that are not a monotone partition of at most
// T*k rows starting at 0 are flagged and give an empty plan (no GEMM work).
__global__ void __launch_bounds__(kScanThreads)
plan_from_offsets_kernel(const int32_t* __restrict__ offsets, int T, int E, int k, int H, int I,
                         int Is, int shared_rows, int* __restrict__ plan_base,
                         uint32_t* __restrict__ status) {
  __shared__ int n_of[kMaxE + 1];
  __shared__ int bad;
  if (threadIdx.x == 0) bad = (offsets[0] != 0 || offsets[E] > T * k) ? 1 : 0;
  __syncthreads();
  for (int g = threadIdx.x; g < E; g += blockDim.x) {
    const int n = offsets[g + 1] - offsets[g];
    if (n < 0) bad = 1;
    n_of[g] = n;
  }
  if (threadIdx.x == 0) n_of[E] = shared_rows;
  __syncthreads();
  if (bad) {
    for (int g = threadIdx.x; g <= E; g += blockDim.x) n_of[g] = 0;
    if (threadIdx.x == 0) set_flag(status, kFlagBounds);
  }
  __syncthreads();
  build_plan(n_of, E, H, I, Is, T, k, plan_view(plan_base, E));
}

}  // namespace

cudaError_t launch_permute(const moe_shape& s, const Layout& L, char* ws, const int32_t* ids,
                           const float* topk_w, int32_t* offsets, int32_t* sorted_token,
                           float* sorted_w, int32_t* assign_row, cudaStream_t st) {
  uint32_t* status = reinterpret_cast<uint32_t*>(ws + L.status);
  uint32_t* blk_mask = reinterpret_cast<uint32_t*>(ws + L.blk_mask);
  int32_t* blk_base = reinterpret_cast<int32_t*>(ws + L.blk_base);
  const size_t smem = (size_t)s.E * 8 * sizeof(uint32_t);
  if (s.T <= kPermBlock) {
    LaunchScope scope(MOE_K_PERMUTE, st);
    dispatch_small_kernel<<<1, kScanThreads, smem, st>>>(
        ids, topk_w, s.T, s.E, s.k, s.H, s.I, s.Is, offsets, reinterpret_cast<int*>(ws + L.plan),
        sorted_token, sorted_w, assign_row, status);
    return cudaGetLastError();
  }
  LaunchScope scope(MOE_K_PERMUTE, st, 3);
  // counts go to blk_base first, the scan rewrites them in place as bases
  dispatch_mask_kernel<<<L.nblk, kPermBlock, smem, st>>>(ids, s.T, s.E, s.k, blk_mask, blk_base,
                                                        status);
  dispatch_scan_kernel<<<1, kScanThreads, 0, st>>>(blk_base, L.nblk, s.T, s.E, s.k, s.H, s.I, s.Is,
                                                   blk_base, offsets,
                                                   reinterpret_cast<int*>(ws + L.plan));
  dispatch_scatter_kernel<<<L.nblk, kPermBlock, 0, st>>>(ids, topk_w, s.T, s.E, s.k, blk_mask,
                                                         blk_base, sorted_token, sorted_w,
                                                         assign_row);
  return cudaGetLastError();
}

cudaError_t launch_plan_from_offsets(const moe_shape& s, const Layout& L, char* ws,
                                     const int32_t* offsets, int shared_rows, cudaStream_t st) {
  LaunchScope scope(MOE_K_PERMUTE, st);
  plan_from_offsets_kernel<<<1, kScanThreads, 0, st>>>(
      offsets, s.T, s.E, s.k, s.H, s.I, s.Is, shared_rows, reinterpret_cast<int*>(ws + L.plan),
      reinterpret_cast<uint32_t*>(ws + L.status));
  return cudaGetLastError();
}

// ---------------------------------------------------------------- no-allocation dispatch
//
// moe_permute_noalloc: the dispatch above for callers that cannot allocate device memory
// (no workspace argument). Its scratch -- status word, per-block token masks and bases,
// GEMM plan -- lives in one file-scope device array that every GPU loading this library
// holds until the process exits. In host code `g_noalloc_scratch` is only a host-side
// stand-in for the symbol; its device address is looked up with cudaGetSymbolAddress,
// once per device, with that device current (the first call on a device does it). The
// address is kept for the life of the process, so the entry point must not be used after a
// cudaDeviceReset (or any teardown of the device's primary context) in the same process.

namespace {

constexpr size_t kNoAllocScratchBytes = 640u * 1024u;
constexpr long long kNoAllocMaxBlockExperts = 16384;  // ceil(T/256) * E
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kNoAllocMaxDevices];

cudaError_t noalloc_scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return cudaSuccess;
}

struct NoAllocLayout {
  size_t status, blk_mask, blk_base, plan, total;
  int nblk;
};

NoAllocLayout noalloc_layout(const moe_shape& s) {
  NoAllocLayout L{};
  L.nblk = (s.T + kPermBlock - 1) / kPermBlock;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes, 256);
    return at;
  };
  L.status = take(256);
  L.blk_mask = take((size_t)L.nblk * s.E * 8 * sizeof(uint32_t));
  L.blk_base = take((size_t)L.nblk * s.E * sizeof(int32_t));
  L.plan = take(plan_ints(s.E) * sizeof(int32_t));
  L.total = o;
  return L;
}

}  // namespace

}  // namespace moe

extern "C" moe_status moe_permute_noalloc(const moe_shape* shape, const int32_t* topk_ids,
                                          int32_t* offsets, int32_t* sorted_token,
                                          int32_t* assign_row, void* stream) {
  using namespace moe;
  if (!shape) return MOE_ERR_INVALID_ARG;
  const moe_shape& s = *shape;
  if (s.T < 0 || s.E <= 0 || s.k <= 0 || s.H <= 0 || s.I <= 0 || s.Is <= 0)
    return MOE_ERR_INVALID_ARG;
  if (s.E > kMaxE || s.k > kMaxK || s.k > s.E || s.H % 64 || s.I % 64 || s.Is % 64)
    return MOE_ERR_UNSUPPORTED;
  auto a16 = [](const void* p) { return p && ((uintptr_t)p & 15u) == 0; };
  if (!a16(topk_ids) || !a16(offsets) || !a16(sorted_token) || !a16(assign_row))
    return MOE_ERR_INVALID_ARG;
  if (s.T == 0) return MOE_OK;
  const NoAllocLayout L = noalloc_layout(s);
  if ((long long)L.nblk * s.E > kNoAllocMaxBlockExperts || L.total > kNoAllocScratchBytes)
    return MOE_ERR_UNSUPPORTED;  // beyond the fixed scratch: use moe_permute with a workspace
  void* base = nullptr;
  if (noalloc_scratch_address(&base) != cudaSuccess) return MOE_ERR_CUDA;
  char* ws = static_cast<char*>(base);
  cudaStream_t st = (cudaStream_t)stream;
  // the array keeps the previous call's contents: clear the status word; the masks are
  // rebuilt in shared memory and the bases and plan are fully rewritten by every call
  if (cudaMemsetAsync(ws + L.status, 0, 256, st) != cudaSuccess) return MOE_ERR_CUDA;
  uint32_t* status = reinterpret_cast<uint32_t*>(ws + L.status);
  uint32_t* blk_mask = reinterpret_cast<uint32_t*>(ws + L.blk_mask);
  int32_t* blk_base = reinterpret_cast<int32_t*>(ws + L.blk_base);
  const size_t smem = (size_t)s.E * 8 * sizeof(uint32_t);
  LaunchScope scope(MOE_K_PERMUTE, st, 3);
  dispatch_mask_kernel<<<L.nblk, kPermBlock, smem, st>>>(topk_ids, s.T, s.E, s.k, blk_mask,
                                                        blk_base, status);
  dispatch_scan_kernel<<<1, kScanThreads, 0, st>>>(blk_base, L.nblk, s.T, s.E, s.k, s.H, s.I,
                                                   s.Is, blk_base, offsets,
                                                   reinterpret_cast<int*>(ws + L.plan));
  dispatch_scatter_kernel<<<L.nblk, kPermBlock, 0, st>>>(topk_ids, nullptr, s.T, s.E, s.k,
                                                         blk_mask, blk_base, sorted_token,
                                                         nullptr, assign_row);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
