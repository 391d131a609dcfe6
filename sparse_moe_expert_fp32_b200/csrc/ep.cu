// ep.cu -- the row movement of expert parallelism (Qwen3.8-Flash-Next architecture study,
// section "Expert parallelism": the routed experts are split across GPUs, and dispatch and
// combine exchange token activations between the ranks that hold a token and the ranks
// that own its experts).
//
// With the experts split into G contiguous slices of E/G, the dispatch order of
// moe_permute (packed rows grouped by expert, experts ascending) is already grouped by
// owner rank: rank d's rows are packed rows [offsets[d E/G], offsets[(d+1) E/G]). So:
//   ep_counts_kernel      per owner rank and local expert, the row counts to send;
//   gather_rows_kernel    the send buffer: token rows in packed order, xs[p] = x[index[p]];
//   ep_regroup_kernel     on the owner, after the exchange: the received rows arrive
//                         grouped by source rank, then by expert; this builds the
//                         expert-major order the grouped GEMMs take (offsets per local
//                         expert, and for each expert-major row the received row it is);
//   scatter_rows_kernel   the return trip: each expert output row goes back to the position
//                         its token row had in the received buffer, so after the reverse
//                         exchange the source rank holds y in its own packed order.
// Indices outside their range are skipped and raise the bounds flag.
#include <algorithm>

#include "device_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

// out[p] = x[index[p]] for p < rows (rows of H bf16); one warp per row, 16-byte copies.
__global__ void __launch_bounds__(256)
gather_rows_bf16_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ index,
                        int64_t rows, int64_t n_src, int H, uint16_t* __restrict__ out,
                        uint32_t* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int vec = H / 8;
  for (int64_t p = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); p < rows; p += warps) {
    const int32_t src = index[p];
    if (src < 0 || src >= n_src) {
      if (lane == 0) set_flag(status, kFlagBounds);
      continue;
    }
    const uint4* a = reinterpret_cast<const uint4*>(x + (size_t)src * H);
    uint4* b = reinterpret_cast<uint4*>(out + (size_t)p * H);
    for (int c = lane; c < vec; c += 32) b[c] = __ldg(a + c);
  }
}

// out[index[p]] = y[p] for p < rows (rows of H fp32); one warp per row.
__global__ void __launch_bounds__(256)
scatter_rows_f32_kernel(const float* __restrict__ y, const int32_t* __restrict__ index,
                        int64_t rows, int64_t n_dst, int H, float* __restrict__ out,
                        uint32_t* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int vec = H / 4;
  for (int64_t p = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); p < rows; p += warps) {
    const int32_t dst = index[p];
    if (dst < 0 || dst >= n_dst) {
      if (lane == 0) set_flag(status, kFlagBounds);
      continue;
    }
    const float4* a = reinterpret_cast<const float4*>(y + (size_t)p * H);
    float4* b = reinterpret_cast<float4*>(out + (size_t)dst * H);
    for (int c = lane; c < vec; c += 32) b[c] = __ldg(a + c);
  }
}

// On the rank holding the tokens: counts[d][e] = rows of owner d's local expert e
// (packed rows of expert d El + e), rows[d] = all of owner d's rows, from moe_permute's
// offsets. One CTA of kScanThreads.
__global__ void __launch_bounds__(kScanThreads)
ep_counts_kernel(const int32_t* __restrict__ offsets, int G, int El, int32_t* __restrict__ counts,
                 int32_t* __restrict__ rows) {
  const int i = threadIdx.x;
  if (i < G * El) counts[i] = offsets[i + 1] - offsets[i];
  if (i < G) rows[i] = offsets[(i + 1) * El] - offsets[i * El];
}

// counts[s][e] = rows source rank s sent for local expert e (G x El <= kMaxE, one CTA of
// kScanThreads). The received buffer holds, source by source, each source's rows for
// expert 0, then expert 1, ...: segment (s, e) starts at seg(s, e), the exclusive prefix
// over the source-major order. The expert-major order puts, expert by expert, each
// source's segment in source order: it starts at dst(e, s), the exclusive prefix over the
// expert-major order. offsets[e] = dst(e, 0); src_index[dst(e, s) + i] = seg(s, e) + i.
__global__ void __launch_bounds__(kScanThreads)
ep_regroup_kernel(const int32_t* __restrict__ counts, int G, int El, int64_t capacity,
                  int32_t* __restrict__ offsets, int32_t* __restrict__ src_index,
                  int32_t* __restrict__ src_rows, uint32_t* __restrict__ status) {
  __shared__ int smem[33];
  __shared__ int cnt[kMaxE];
  __shared__ int seg[kMaxE];
  __shared__ int dst[kMaxE];
  const int n = G * El;
  const int i = threadIdx.x;
  if (i < n) {
    int c = counts[i];
    if (c < 0) {
      set_flag(status, kFlagBounds);
      c = 0;
    }
    cnt[i] = c;
  }
  __syncthreads();
  int total;
  const int a = block_exclusive_scan(i < n ? cnt[i] : 0, smem, &total);  // source-major
  if (i < n) seg[i] = a;
  // thread j = e * G + s carries segment (s, e) in expert-major order
  const int e = i / G, s = i - (i / G) * G;
  const int b = block_exclusive_scan(i < n ? cnt[s * El + e] : 0, smem, &total);
  if (i < n) dst[i] = b;
  __syncthreads();
  if (i < El) offsets[i] = dst[i * G];
  if (src_rows && i < G) {  // rows received from source i
    const int end = (i + 1 < G) ? seg[(i + 1) * El] : total;
    src_rows[i] = end - seg[i * El];
  }
  if (i == 0) {
    offsets[El] = (int64_t)total < capacity ? total : (int)capacity;
    if ((int64_t)total > capacity) set_flag(status, kFlagBounds);
  }
  // fill: warp w takes segments w, w + 32, ... (expert-major order), lanes take rows
  const int lane = i & 31, warp = i >> 5;
  for (int j = warp; j < n; j += kScanThreads / 32) {
    const int ee = j / G, ss = j - (j / G) * G;
    const int c = cnt[ss * El + ee];
    const int from = seg[ss * El + ee], to = dst[j];
    for (int r = lane; r < c; r += 32)
      if ((int64_t)to + r < capacity) src_index[to + r] = from + r;
  }
}

}  // namespace

cudaError_t launch_gather_rows_bf16(const uint16_t* x, const int32_t* index, int64_t rows,
                                    int64_t n_src, int H, uint16_t* out, uint32_t* status,
                                    int sms, cudaStream_t st) {
  LaunchScope scope(MOE_K_OTHER, st);
  const int64_t blocks = std::min<int64_t>((rows + 7) / 8, (int64_t)sms * 16);
  gather_rows_bf16_kernel<<<(unsigned)std::max<int64_t>(blocks, 1), 256, 0, st>>>(
      x, index, rows, n_src, H, out, status);
  return cudaGetLastError();
}

cudaError_t launch_scatter_rows_f32(const float* y, const int32_t* index, int64_t rows,
                                    int64_t n_dst, int H, float* out, uint32_t* status, int sms,
                                    cudaStream_t st) {
  LaunchScope scope(MOE_K_OTHER, st);
  const int64_t blocks = std::min<int64_t>((rows + 7) / 8, (int64_t)sms * 16);
  scatter_rows_f32_kernel<<<(unsigned)std::max<int64_t>(blocks, 1), 256, 0, st>>>(
      y, index, rows, n_dst, H, out, status);
  return cudaGetLastError();
}

cudaError_t launch_ep_regroup(const int32_t* counts, int G, int El, int64_t capacity,
                              int32_t* offsets, int32_t* src_index, int32_t* src_rows,
                              uint32_t* status, cudaStream_t st) {
  LaunchScope scope(MOE_K_PERMUTE, st);
  ep_regroup_kernel<<<1, kScanThreads, 0, st>>>(counts, G, El, capacity, offsets, src_index,
                                                src_rows, status);
  return cudaGetLastError();
}

cudaError_t launch_ep_counts(const int32_t* offsets, int G, int El, int32_t* counts,
                             int32_t* rows, cudaStream_t st) {
  LaunchScope scope(MOE_K_PERMUTE, st);
  ep_counts_kernel<<<1, kScanThreads, 0, st>>>(offsets, G, El, counts, rows);
  return cudaGetLastError();
}

}  // namespace moe
