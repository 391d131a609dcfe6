// compact.cu -- zero-channel compaction of structurally sparse routed experts, a weight
// pre-pass (not a step of the layer).
//
// The 2.4T checkpoint's tensor table (Qwen3.8-2.4T-A95B discussion #29) shows 71.0% of the
// rows of ffn_gate_exps and ffn_up_exps as exact zeros. Channel c of routed expert e is
// dead when its gate row W_gate,e[c,:] or its up row W_up,e[c,:] is all zero: then
// g_c = 0 (SiLU(0) = 0) or u_c = 0, so h_c = SiLU(g_c) * u_c = 0 exactly and column c of
// W_down,e contributes nothing to expert(x) = W_down (SiLU(W_gate x) * W_up x). Dropping
// the dead channels therefore leaves every expert's output unchanged (up to the order of
// fp32 additions), and removes their gate/up rows, down columns and FLOPs.
//
// Layout of the result: every expert keeps its live channels in their original order,
// packed to the front of a common width I_c (>= the largest live count), the rest zero:
//   gate_up_c [E][2 I_c][H]  rows 0..I_c-1 gate, I_c..2 I_c-1 up
//   down_c    [E][H][I_c]
// so the layer runs on the compacted bank with moe_shape.I = I_c and no other change.
// A zero row is one whose bf16 elements are all +0 or -0.
#include "device_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kMaskWarps = 8;

// live[e][c] = 1 if gate row c and up row I + c of expert e both hold a nonzero element.
// One warp per channel, 16-byte loads.
__global__ void __launch_bounds__(kMaskWarps * 32)
zero_channel_mask_kernel(const uint16_t* __restrict__ w_gate_up, int E, int I, int H,
                         uint8_t* __restrict__ live) {
  const int lane = threadIdx.x & 31;
  const long long ch = (long long)blockIdx.x * kMaskWarps + (threadIdx.x >> 5);
  if (ch >= (long long)E * I) return;
  const int e = (int)(ch / I), c = (int)(ch % I);
  const uint4* g = reinterpret_cast<const uint4*>(w_gate_up + ((size_t)e * 2 * I + c) * H);
  const uint4* u = reinterpret_cast<const uint4*>(w_gate_up + ((size_t)e * 2 * I + I + c) * H);
  uint32_t gor = 0, uor = 0;
  for (int i = lane; i < H / 8; i += 32) {
    const uint4 a = ld_stream_v4(g + i), b = ld_stream_v4(u + i);
    gor |= (a.x | a.y | a.z | a.w) & 0x7FFF7FFFu;  // ignore the sign bits: -0 is zero
    uor |= (b.x | b.y | b.z | b.w) & 0x7FFF7FFFu;
  }
  const bool gl = __any_sync(0xffffffffu, gor != 0);
  const bool ul = __any_sync(0xffffffffu, uor != 0);
  if (lane == 0) live[ch] = (gl && ul) ? 1 : 0;
}

// One block per expert: src[e][j] = the j-th live channel (j < count), -1 for j in
// [count, Ic); count[e] = number of live channels. A count above Ic is flagged.
__global__ void __launch_bounds__(kScanThreads)
zero_channel_scan_kernel(const uint8_t* __restrict__ live, int E, int I, int Ic,
                         int32_t* __restrict__ src, int32_t* __restrict__ count,
                         uint32_t* __restrict__ status) {
  __shared__ int warp_sums[kScanThreads / 32];
  __shared__ int base;
  const int e = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) base = 0;
  __syncthreads();
  for (int c0 = 0; c0 < I; c0 += kScanThreads) {
    const int c = c0 + threadIdx.x;
    const int v = (c < I) ? live[(size_t)e * I + c] : 0;
    const unsigned ballot = __ballot_sync(0xffffffffu, v);
    const int in_warp = __popc(ballot & ((1u << lane) - 1u));
    if (lane == 0) warp_sums[warp] = __popc(ballot);
    __syncthreads();
    if (warp == 0) {
      const int s = warp_sums[lane];
      int incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      warp_sums[lane] = incl - s;  // exclusive prefix of the warp totals
    }
    __syncthreads();
    const int j = base + warp_sums[warp] + in_warp;
    if (v) {
      if (j < Ic) src[(size_t)e * Ic + j] = c;
      else set_flag(status, kFlagBounds);
    }
    __syncthreads();
    if (threadIdx.x == kScanThreads - 1) base = j + v;
    __syncthreads();
  }
  for (int j = base + threadIdx.x; j < Ic; j += kScanThreads) src[(size_t)e * Ic + j] = -1;
  if (threadIdx.x == 0) count[e] = base;
}

// Rows of the compacted gate|up bank: row r < Ic copies gate row src[r], row Ic + r up row
// I + src[r]; padding rows are zero. One warp per row, 16-byte copies.
__global__ void __launch_bounds__(256)
compact_gate_up_kernel(const uint16_t* __restrict__ w_gate_up, const int32_t* __restrict__ src,
                       int E, int I, int H, int Ic, uint16_t* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (row >= (long long)E * 2 * Ic) return;
  const int e = (int)(row / (2 * Ic)), r = (int)(row % (2 * Ic));
  const int up = r >= Ic, j = up ? r - Ic : r;
  const int c = src[(size_t)e * Ic + j];
  uint4* dst = reinterpret_cast<uint4*>(out + (size_t)row * H);
  if (c < 0 || c >= I) {
    for (int i = lane; i < H / 8; i += 32) dst[i] = make_uint4(0, 0, 0, 0);
    return;
  }
  const uint4* s = reinterpret_cast<const uint4*>(
      w_gate_up + ((size_t)e * 2 * I + (up ? I : 0) + c) * H);
  for (int i = lane; i < H / 8; i += 32) dst[i] = ld_stream_v4(s + i);
}

// Rows of the compacted down bank: out[e][m][j] = W_down[e][m][src[j]] (0 for padding).
// A block holds its expert's channel map in shared memory and stages each source row there.
constexpr int kDownRowsPerBlock = 16;
__global__ void __launch_bounds__(256)
compact_down_kernel(const uint16_t* __restrict__ w_down, const int32_t* __restrict__ src,
                    int E, int I, int H, int Ic, uint16_t* __restrict__ out) {
  extern __shared__ uint8_t sm[];
  int32_t* map = reinterpret_cast<int32_t*>(sm);                 // [Ic]
  uint16_t* row = reinterpret_cast<uint16_t*>(sm + (size_t)Ic * 4);  // [I]
  const int blocks_per_e = (H + kDownRowsPerBlock - 1) / kDownRowsPerBlock;
  const int e = blockIdx.x / blocks_per_e;
  const int m0 = (blockIdx.x % blocks_per_e) * kDownRowsPerBlock;
  if (e >= E) return;
  for (int j = threadIdx.x; j < Ic; j += blockDim.x) map[j] = src[(size_t)e * Ic + j];
  for (int m = m0; m < m0 + kDownRowsPerBlock && m < H; ++m) {
    __syncthreads();  // the map is ready; the previous row is no longer read
    const uint4* s = reinterpret_cast<const uint4*>(w_down + ((size_t)e * H + m) * I);
    for (int i = threadIdx.x; i < I / 8; i += blockDim.x) reinterpret_cast<uint4*>(row)[i] = ld_stream_v4(s + i);
    __syncthreads();
    uint16_t* d = out + ((size_t)e * H + m) * Ic;
    for (int j = threadIdx.x; j < Ic; j += blockDim.x) {
      const int c = map[j];
      d[j] = (c >= 0 && c < I) ? row[c] : (uint16_t)0;
    }
  }
}

}  // namespace

size_t compact_workspace_bytes(const moe_shape& s) {
  const size_t E = (size_t)s.E, I = (size_t)s.I;
  return 256 + align_up(E * I, 256) + align_up(E * I * 4, 256) + align_up(E * 4, 256);
}

// Regions of the compaction workspace: status word, live mask, channel map, counts.
struct CompactLayout {
  size_t status, live, src, count;
};

static CompactLayout compact_layout(const moe_shape& s) {
  const size_t E = (size_t)s.E, I = (size_t)s.I;
  CompactLayout L;
  L.status = 0;
  L.live = 256;
  L.src = L.live + align_up(E * I, 256);
  L.count = L.src + align_up(E * I * 4, 256);
  return L;
}

cudaError_t launch_zero_channel_map(const moe_shape& s, const uint16_t* w_gate_up, int Ic,
                                    char* ws, int32_t** src, int32_t** count, cudaStream_t st) {
  const CompactLayout L = compact_layout(s);
  uint8_t* live = reinterpret_cast<uint8_t*>(ws + L.live);
  *src = reinterpret_cast<int32_t*>(ws + L.src);
  *count = reinterpret_cast<int32_t*>(ws + L.count);
  LaunchScope scope(MOE_K_OTHER, st, 2);
  const long long nch = (long long)s.E * s.I;
  zero_channel_mask_kernel<<<(unsigned)((nch + kMaskWarps - 1) / kMaskWarps), kMaskWarps * 32, 0,
                             st>>>(w_gate_up, s.E, s.I, s.H, live);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  zero_channel_scan_kernel<<<s.E, kScanThreads, 0, st>>>(
      live, s.E, s.I, Ic, *src, *count, reinterpret_cast<uint32_t*>(ws + L.status));
  return cudaGetLastError();
}

cudaError_t launch_compact_banks(const moe_shape& s, const uint16_t* w_gate_up,
                                 const uint16_t* w_down, const int32_t* src, int Ic,
                                 uint16_t* gate_up_c, uint16_t* down_c, cudaStream_t st) {
  LaunchScope scope(MOE_K_OTHER, st, 2);
  const long long rows = (long long)s.E * 2 * Ic;
  compact_gate_up_kernel<<<(unsigned)((rows * 32 + 255) / 256), 256, 0, st>>>(
      w_gate_up, src, s.E, s.I, s.H, Ic, gate_up_c);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = (size_t)Ic * 4 + (size_t)s.I * 2;
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(compact_down_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
  }
  const int blocks_per_e = (s.H + kDownRowsPerBlock - 1) / kDownRowsPerBlock;
  compact_down_kernel<<<(unsigned)s.E * blocks_per_e, 256, smem, st>>>(w_down, src, s.E, s.I, s.H,
                                                                       Ic, down_c);
  return cudaGetLastError();
}

}  // namespace moe
