// stream_swiglu.cu -- stage 4, "Grouped expert GEMMs", for decode-size batches: the
// expert formula expert(x) = W_down(SiLU(W_gate x) * W_up x) (Qwen3.8-Flash-Next
// architecture study, MoE section) evaluated by streaming each activated expert's weight
// rows once from HBM through CUDA-core FMAs.
//
// With a few tokens per expert (decode: 64 tokens x 10 / 512 experts ~ 1.25) the work is
// bound by reading the activated experts' weights, so each warp streams 8 weight rows
// with 16-byte loads (no L1 allocation) and applies them to up to 4 tokens held in
// registers; 32 partial sums are combined by one warp transpose-reduction.
//
//   stream_gate_up_kernel : h[p, c] = SiLU(gate_c . x_p) * (up_c . x_p), kept as the bf16
//                           pair hi = bf16(h), lo = bf16(h - hi) (about 16 significant bits)
//   stream_down_kernel    : y[p, m] = W_down[m, :] . (hi + lo)[p, :]; stored per packed row, or
//                           scaled by the routing weight (shared gate for the shared
//                           expert) and added into out[token, m] ("Weighted combine").
#include "device_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kWarps = 8;
constexpr int kTok = 4;       // tokens per warp pass
constexpr int kChPerWarp = 4; // gate|up: 4 channels = 8 weight rows
constexpr int kRowsDown = 8;  // down: 8 output rows

// Token of packed row p: routed rows [0, R) via sorted_token, shared rows R.. in order.
// A routed token outside [0, T) (caller-supplied dispatch) is replaced by 0 and flagged.
__device__ __forceinline__ int token_of(const int32_t* sorted_token, int p, int R, int T,
                                        uint32_t* status) {
  if (p >= R) return p - R;
  const int t = sorted_token[p];
  if ((unsigned)t >= (unsigned)T) {
    set_flag(status, kFlagBounds);
    return 0;
  }
  return t;
}

// grid: (Imax / 32, E + 1); blockIdx.y indexes the active-group list.
__global__ void __launch_bounds__(kWarps * 32)
stream_gate_up_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ sorted_token,
                      const int* __restrict__ plan_base, const uint16_t* __restrict__ w_gate_up,
                      const uint16_t* __restrict__ ws_gate_up, uint16_t* __restrict__ h,
                      size_t h_plane, int T, int H, int E, int I, int Is, int ldh,
                      uint32_t* __restrict__ status) {
  const PlanView pv = plan_view(const_cast<int*>(plan_base), E);
  const int gi = blockIdx.y;
  if (gi >= *pv.n_active) return;
  const int g = pv.active[gi];
  const int Ig = g < E ? I : Is;
  const uint16_t* W = g < E ? w_gate_up + (size_t)g * 2 * I * H : ws_gate_up;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c0 = (blockIdx.x * kWarps + warp) * kChPerWarp;
  if (c0 >= Ig) return;
  const int row0 = pv.row0[g];
  const int n = pv.row0[g + 1] - row0;
  const int R = pv.row0[E];  // routed rows actually dispatched

  const uint16_t* wrow[8];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    wrow[r] = W + (size_t)(c0 + r) * H;           // gate rows
    wrow[4 + r] = W + (size_t)(Ig + c0 + r) * H;  // up rows
  }
  const int nchunk = H / 8;

  for (int s = 0; s < n; s += kTok) {
    const uint16_t* xrow[kTok];
#pragma unroll
    for (int q = 0; q < kTok; ++q) {
      const int p = row0 + s + (s + q < n ? q : 0);
      xrow[q] = x + (size_t)token_of(sorted_token, p, R, T, status) * H;
    }
    float acc[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] = 0.f;
    for (int c = lane; c < nchunk; c += 32) {
      uint4 wv[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) wv[r] = ld_stream_v4(wrow[r] + 8 * c);
#pragma unroll
      for (int q = 0; q < kTok; ++q) {
        float xf[8];
        unpack8(ld_v4(xrow[q] + 8 * c), xf);
#pragma unroll
        for (int r = 0; r < 8; ++r) acc[r * 4 + q] = dot8_acc(wv[r], xf, acc[r * 4 + q]);
      }
    }
    // lane l: weight row l/4 (0..3 gate, 4..7 up of the same channels), token l%4
    const float v = warp_transpose_sum32(acc, lane);
    const float up = __shfl_down_sync(0xffffffffu, v, 16);
    const int q = lane & 3;
    if (lane < 16 && s + q < n) {
      const float gate = v;
      const float hv = gate / (1.f + expf(-gate)) * up;
      const uint16_t hi = f32_to_bf16_rn(hv);
      const size_t at = (size_t)(row0 + s + q) * ldh + c0 + (lane >> 2);
      h[at] = hi;
      h[h_plane + at] = f32_to_bf16_rn(hv - bf16lo(hi));
    }
  }
}

// grid: (H / 64, E + 1)
__global__ void __launch_bounds__(kWarps * 32)
stream_down_kernel(const uint16_t* __restrict__ h, size_t h_plane,
                   const int32_t* __restrict__ sorted_token,
                   const float* __restrict__ sorted_w, const float* __restrict__ sgate,
                   const int* __restrict__ plan_base, const uint16_t* __restrict__ w_down,
                   const uint16_t* __restrict__ ws_down, float* __restrict__ y,
                   float* __restrict__ y_shared, float* __restrict__ out, int T, int H, int E,
                   int I, int Is, int ldh, uint32_t* __restrict__ status) {
  const PlanView pv = plan_view(const_cast<int*>(plan_base), E);
  const int gi = blockIdx.y;
  if (gi >= *pv.n_active) return;
  const int g = pv.active[gi];
  const int Ig = g < E ? I : Is;
  const uint16_t* W = g < E ? w_down + (size_t)g * H * I : ws_down;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int m0 = (blockIdx.x * kWarps + warp) * kRowsDown;
  if (m0 >= H) return;
  const int row0 = pv.row0[g];
  const int n = pv.row0[g + 1] - row0;
  const int R = pv.row0[E];
  const int nchunk = Ig / 8;

  for (int s = 0; s < n; s += kTok) {
    const uint16_t* hrow[kTok];
#pragma unroll
    for (int q = 0; q < kTok; ++q) hrow[q] = h + (size_t)(row0 + s + (s + q < n ? q : 0)) * ldh;
    float acc[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] = 0.f;
    for (int c = lane; c < nchunk; c += 32) {
      uint4 wv[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) wv[r] = ld_stream_v4(W + (size_t)(m0 + r) * Ig + 8 * c);
#pragma unroll
      for (int q = 0; q < kTok; ++q) {
        float hf[8], lf[8];
        unpack8(ld_v4(hrow[q] + 8 * c), hf);
        unpack8(ld_v4(hrow[q] + h_plane + 8 * c), lf);
#pragma unroll
        for (int i = 0; i < 8; ++i) hf[i] += lf[i];
#pragma unroll
        for (int r = 0; r < 8; ++r) acc[r * 4 + q] = dot8_acc(wv[r], hf, acc[r * 4 + q]);
      }
    }
    const float v = warp_transpose_sum32(acc, lane);
    const int q = lane & 3;
    const int m = m0 + (lane >> 2);
    if (s + q < n) {
      const int p = row0 + s + q;
      if (out) {
        const int t = token_of(sorted_token, p, R, T, status);
        const float wgt = p < R ? sorted_w[p] : sgate[t];
        atomicAdd(out + (size_t)t * H + m, wgt * v);
      } else if (p < R) {
        y[(size_t)p * H + m] = v;
      } else {
        y_shared[(size_t)(p - R) * H + m] = v;
      }
    }
  }
}

}  // namespace

cudaError_t launch_stream_gate_up(const moe_shape& s, const Layout& L, char* ws, const uint16_t* x,
                                  const int32_t* sorted_token, const moe_weights& w,
                                  cudaStream_t st) {
  LaunchScope scope(MOE_K_GATE_UP, st);
  const int imax = s.I > s.Is ? s.I : s.Is;
  dim3 grid((imax + kWarps * kChPerWarp - 1) / (kWarps * kChPerWarp), s.E + 1);
  stream_gate_up_kernel<<<grid, kWarps * 32, 0, st>>>(
      x, sorted_token, reinterpret_cast<const int*>(ws + L.plan),
      static_cast<const uint16_t*>(w.w_gate_up), static_cast<const uint16_t*>(w.ws_gate_up),
      reinterpret_cast<uint16_t*>(ws + L.h), L.h_plane, s.T, s.H, s.E, s.I, s.Is, L.ldh,
      reinterpret_cast<uint32_t*>(ws + L.status));
  return cudaGetLastError();
}

cudaError_t launch_stream_down(const moe_shape& s, const Layout& L, char* ws,
                               const int32_t* sorted_token, const float* sorted_w,
                               const float* sgate, const moe_weights& w, float* y,
                               float* y_shared, float* out, cudaStream_t st) {
  LaunchScope scope(MOE_K_DOWN, st);
  dim3 grid((s.H + kWarps * kRowsDown - 1) / (kWarps * kRowsDown), s.E + 1);
  stream_down_kernel<<<grid, kWarps * 32, 0, st>>>(
      reinterpret_cast<const uint16_t*>(ws + L.h), L.h_plane, sorted_token, sorted_w, sgate,
      reinterpret_cast<const int*>(ws + L.plan), static_cast<const uint16_t*>(w.w_down),
      static_cast<const uint16_t*>(w.ws_down), y, y_shared, out, s.T, s.H, s.E, s.I, s.Is, L.ldh,
      reinterpret_cast<uint32_t*>(ws + L.status));
  return cudaGetLastError();
}

}  // namespace moe
