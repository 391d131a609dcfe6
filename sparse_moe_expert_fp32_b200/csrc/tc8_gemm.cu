// tc8_gemm.cu -- stage 4, "Grouped expert GEMMs" (Qwen3.8-Flash-Next architecture study,
// MoE pipeline diagram), with the routed experts' weights stored in FP8 ("Qwen3.8, weights
// in hand: 98% of a 2.4T model is routed experts", section "What FP8 actually quantizes":
// routed experts in FP8, the shared expert in bf16). Each weight row carries an fp32 scale
// that multiplies its accumulator row in the epilogue, so the layer sees
// decode(code) * scale. What changes against the bf16 layer is the bytes: one per routed
// weight instead of two. Both GEMMs feed the codes as loaded (TMA, 128-byte swizzle, 128
// codes per row and stage) to tcgen05.mma kind::f8f6f4, so shared memory carries each code
// once (TMA write, MMA read), as in the bf16 kernels. The token operand goes in as E4M3
// pieces with a power-of-two scale per row (exact arithmetic, described above each kernel):
// x as two pieces (a bf16 value has 8 significant bits), h as four (it carries 16). One CTA
// per tile, swap AB (2 x 128 weight rows on the MMA's M side, tokens on N). The shared
// expert's tiles (bf16 weights) run kind::f16 MMAs on 64-wide K stages of the same 128-byte
// rows, in the same ring, and are handed out first, being the longest tiles. Tiles take at
// most 64 token rows (gate|up) or 32 (down) at every batch size (plan prefixes tp4, tp5).
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <algorithm>

#include "tc_common.cuh"
#include "tc_gemm.h"

namespace moe {
namespace {

constexpr int kQueue8 = 4;
constexpr uint32_t kTmemCols8 = 512;
constexpr uint32_t kSlotCols8 = 256;
constexpr int kBoxHeights8 = 4;  // token boxes of 128, 64, 32, 16 rows

struct TokenMaps8 {
  CUtensorMap m[kBoxHeights8];
};

// Piece j of an N-row token tile (N a multiple of 16): 128-row boxes, then one box for each
// binary digit of the remainder. False past the last piece.
__device__ __forceinline__ bool token_piece8(int N, int j, int& row, int& hidx) {
  const int n128 = N >> 7;
  if (j < n128) {
    row = j * 128;
    hidx = 0;
    return true;
  }
  j -= n128;
  int r = n128 * 128;
#pragma unroll
  for (int h = 1; h < kBoxHeights8; ++h) {
    const int rows = 128 >> h;
    if (N & rows) {
      if (j == 0) {
        row = r;
        hidx = h;
        return true;
      }
      --j;
      r += rows;
    }
  }
  return false;
}

// The two 256-column TMEM slots, handed to tiles in turn (a tile needing more than 128
// columns per accumulator takes both).
struct Slots8 {
  int next = 0;
  uint32_t uses[2] = {0u, 0u};
  __device__ __forceinline__ void take(int cols, int& first, int& count) const {
    count = cols > 128 ? 2 : 1;
    first = count == 2 ? 0 : next;
  }
  __device__ __forceinline__ void done(int first, int count) {
    for (int i = 0; i < count; ++i) uses[(first + i) & 1]++;
    next = count == 2 ? 0 : (first ^ 1);
  }
};

// ================================================================ gate|up on FP8 tensor cores
// The gate|up GEMM reads its weights as E4M3 codes straight into the MMA
// (tcgen05.mma kind::f8f6f4): no widening pass, so shared memory carries each code once
// (TMA write, MMA read) as in the bf16 kernels. The token rows go in as E4M3 too, each
// row split into two pieces with a power-of-two row scale 2^k (the row's largest
// magnitude times 2^k in [128, 256)):
//   hi = E4M3(x 2^k),  lo = E4M3(x 2^k - hi),  x 2^k = hi + lo
// exactly for every element within 2^9 of the row's largest magnitude (a bf16 value has 8
// significant bits, hi keeps 4, the rest fits lo); smaller elements keep an absolute error
// below 2^-(10+k), i.e. about 2^-17 of the row's largest magnitude. The hi rows and the lo
// rows of a tile follow each other in shared memory, so one MMA of N = 2 x rows gives
// W hi in columns [0, N) and W lo in [N, 2N); the epilogue adds them and multiplies by the
// weight row's scale and the token row's 2^-k. K = 128 codes per stage (128-byte rows).
// The shared expert's tiles (bf16 weights, bf16 x) run kind::f16 MMAs on 64-wide K stages
// of the same 128-byte rows, in the same ring. Roles as in the bf16 one-CTA kernel: warp 0
// TMA producer, warp 1 TMEM owner and MMA issuer, warps 2-9 epilogue.

constexpr int kEpiWarpsQ = 8;
constexpr int kThreadsQ = 64 + 32 * kEpiWarpsQ;
constexpr int kMaxTileQ = kTcChunkGateUp8;                  // 64 token rows per tile
constexpr uint32_t kABytesQ = 2 * 128 * 128;                // 2 x 128 weight rows x 128 B
constexpr uint32_t kBBytesQ = 2 * kMaxTileQ * 128;          // hi and lo token rows x 128 B
constexpr uint32_t kStageQ = kABytesQ + kBBytesQ;
constexpr int kStagesQ = 4;

struct SharedQ {
  uint64_t full[kStagesQ];
  uint64_t empty[kStagesQ];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t q_full[kQueue8];
  uint64_t q_empty[kQueue8];
  uint64_t drain;
  uint32_t tmem_base;
  volatile int abort;
  int q[kQueue8];
  int tp[kMaxE + 2];
  int row0[kMaxE + 2];
};

constexpr size_t smemq_bytes() { return 1024 + (size_t)kStagesQ * kStageQ + sizeof(SharedQ); }
static_assert(smemq_bytes() <= 232448, "over the 227 KB of shared memory a CTA may use");

struct GateUpQArgs {
  TcArgs a;
  const float* scale;    // fp32 [E][2I] weight row scales
  const float* x_scale;  // fp32 [R] 2^-k of each packed token row
};

// Instruction descriptor of kind::f8f6f4: fp32 accumulator, E4M3 A and B, both K-major.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
  return (1u << 4) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// four kind::f8f6f4 MMAs over one 128-wide K stage (32 codes = 32 bytes each)
__device__ __forceinline__ void umma_e4m3_x4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                             uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n"
      " .reg .pred p;\n"
      " .reg .b64 a1, a2, a3, b1, b2, b3;\n"
      " setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n"
      " add.s64 a1, %1, 2;\n add.s64 b1, %2, 2;\n"
      " tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a1, b1, %3, 1;\n"
      " add.s64 a2, %1, 4;\n add.s64 b2, %2, 4;\n"
      " tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a2, b2, %3, 1;\n"
      " add.s64 a3, %1, 6;\n add.s64 b3, %2, 6;\n"
      " tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a3, b3, %3, 1;\n"
      "}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
      : "memory");
}

struct GeomQ {
  Tile t;
  int a_row0, a_row1, b_row0, nk;
  bool shared;
};

// Tile order: the shared expert's tiles first (twice the stages of a routed tile), then the
// routed groups in order.
__device__ __forceinline__ GeomQ geomq(const TcArgs& a, const SharedQ& S, int tile, int total,
                                       int R) {
  const int tpE = S.tp[a.E];
  const int nsh = total - tpE;
  const int t2 = tile < nsh ? tpE + tile : tile - nsh;
  GeomQ G;
  G.t = decode_tile(S.row0, S.tp, a.E, t2, kMaxTileQ);
  G.shared = G.t.g == a.E;
  const int Ig = G.shared ? a.Is : a.I;
  const int base = G.shared ? 0 : G.t.g * 2 * a.I;
  G.a_row0 = base + G.t.m * 128;
  G.a_row1 = base + Ig + G.t.m * 128;
  G.b_row0 = G.shared ? G.t.p0 - R : G.t.p0;
  G.nk = G.shared ? a.H / 64 : a.H / 128;
  return G;
}

__global__ void __launch_bounds__(kThreadsQ, 1)
tc8_gate_up_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_a_sh,
                   const __grid_constant__ TokenMaps8 tm_x8, const __grid_constant__ TokenMaps8 tm_x_sh,
                   const GateUpQArgs aq) {
  const TcArgs& args = aq.a;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  SharedQ& S = *reinterpret_cast<SharedQ*>(smem + kStagesQ * kStageQ);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = args.E;
  const PlanView pv = plan_view(const_cast<int*>(args.plan), E);
  for (int g = threadIdx.x; g < E + 2; g += blockDim.x) {
    S.tp[g] = pv.tp4[g];
    S.row0[g] = pv.row0[g];
  }
  const int total = pv.tp4[E + 1];
  const int R = pv.row0[E];

  if (blockIdx.x == 0 && threadIdx.x == 0) *args.counter_next = 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesQ; ++s) {
      ptx::mbar_init(&S.full[s], 1);
      ptx::mbar_init(&S.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&S.tmem_full[b], 1);
      ptx::mbar_init(&S.tmem_empty[b], 32 * kEpiWarpsQ);
    }
    for (int i = 0; i < kQueue8; ++i) {
      ptx::mbar_init(&S.q_full[i], 1);
      ptx::mbar_init(&S.q_empty[i], 1 + kEpiWarpsQ);
    }
    ptx::mbar_init(&S.drain, 1);
    S.abort = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tm_q);
    ptx::prefetch_tmap(&tm_a_sh);
    for (int i = 0; i < kBoxHeights8; ++i) {
      ptx::prefetch_tmap(&tm_x8.m[i]);
      ptx::prefetch_tmap(&tm_x_sh.m[i]);
    }
  }
  if (warp == 1) {
    ptx::tmem_alloc(&S.tmem_base, kTmemCols8);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = S.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    int it = 0;
    int armed[kStagesQ];
#pragma unroll
    for (int s = 0; s < kStagesQ; ++s) armed[s] = -1;
    bool aborted = false;
    int ahead = (lane == 0) ? atomicAdd(args.counter, 1) : 0;
    for (int qi = 0; !aborted; ++qi) {
      const int slot = qi % kQueue8;
      int tile = 0;
      if (lane == 0) {
        if (!wait_phase(&S.q_empty[slot], ((uint32_t)(qi / kQueue8) & 1u) ^ 1u, S, args.status)) {
          tile = -2;
        } else {
          tile = ahead;
          if (tile >= total) tile = -1;
          else ahead = atomicAdd(args.counter, 1);
          S.q[slot] = tile;
          ptx::mbar_arrive(&S.q_full[slot]);
        }
      }
      tile = __shfl_sync(0xffffffffu, tile, 0);
      if (tile == -2) aborted = true;
      if (tile < 0) break;
      const GeomQ G = geomq(args, S, tile, total, R);
      const int planes = G.shared ? 1 : 2;  // routed: hi and lo rows of x
      const int kstep = G.shared ? 64 : 128;  // elements per 128-byte row
      const CUtensorMap* my_map = nullptr;
      uint32_t my_off = 0;
      int my_row = 0;
      if (lane < 2) {
        my_map = G.shared ? &tm_a_sh : &tm_q;
        my_off = lane * (kABytesQ / 2);
        my_row = lane ? G.a_row1 : G.a_row0;
      } else {
        int np = 0, r, h;
        while (token_piece8(G.t.N, np, r, h)) ++np;
        const int j = lane - 2;
        if (j < np * planes) {
          const int plane = j / np;
          token_piece8(G.t.N, j - plane * np, r, h);
          my_map = G.shared ? &tm_x_sh.m[h] : &tm_x8.m[h];
          my_off = kABytesQ + (uint32_t)(plane * G.t.N + r) * 128u;
          my_row = G.b_row0 + r + plane * R;
        }
      }
      const uint32_t bytes = kABytesQ + (uint32_t)planes * G.t.N * 128u;
      for (int ks = 0; ks < G.nk; ++ks, ++it) {
        const int s = it % kStagesQ;
        const uint32_t ph = (uint32_t)(it / kStagesQ) & 1u;
        bool ok = true;
        if (lane == 0) {
          ok = wait_phase(&S.empty[s], ph ^ 1u, S, args.status);
          if (ok) {
            ptx::mbar_arrive_expect_tx(&S.full[s], bytes);
            armed[s] = (int)ph;
          }
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) {
          aborted = true;
          break;
        }
        if (my_map)
          ptx::tma_load_2d(smem + s * kStageQ + my_off, my_map, &S.full[s], ks * kstep, my_row);
      }
    }
    if (aborted && lane == 0) {
      for (int s = 0; s < kStagesQ; ++s)
        if (armed[s] >= 0) drain_phase(&S.full[s], (uint32_t)armed[s]);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      Slots8 sl;
      bool aborted = false;
      const uint64_t desc0 = ptx::smem_desc_kmajor<128>(smem);
      for (int qi = 0; !aborted; ++qi) {
        const int slot = qi % kQueue8;
        if (!wait_phase(&S.q_full[slot], (uint32_t)(qi / kQueue8) & 1u, S, args.status)) {
          aborted = true;
          break;
        }
        const int tile = S.q[slot];
        ptx::mbar_arrive(&S.q_empty[slot]);
        if (tile < 0) break;
        const GeomQ G = geomq(args, S, tile, total, R);
        // routed: columns [0, N) W hi, [N, 2N) W lo; N <= 64, so one 256-column slot holds
        // both accumulators (the second at +128)
        const uint32_t idesc =
            G.shared ? ptx::idesc_bf16_f32(128, G.t.N) : idesc_e4m3_f32(128, 2 * G.t.N);
        int first, count;
        sl.take(128, first, count);
        if (!wait_phase(&S.tmem_empty[first], (sl.uses[first] & 1u) ^ 1u, S, args.status)) {
          aborted = true;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d0 = tmem + first * kSlotCols8;
        const uint32_t d1 = d0 + 128u;
        for (int ks = 0; ks < G.nk; ++ks) {
          if (!wait_phase(&S.full[s], ph, S, args.status)) {
            aborted = true;
            break;
          }
          const uint64_t a0 = desc0 + (uint64_t)s * (kStageQ >> 4);
          const uint64_t bd = a0 + (kABytesQ >> 4);
          const uint32_t acc = ks > 0 ? 1u : 0u;
          if (G.shared) {
            ptx::umma_bf16_x4(d0, a0, bd, idesc, acc);
            ptx::umma_bf16_x4(d1, a0 + ((kABytesQ / 2) >> 4), bd, idesc, acc);
          } else {
            umma_e4m3_x4(d0, a0, bd, idesc, acc);
            umma_e4m3_x4(d1, a0 + ((kABytesQ / 2) >> 4), bd, idesc, acc);
          }
          ptx::umma_commit(&S.empty[s]);
          if (++s == kStagesQ) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (aborted) break;
        ptx::umma_commit(&S.tmem_full[first]);
        sl.done(first, count);
      }
      if (aborted) {
        ptx::umma_commit(&S.drain);
        drain_phase(&S.drain, 0);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int qd = warp & 3;
    const int c0 = ((warp - 2) / 4) * 32;  // this warp's 32 token columns
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
    Slots8 sl;
    for (int qi = 0;; ++qi) {
      const int slot = qi % kQueue8;
      const bool got = wait_phase(&S.q_full[slot], (uint32_t)(qi / kQueue8) & 1u, S, args.status);
      if (!__all_sync(0xffffffffu, got)) break;
      const int tile = S.q[slot];
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&S.q_empty[slot]);
      if (tile < 0) break;
      const GeomQ G = geomq(args, S, tile, total, R);
      const Tile& tl = G.t;
      int first, count;
      sl.take(128, first, count);
      const uint32_t b0 = tmem + lane_off + first * kSlotCols8;
      const uint32_t b1 = b0 + 128u;
      const int ch = tl.m * 128 + qd * 32 + lane;  // this lane's channel
      float sg = 1.f, su = 1.f, xsc = 0.f;
      if (!G.shared) {
        const float* sp = aq.scale + (size_t)tl.g * 2 * args.I + ch;
        sg = __ldg(sp);
        su = __ldg(sp + args.I);
        if (c0 + lane < tl.nvalid) xsc = __ldg(aq.x_scale + tl.p0 + c0 + lane);
      }
      const bool ok = wait_phase(&S.tmem_full[first], sl.uses[first] & 1u, S, args.status);
      if (!__all_sync(0xffffffffu, ok)) break;
      ptx::tc_fence_after();
      if (c0 < tl.nvalid) {
        uint32_t r0[32], r1[32];
        ptx::tmem_ld32(b0 + c0, r0);
        ptx::tmem_ld32(b1 + c0, r1);
        if (!G.shared) {
          // add the lo columns (N + c0 + 31 < 128: N <= 64, c0 <= 32)
          uint32_t l0[32], l1[32];
          ptx::tmem_ld32(b0 + tl.N + c0, l0);
          ptx::tmem_ld32(b1 + tl.N + c0, l1);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float xs = __shfl_sync(0xffffffffu, xsc, j);
            r0[j] = __float_as_uint((__uint_as_float(r0[j]) + __uint_as_float(l0[j])) * sg * xs);
            r1[j] = __float_as_uint((__uint_as_float(r1[j]) + __uint_as_float(l1[j])) * su * xs);
          }
        } else {
          ptx::tmem_ld_wait();
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          if (c0 + j < tl.nvalid) {
            const float gv = __uint_as_float(r0[j]);
            // SiLU(g) = g / (1 + e^-g), fast exponential and division. Routed rows: the
            // bf16 pair (16 significant bits), split into E4M3 pieces before the down GEMM;
            // shared rows: the pair, or fp16(h 2^-8) for the fp16 down operands
            const float hv = __fdividef(gv, 1.f + __expf(-gv)) * __uint_as_float(r1[j]);
            const size_t at = (size_t)(tl.p0 + c0 + j) * args.ldh + ch;
            store_h(args.h, args.h_plane, at, hv, G.shared ? args.h_f16 : 0, args.status);
          }
        }
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(&S.tmem_empty[first]);
      sl.done(first, count);
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols8);
  }
}

// Token rows in dispatch order as two E4M3 pieces with a power-of-two row scale (see the
// gate|up kernel above): xs8[0][p] = hi, xs8[1][p] = lo, x_scale[p] = 2^-k. One warp per
// packed row; also zeroes the gate|up kernel's tile counter.
__global__ void __launch_bounds__(256)
gather_rows_e4m3_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ sorted_token,
                        const int* __restrict__ plan, int E, int T, int H, uint8_t* __restrict__ xs8,
                        float* __restrict__ x_scale, uint32_t* __restrict__ status,
                        int* __restrict__ counter) {
  if (blockIdx.x == 0 && threadIdx.x == 0) *counter = 0;
  const int R = plan_view(const_cast<int*>(plan), E).row0[E];
  const int lane = threadIdx.x & 31;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  for (int p = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; p < R; p += nwarps) {
    int t = sorted_token[p];
    if ((unsigned)t >= (unsigned)T) {
      set_flag(status, kFlagBounds);
      t = 0;
    }
    const uint16_t* src = x + (size_t)t * H;
    float amax = 0.f;
    for (int c = lane * 8; c < H; c += 256) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + c));
      amax = fmaxf(amax, fmaxf(fmaxf(fabsf(bf16lo(v.x)), fabsf(bf16hi(v.x))),
                               fmaxf(fabsf(bf16lo(v.y)), fabsf(bf16hi(v.y)))));
      amax = fmaxf(amax, fmaxf(fmaxf(fabsf(bf16lo(v.z)), fabsf(bf16hi(v.z))),
                               fmaxf(fabsf(bf16lo(v.w)), fabsf(bf16hi(v.w)))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    // k with amax * 2^k in [128, 256): k = 7 - floor(log2 amax), kept inside the normal range
    int k = 0;
    if (amax > 0.f) {
      const int e = (int)((__float_as_uint(amax) >> 23) & 0xFF) - 127;
      k = min(max(7 - e, -120), 120);
    }
    const float up = __uint_as_float((uint32_t)(127 + k) << 23);
    if (lane == 0) x_scale[p] = __uint_as_float((uint32_t)(127 - k) << 23);
    uint8_t* hi_row = xs8 + (size_t)p * H;
    uint8_t* lo_row = xs8 + ((size_t)R + p) * H;
    for (int c = lane * 16; c < H; c += 512) {
      const uint4 v0 = __ldg(reinterpret_cast<const uint4*>(src + c));
      const uint4 v1 = __ldg(reinterpret_cast<const uint4*>(src + c + 8));
      const uint32_t u[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
      uint32_t hw[4] = {0u, 0u, 0u, 0u}, lw[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const uint32_t bits = (i & 1) ? (u[i >> 1] >> 16) : (u[i >> 1] & 0xFFFFu);
        const float v = __uint_as_float(bits << 16) * up;  // exact: a power of two
        const __nv_fp8_storage_t h8 = __nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
        const float hv = __half2float(__half(__nv_cvt_fp8_to_halfraw(h8, __NV_E4M3)));
        const __nv_fp8_storage_t l8 = __nv_cvt_float_to_fp8(v - hv, __NV_SATFINITE, __NV_E4M3);
        hw[i >> 2] |= (uint32_t)h8 << (8 * (i & 3));
        lw[i >> 2] |= (uint32_t)l8 << (8 * (i & 3));
      }
      *reinterpret_cast<uint4*>(hi_row + c) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4*>(lo_row + c) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
  }
}


// ================================================================ down on FP8 tensor cores
// h (the SwiGLU intermediate) carries more significant bits than x: the gate|up epilogue
// stores the routed rows as the bf16 pair hi + lo (16 bits). Before the down GEMM each row
// is split into four E4M3 pieces with a power-of-two row scale 2^k (the row's largest |h|
// times 2^k in [128, 256)):
//   v = h 2^k,  p1 = E4M3(v),  r1 = v - p1,  p(i+1) = E4M3(16 ri),  r(i+1) = 16 ri - p(i+1),
//   v = p1 + p2 / 16 + p3 / 256 + p4 / 4096 + r4 / 4096.
// Rounding to nearest leaves each remainder within half a unit of its piece's last place,
// so 16 times it fits E4M3 again (|16 ri| <= 128), every subtraction is exact, and the
// neglected r4 / 4096 is at most 2^-16 |v| (or 2^-22 below E4M3's normal range, against
// the row's largest |v| >= 128): the pair's precision. The four pieces of a tile's rows
// follow each other in shared memory, so one MMA of N = 4 x rows gives W p1 .. W p4 in four
// column blocks; the epilogue folds them (p4 / 16 + p3) / 16 ... and multiplies by the
// weight row's scale, the token row's 2^-k and its routing weight. K = 128 codes per stage;
// tiles of at most 32 token rows, so that a tile's two accumulators (4 x 32 columns each)
// share one 256-column TMEM slot and the next tile's MMAs overlap this tile's epilogue.
// Roles: warp 0 TMA producer, warp 1 TMEM owner and MMA issuer, warps 2-9 epilogue (warp w
// reads TMEM lanes 32 (w % 4) .. of accumulator (w - 2) / 4).

constexpr int kPiecesD = 4;
constexpr int kEpiWarpsD = 8;
constexpr int kThreadsD = 64 + 32 * kEpiWarpsD;
constexpr int kMaxTileD = kTcChunkDown8;                  // 32 token rows per tile
constexpr uint32_t kABytesD = 2 * 128 * 128;              // 2 x 128 weight rows x 128 B
constexpr uint32_t kBBytesD = kPiecesD * kMaxTileD * 128;  // 4 pieces x 32 rows x 128 B
constexpr uint32_t kStageD = kABytesD + kBBytesD;
constexpr int kStagesD = 4;
constexpr int kBoxHeightsD = 2;  // token boxes of 32 and 16 rows
static_assert(kPiecesD * kMaxTileD <= 128, "both accumulators must fit one TMEM slot");

struct SharedD {
  uint64_t full[kStagesD];
  uint64_t empty[kStagesD];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t q_full[kQueue8];
  uint64_t q_empty[kQueue8];
  uint64_t drain;
  uint32_t tmem_base;
  volatile int abort;
  int q[kQueue8];
  int tp[kMaxE + 2];
  int row0[kMaxE + 2];
  float4 xpose[kEpiWarpsD][8][8];  // per warp, 8 tokens x 32 channels
};

constexpr size_t smemd_bytes() { return 1024 + (size_t)kStagesD * kStageD + sizeof(SharedD); }
static_assert(smemd_bytes() <= 232448, "over the 227 KB of shared memory a CTA may use");
static_assert(kStageD % 1024 == 0, "stages must keep 1024-byte alignment for the 128-byte swizzle");

struct TokenMapsD {
  CUtensorMap m[kBoxHeightsD];
};

struct DownQArgs {
  TcArgs a;
  const float* scale;    // fp32 [E][H] weight row scales
  const float* h_scale;  // fp32 [R] 2^-k of each packed row's pieces
  int plane_rows;        // rows per plane of h (the shared rows' lo plane follows at this offset)
  int shared_f16;        // shared rows of h as fp16(h 2^-8) against fp16(W 2^8), else the pair
};

struct GeomD {
  Tile t;
  int a_row0, a_row1, nk, nb, hidx;  // nb: token row blocks (pieces, or planes of h)
  bool shared;
};

// Tile order: the shared expert's tiles first, then the routed groups in order.
__device__ __forceinline__ GeomD geomd(const DownQArgs& aq, const SharedD& S, int tile,
                                       int total) {
  const TcArgs& a = aq.a;
  const int tpE = S.tp[a.E];
  const int nsh = total - tpE;
  const int t2 = tile < nsh ? tpE + tile : tile - nsh;
  GeomD G;
  G.t = decode_tile(S.row0, S.tp, a.E, t2, kMaxTileD);
  G.shared = G.t.g == a.E;
  const int base = G.shared ? 0 : G.t.g * a.H;
  G.a_row0 = base + G.t.m * 256;
  G.a_row1 = G.a_row0 + 128;
  G.nk = G.shared ? a.Is / 64 : a.I / 128;
  G.nb = G.shared ? (aq.shared_f16 ? 1 : 2) : kPiecesD;
  G.hidx = G.t.N > 16 ? 0 : 1;
  return G;
}

// The routed rows of h (packed rows [0, R)) as four E4M3 pieces and a row scale:
// hp[i][p] = piece i + 1 of row p (I codes; plane stride R rows), h_scale[p] = 2^-k.
// One warp per row; pairs of values go through the paired conversions.
__global__ void __launch_bounds__(256)
h_pieces_e4m3_kernel(const uint16_t* __restrict__ h, size_t h_plane, int ldh,
                     const int* __restrict__ plan, int E, int I, uint8_t* __restrict__ hp,
                     float* __restrict__ h_scale, uint32_t* __restrict__ status) {
  const int R = plan_view(const_cast<int*>(plan), E).row0[E];
  const int lane = threadIdx.x & 31;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  for (int p = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; p < R; p += nwarps) {
    const uint16_t* hi = h + (size_t)p * ldh;
    const uint16_t* lo = hi + h_plane;
    float amax = 0.f;
    for (int c = lane * 8; c < I; c += 256) {
      const uint4 a = __ldg(reinterpret_cast<const uint4*>(hi + c));
      const uint4 b = __ldg(reinterpret_cast<const uint4*>(lo + c));
      const uint32_t ua[4] = {a.x, a.y, a.z, a.w}, ub[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
        amax = fmaxf(amax, fmaxf(fabsf(bf16lo(ua[i]) + bf16lo(ub[i])),
                                 fabsf(bf16hi(ua[i]) + bf16hi(ub[i]))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (!(amax <= 3.0e38f) && lane == 0) set_flag(status, kFlagRange);  // inf or NaN in h
    // k with amax 2^k in [128, 256): k = 7 - floor(log2 amax), inside the normal range
    int k = 0;
    if (amax > 0.f) {
      const int e = (int)((__float_as_uint(amax) >> 23) & 0xFF) - 127;
      k = min(max(7 - e, -120), 120);
    }
    const float up = __uint_as_float((uint32_t)(127 + k) << 23);
    if (lane == 0) h_scale[p] = __uint_as_float((uint32_t)(127 - k) << 23);
    for (int c = lane * 8; c < I; c += 256) {
      const uint4 a = __ldg(reinterpret_cast<const uint4*>(hi + c));
      const uint4 b = __ldg(reinterpret_cast<const uint4*>(lo + c));
      const uint32_t ua[4] = {a.x, a.y, a.z, a.w}, ub[4] = {b.x, b.y, b.z, b.w};
      uint32_t q[kPiecesD][2] = {};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        // hi + lo is exact in fp32 (lo is below half a unit of hi's last place); the power
        // of two is exact too
        float2 r = make_float2((bf16lo(ua[i]) + bf16lo(ub[i])) * up,
                               (bf16hi(ua[i]) + bf16hi(ub[i])) * up);
#pragma unroll
        for (int j = 0; j < kPiecesD; ++j) {
          const __nv_fp8x2_storage_t e8 = __nv_cvt_float2_to_fp8x2(r, __NV_SATFINITE, __NV_E4M3);
          const float2 back = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2(e8, __NV_E4M3)));
          q[j][i >> 1] |= (uint32_t)e8 << (16 * (i & 1));
          r = make_float2((r.x - back.x) * 16.f, (r.y - back.y) * 16.f);
        }
      }
#pragma unroll
      for (int j = 0; j < kPiecesD; ++j)
        *reinterpret_cast<uint2*>(hp + ((size_t)j * R + p) * I + c) = make_uint2(q[j][0], q[j][1]);
    }
  }
}

__global__ void __launch_bounds__(kThreadsD, 1)
tc8_down_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_a_sh,
                const __grid_constant__ TokenMapsD tm_hp, const __grid_constant__ TokenMapsD tm_hs,
                const DownQArgs aq) {
  const TcArgs& args = aq.a;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  SharedD& S = *reinterpret_cast<SharedD*>(smem + kStagesD * kStageD);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = args.E;
  const PlanView pv = plan_view(const_cast<int*>(args.plan), E);
  for (int g = threadIdx.x; g < E + 2; g += blockDim.x) {
    S.tp[g] = pv.tp5[g];
    S.row0[g] = pv.row0[g];
  }
  const int total = pv.tp5[E + 1];
  const int R = pv.row0[E];

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesD; ++s) {
      ptx::mbar_init(&S.full[s], 1);
      ptx::mbar_init(&S.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&S.tmem_full[b], 1);
      ptx::mbar_init(&S.tmem_empty[b], 32 * kEpiWarpsD);
    }
    for (int i = 0; i < kQueue8; ++i) {
      ptx::mbar_init(&S.q_full[i], 1);
      ptx::mbar_init(&S.q_empty[i], 1 + kEpiWarpsD);
    }
    ptx::mbar_init(&S.drain, 1);
    S.abort = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tm_q);
    ptx::prefetch_tmap(&tm_a_sh);
    for (int i = 0; i < kBoxHeightsD; ++i) {
      ptx::prefetch_tmap(&tm_hp.m[i]);
      ptx::prefetch_tmap(&tm_hs.m[i]);
    }
  }
  if (warp == 1) {
    ptx::tmem_alloc(&S.tmem_base, kTmemCols8);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = S.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    int it = 0;
    int armed[kStagesD];
#pragma unroll
    for (int s = 0; s < kStagesD; ++s) armed[s] = -1;
    bool aborted = false;
    int ahead = (lane == 0) ? atomicAdd(args.counter, 1) : 0;
    for (int qi = 0; !aborted; ++qi) {
      const int slot = qi % kQueue8;
      int tile = 0;
      if (lane == 0) {
        if (!wait_phase(&S.q_empty[slot], ((uint32_t)(qi / kQueue8) & 1u) ^ 1u, S, args.status)) {
          tile = -2;
        } else {
          tile = ahead;
          if (tile >= total) tile = -1;
          else ahead = atomicAdd(args.counter, 1);
          S.q[slot] = tile;
          ptx::mbar_arrive(&S.q_full[slot]);
        }
      }
      tile = __shfl_sync(0xffffffffu, tile, 0);
      if (tile == -2) aborted = true;
      if (tile < 0) break;
      const GeomD G = geomd(aq, S, tile, total);
      const int kstep = G.shared ? 64 : 128;  // elements per 128-byte row
      // lanes 0, 1: the two accumulators' weight rows; lanes 2 ..: one token row block each
      // (routed: piece j of the rows; shared: plane j of h)
      const CUtensorMap* my_map = nullptr;
      uint32_t my_off = 0;
      int my_row = 0;
      if (lane < 2) {
        my_map = G.shared ? &tm_a_sh : &tm_q;
        my_off = lane * (kABytesD / 2);
        my_row = lane ? G.a_row1 : G.a_row0;
      } else if (lane - 2 < G.nb) {
        const int j = lane - 2;
        my_map = G.shared ? &tm_hs.m[G.hidx] : &tm_hp.m[G.hidx];
        my_off = kABytesD + (uint32_t)(j * G.t.N) * 128u;
        my_row = G.t.p0 + j * (G.shared ? aq.plane_rows : R);
      }
      const uint32_t bytes = kABytesD + (uint32_t)G.nb * G.t.N * 128u;
      for (int ks = 0; ks < G.nk; ++ks, ++it) {
        const int s = it % kStagesD;
        const uint32_t ph = (uint32_t)(it / kStagesD) & 1u;
        bool ok = true;
        if (lane == 0) {
          ok = wait_phase(&S.empty[s], ph ^ 1u, S, args.status);
          if (ok) {
            ptx::mbar_arrive_expect_tx(&S.full[s], bytes);
            armed[s] = (int)ph;
          }
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) {
          aborted = true;
          break;
        }
        if (my_map)
          ptx::tma_load_2d(smem + s * kStageD + my_off, my_map, &S.full[s], ks * kstep, my_row);
      }
    }
    if (aborted && lane == 0) {
      for (int s = 0; s < kStagesD; ++s)
        if (armed[s] >= 0) drain_phase(&S.full[s], (uint32_t)armed[s]);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      Slots8 sl;
      bool aborted = false;
      const uint64_t desc0 = ptx::smem_desc_kmajor<128>(smem);
      for (int qi = 0; !aborted; ++qi) {
        const int slot = qi % kQueue8;
        if (!wait_phase(&S.q_full[slot], (uint32_t)(qi / kQueue8) & 1u, S, args.status)) {
          aborted = true;
          break;
        }
        const int tile = S.q[slot];
        ptx::mbar_arrive(&S.q_empty[slot]);
        if (tile < 0) break;
        const GeomD G = geomd(aq, S, tile, total);
        // routed: columns [jN, (j+1)N) W p(j+1); shared: [0, N) W h_hi (or W' h'), [N, 2N)
        // W h_lo. At most 128 columns: the second accumulator at +128
        const int cols = G.nb * G.t.N;
        const uint32_t idesc = !G.shared      ? idesc_e4m3_f32(128, cols)
                               : aq.shared_f16 ? ptx::idesc_f16_f32(128, cols)
                                               : ptx::idesc_bf16_f32(128, cols);
        int first, count;
        sl.take(128, first, count);
        if (!wait_phase(&S.tmem_empty[first], (sl.uses[first] & 1u) ^ 1u, S, args.status)) {
          aborted = true;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d0 = tmem + first * kSlotCols8;
        const uint32_t d1 = d0 + 128u;
        for (int ks = 0; ks < G.nk; ++ks) {
          if (!wait_phase(&S.full[s], ph, S, args.status)) {
            aborted = true;
            break;
          }
          const uint64_t a0 = desc0 + (uint64_t)s * (kStageD >> 4);
          const uint64_t bd = a0 + (kABytesD >> 4);
          const uint32_t acc = ks > 0 ? 1u : 0u;
          if (G.shared) {
            ptx::umma_bf16_x4(d0, a0, bd, idesc, acc);
            ptx::umma_bf16_x4(d1, a0 + ((kABytesD / 2) >> 4), bd, idesc, acc);
          } else {
            umma_e4m3_x4(d0, a0, bd, idesc, acc);
            umma_e4m3_x4(d1, a0 + ((kABytesD / 2) >> 4), bd, idesc, acc);
          }
          ptx::umma_commit(&S.empty[s]);
          if (++s == kStagesD) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (aborted) break;
        ptx::umma_commit(&S.tmem_full[first]);
        sl.done(first, count);
      }
      if (aborted) {
        ptx::umma_commit(&S.drain);
        drain_phase(&S.drain, 0);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;               // 0 .. kEpiWarpsD - 1
    const int accn = ew >> 2;              // accumulator 0 or 1 (weight rows +128)
    const int qd = warp & 3;               // TMEM lanes 32*qd .. +31 (warp % 4 rule)
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
    Slots8 sl;
    for (int qi = 0;; ++qi) {
      const int slot = qi % kQueue8;
      const bool got = wait_phase(&S.q_full[slot], (uint32_t)(qi / kQueue8) & 1u, S, args.status);
      if (!__all_sync(0xffffffffu, got)) break;
      const int tile = S.q[slot];
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&S.q_empty[slot]);
      if (tile < 0) break;
      const GeomD G = geomd(aq, S, tile, total);
      const Tile& tl = G.t;
      int first, count;
      sl.take(128, first, count);
      const uint32_t b0 = tmem + lane_off + first * kSlotCols8 + accn * 128u;
      const int mrow0 = tl.m * 256 + accn * 128 + qd * 32;  // this warp's first weight row
      // this lane's weight row scale (1 for the bf16 shared expert), and the token and
      // weight of column `lane`: routing weight x 2^-k (routed), shared gate (shared)
      const float sc = G.shared ? 1.f : __ldg(aq.scale + (size_t)tl.g * args.H + mrow0 + lane);
      int col_tok = 0;
      float col_w = 0.f;
      if (lane < tl.nvalid) {
        const int p = tl.p0 + lane;
        col_tok = token_of_row(args, p, R);
        col_w = G.shared ? args.sgate[col_tok] : args.sorted_w[p] * aq.h_scale[p];
      }
      const bool ok = wait_phase(&S.tmem_full[first], sl.uses[first] & 1u, S, args.status);
      if (!__all_sync(0xffffffffu, ok)) break;
      ptx::tc_fence_after();
      uint32_t r[32];
      {
        const int N = tl.N;
        uint32_t r2[32];
        ptx::tmem_ld32(b0, r);
        if (!G.shared) {
          uint32_t r3[32], r4[32];
          ptx::tmem_ld32(b0 + N, r2);
          ptx::tmem_ld32(b0 + 2 * N, r3);
          ptx::tmem_ld32(b0 + 3 * N, r4);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            float v = fmaf(__uint_as_float(r4[j]), 0.0625f, __uint_as_float(r3[j]));
            v = fmaf(v, 0.0625f, __uint_as_float(r2[j]));
            v = fmaf(v, 0.0625f, __uint_as_float(r[j]));
            r[j] = __float_as_uint(v * sc);
          }
        } else if (!aq.shared_f16) {
          ptx::tmem_ld32(b0 + N, r2);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j)
            r[j] = __float_as_uint(__uint_as_float(r[j]) + __uint_as_float(r2[j]));
        } else {
          ptx::tmem_ld_wait();
        }
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(&S.tmem_empty[first]);  // the accumulator is in registers now
      sl.done(first, count);
      // 32 channels (lanes) x 32 tokens (registers), regrouped through shared memory 8
      // tokens at a time so that each 16-byte atomic add of a warp lands in whole 128-byte
      // lines of one token's output row
      const int m = mrow0 + 4 * (lane & 7);
      float4(&xp)[8][8] = S.xpose[ew];
      float* xs = reinterpret_cast<float*>(&xp[0][0]);
#pragma unroll
      for (int sb = 0; sb < 4; ++sb) {
        if (sb * 8 >= tl.nvalid) break;
        __syncwarp();
#pragma unroll
        for (int q = 0; q < 8; ++q) xs[q * 32 + lane] = __uint_as_float(r[sb * 8 + q]);
        __syncwarp();
#pragma unroll
        for (int hq = 0; hq < 2; ++hq) {
          const int q = hq * 4 + (lane >> 3);
          const float4 v = xp[q][lane & 7];
          const int col = sb * 8 + q;
          const int t = __shfl_sync(0xffffffffu, col_tok, col);
          const float w = __shfl_sync(0xffffffffu, col_w, col);
          if (col < tl.nvalid)
            atomicAdd(reinterpret_cast<float4*>(args.out + (size_t)t * args.H + m),
                      make_float4(w * v.x, w * v.y, w * v.z, w * v.w));
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols8);
  }
}

// ---------------------------------------------------------------- host side

// 2-D E4M3 tensor [outer][inner] in boxes of box_outer rows x 128 codes, 128-byte swizzle
// (the operand layout of the kind::f8f6f4 MMAs).
bool make_map_e4m3_sw128(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                         uint32_t box_outer) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner};
  cuuint32_t box[2] = {128, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_token_maps8(TokenMaps8* b, const void* base, uint64_t inner, uint64_t outer) {
  for (int i = 0; i < kBoxHeights8; ++i)
    if (!make_map(&b->m[i], base, inner, outer, 64, (uint32_t)(128 >> i))) return false;
  return true;
}

}  // namespace

bool tc8_supported(const moe_shape& s) { return tc_supported(s); }

cudaError_t launch_tc8_gate_up(const moe_shape& s, const Layout& L, char* ws, const uint16_t* x,
                               const int32_t* sorted_token, const moe_weights& w,
                               const moe_fp8_experts& q, cudaStream_t st) {
  // token rows as E4M3 pieces into the bf16 gather buffer (2 x R x H bytes = its size) and
  // their row scales into the router-logit buffer (read by the top-k kernel before this)
  uint8_t* xs8 = reinterpret_cast<uint8_t*>(ws + L.xs);
  float* x_scale = reinterpret_cast<float*>(ws + L.logits);
  {
    LaunchScope scope(MOE_K_OTHER, st);
    gather_rows_e4m3_kernel<<<sm_count() * 8, 256, 0, st>>>(
        x, sorted_token, reinterpret_cast<const int*>(ws + L.plan), s.E, s.T, s.H, xs8, x_scale,
        reinterpret_cast<uint32_t*>(ws + L.status), reinterpret_cast<int*>(ws + L.sched) + 0);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const uint64_t R = (uint64_t)s.T * s.k;
  CUtensorMap qm, a_sh;
  TokenMaps8 b8, b_sh;
  bool ok = make_map_e4m3_sw128(&qm, q.q_gate_up, s.H, (uint64_t)s.E * 2 * s.I, 128) &&
            make_map(&a_sh, w.ws_gate_up, s.H, 2ull * s.Is, 64, 128) &&
            make_token_maps8(&b_sh, x, s.H, (uint64_t)s.T);
  for (int i = 0; ok && i < kBoxHeights8; ++i)
    ok = make_map_e4m3_sw128(&b8.m[i], xs8, s.H, 2 * R, (uint32_t)(128 >> i));
  if (!ok) return cudaErrorInvalidValue;
  GateUpQArgs args{};
  args.a = base_args(s, L, ws);
  args.a.sorted_token = sorted_token;
  args.a.counter = reinterpret_cast<int*>(ws + L.sched) + 0;
  args.a.counter_next = reinterpret_cast<int*>(ws + L.sched) + 1;
  args.scale = q.s_gate_up;
  args.x_scale = x_scale;
  args.a.h_f16 = w.ws_down_f16 ? 1 : 0;  // shared rows of h as fp16(h 2^-8)
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(tc8_gate_up_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)smemq_bytes());
  });
  if (attr_err != cudaSuccess) return attr_err;
  LaunchScope scope(MOE_K_GATE_UP, st);
  tc8_gate_up_kernel<<<sm_count(), kThreadsQ, smemq_bytes(), st>>>(qm, a_sh, b8, b_sh, args);
  return cudaGetLastError();
}


cudaError_t launch_tc8_down(const moe_shape& s, const Layout& L, char* ws,
                            const int32_t* sorted_token, const float* sorted_w, const float* sgate,
                            const moe_weights& w, const moe_fp8_experts& q, float* out,
                            cudaStream_t st) {
  // h's routed rows as E4M3 pieces into the gather buffer (free once gate|up has run)
  uint8_t* hp = reinterpret_cast<uint8_t*>(ws + L.xs);
  float* h_scale = reinterpret_cast<float*>(ws + L.xs + fp8_h_pieces_bytes(s));
  {
    LaunchScope scope(MOE_K_OTHER, st);
    h_pieces_e4m3_kernel<<<sm_count() * 8, 256, 0, st>>>(
        reinterpret_cast<const uint16_t*>(ws + L.h), L.h_plane, L.ldh,
        reinterpret_cast<const int*>(ws + L.plan), s.E, s.I, hp, h_scale,
        reinterpret_cast<uint32_t*>(ws + L.status));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const bool f16 = w.ws_down_f16 != nullptr;  // then the shared rows of h are fp16(h 2^-8)
  const CUtensorMapDataType dt =
      f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const uint64_t Rcap = (uint64_t)s.T * s.k;
  const uint64_t plane_rows = L.h_plane / L.ldh;
  CUtensorMap qm, a_sh;
  TokenMapsD bp, bs;
  bool ok = make_map_e4m3_sw128(&qm, q.q_down, s.I, (uint64_t)s.E * s.H, 128) &&
            make_map(&a_sh, f16 ? w.ws_down_f16 : w.ws_down, s.Is, (uint64_t)s.H, 64, 128, dt);
  for (int i = 0; ok && i < kBoxHeightsD; ++i) {
    const uint32_t rows = (uint32_t)kMaxTileD >> i;
    ok = make_map_e4m3_sw128(&bp.m[i], hp, s.I, kPiecesD * Rcap, rows) &&
         make_map(&bs.m[i], ws + L.h, L.ldh, 2 * plane_rows, 64, rows, dt);
  }
  if (!ok) return cudaErrorInvalidValue;
  DownQArgs args{};
  args.a = base_args(s, L, ws);
  args.a.sorted_token = sorted_token;
  args.a.sorted_w = sorted_w;
  args.a.sgate = sgate;
  args.a.out = out;
  args.a.counter = reinterpret_cast<int*>(ws + L.sched) + 1;  // zeroed by the gate|up kernel
  args.scale = q.s_down;
  args.h_scale = h_scale;
  args.plane_rows = (int)plane_rows;
  args.shared_f16 = f16 ? 1 : 0;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(tc8_down_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)smemd_bytes());
  });
  if (attr_err != cudaSuccess) return attr_err;
  LaunchScope scope(MOE_K_DOWN, st);
  tc8_down_kernel<<<sm_count(), kThreadsD, smemd_bytes(), st>>>(qm, a_sh, bp, bs, args);
  return cudaGetLastError();
}

}  // namespace moe
