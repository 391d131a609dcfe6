// tc8_gemm.cu -- stage 4, "Grouped expert GEMMs" (Qwen3.8-Flash-Next architecture study,
// MoE pipeline diagram), with the routed experts' weights stored in FP8 ("Qwen3.8, weights
// in hand: 98% of a 2.4T model is routed experts", section "What FP8 actually quantizes":
// routed experts in FP8, the shared expert in bf16). Each weight row carries an fp32 scale
// that multiplies its accumulator row in the epilogue, so the layer sees
// decode(code) * scale. What changes against the bf16 layer is the bytes: one per routed
// weight instead of two, which is what bounds a decode-size batch. Two kernels, one CTA per
// tile, swap AB as in the bf16 kernels (2 x 128 weight rows on the MMA's M side, tokens on N):
//
// down (tc8_down_kernel): weight-only. The E4M3 codes are widened in shared memory
// (exactly: a code has a 4-bit significand) and the tensor cores run the MMAs of the bf16
// layer, K = 64 per stage. Two forms (template F16): widened to bf16 against h's hi and lo
// rows (one MMA of N = 2 x rows, up to 128 rows); or, when the fp16 down operands are given
// (the shared expert's fp16(W x 2^8) and h' = fp16(h x 2^-8)), widened to fp16 against the
// one h' plane (N = rows), which halves the h rows a staging slot holds, so four slots fit
// where three did. Roles of the 320 threads:
//   warp 0      TMA producer over a ring of staging slots: per stage, the E4M3 codes of
//               the 256 weight rows (16 KB, plain 64-byte rows) and the h rows;
//   warp 1      TMEM owner and MMA issuer (lane 0);
//   warps 2-5   converters: E4M3 staging -> bf16 operand in a two-slot ring, in the
//               128-byte-swizzled K-major layout the MMA reads (the layout a TMA copy
//               with that swizzle writes);
//   warps 6-9   epilogue (one warp per 32 TMEM lanes, all column chunks).
// The shared expert's tiles load bf16 weights straight into the staging slot, one
// accumulator's 128 rows (16 KB) per stage, so they take twice the stages and skip the
// converters; they are handed out first, being the longest tiles.
// Barriers: staging full/empty (TMA bytes / MMA commit), operand ready/free (converter
// warps / MMA commit), TMEM full/empty, a tile queue. Every wait is bounded (2 s).
//
// gate|up (tc8_gate_up_kernel): E4M3 MMAs (kind::f8f6f4) on the codes as loaded, with the
// token rows split into two E4M3 pieces; described above the kernel.
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <algorithm>

#include "tc_common.cuh"
#include "tc_gemm.h"

namespace moe {
namespace {

constexpr int kConvWarps = 4;
constexpr int kEpiWarps8 = 4;
constexpr int kThreads8 = 64 + 32 * (kConvWarps + kEpiWarps8);
constexpr int kQueue8 = 4;
constexpr uint32_t kTmemCols8 = 512;
constexpr uint32_t kSlotCols8 = 256;
constexpr int kBK8 = 64;                       // K per stage
constexpr uint32_t kRowB = 128;                // one bf16 operand row of a stage (64 K)
constexpr uint32_t kAccBytes = 128 * kRowB;    // 128 weight rows of bf16: one accumulator
constexpr uint32_t kQRowB = 64;                // one E4M3 row of a stage
constexpr uint32_t kQBytes = 256 * kQRowB;     // 256 weight rows of E4M3 (= kAccBytes)
constexpr int kBoxHeights8 = 4;                // token boxes of 128, 64, 32, 16 rows
constexpr int kARing = 2;                      // widened operand slots
constexpr int kMaxSlots8 = 4;

template <bool F16>
struct Cfg8 {
  static constexpr int kMaxTile = kTcChunkDown;
  static constexpr int kBTiles = F16 ? 1 : 2;  // h' rows, or hi and lo rows of h
  static constexpr uint32_t kBBytes = (uint32_t)kBTiles * kMaxTile * kRowB;
  static constexpr uint32_t kSlotBytes = kQBytes + kBBytes;  // a multiple of 1024
  static constexpr int kSlots = F16 ? 4 : 3;
  static constexpr uint32_t kAStage = 2 * kAccBytes;
};

struct Shared8 {
  uint64_t sfull[kMaxSlots8];
  uint64_t sempty[kMaxSlots8];
  uint64_t aready[kARing];
  uint64_t afree[kARing];
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
  float4 xpose[kEpiWarps8][8][8];  // down epilogue: per warp, 8 tokens x 32 channels
};

template <bool F16>
constexpr size_t smem8_bytes() {
  using C = Cfg8<F16>;
  return 1024 + (size_t)C::kSlots * C::kSlotBytes + (size_t)kARing * C::kAStage + sizeof(Shared8);
}
static_assert(smem8_bytes<false>() <= 232448 && smem8_bytes<true>() <= 232448,
              "over the 227 KB of shared memory a CTA may use");
static_assert(Cfg8<false>::kSlotBytes % 1024 == 0 && Cfg8<true>::kSlotBytes % 1024 == 0,
              "staging slots must keep 1024-byte alignment for the 128-byte swizzle");
static_assert(Cfg8<true>::kSlots <= kMaxSlots8 && Cfg8<false>::kSlots <= kMaxSlots8, "slots");

struct TokenMaps8 {
  CUtensorMap m[kBoxHeights8];
};

struct Tc8Args {
  TcArgs a;
  const float* scale;  // fp32 row scales of the E4M3 bank: [E][2I] (gate|up) or [E][H] (down)
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

struct Geom8 {
  Tile t;
  int a_row0, a_row1;  // weight rows of the two accumulators
  int b_row0;          // first row of the token tile in its tensor map
  int nk;              // stages: K / 64 for E4M3 tiles, 2 K / 64 for the shared expert's
  bool shared;
};

// Tile order: the shared expert's tiles first (group E), then the routed groups in order.
__device__ __forceinline__ Geom8 geom8(const TcArgs& a, const Shared8& S, int tile, int total,
                                       int R) {
  const int tpE = S.tp[a.E];
  const int nsh = total - tpE;
  const int t2 = tile < nsh ? tpE + tile : tile - nsh;
  Geom8 G;
  G.t = decode_tile(S.row0, S.tp, a.E, t2, Cfg8<false>::kMaxTile);
  G.shared = G.t.g == a.E;
  const int base = G.shared ? 0 : G.t.g * a.H;
  G.a_row0 = base + G.t.m * 256;
  G.a_row1 = G.a_row0 + 128;
  G.b_row0 = G.t.p0;
  const int K = G.shared ? a.Is : a.I;
  G.nk = (G.shared ? 2 : 1) * (K / kBK8);
  return G;
}

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

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Two E4M3 codes (bytes 2i and 2i+1 of w, i = 0 or 1 by the selector) -> two bf16, exactly.
// prmt puts each code in the low byte of a 16-bit lane and its sign, replicated, in the high
// byte; shifting left by 4 and masking leaves sign | exponent(4) | mantissa(3) << 4, the
// bf16 pattern of code * 2^-120 (E4M3 subnormals become bf16 subnormals with the same
// value relation); the bf16 multiply by 2^120 then gives the code's value, exact because the
// result has at most 4 significant bits.
template <uint32_t kSel>
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t w) {
  uint32_t t, r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(t) : "r"(w), "r"(0u), "r"(kSel));
  t = (t << 4) & 0x87F087F0u;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(t), "r"(0x7B807B80u), "r"(0x80008000u));
  return r;
}

// The same to two fp16. Shifting left by 7 and masking leaves sign | 0 | exponent(4) |
// mantissa(3) << 7, the fp16 pattern of code * 2^-8 (fp16's exponent bias is 8 above E4M3's;
// E4M3 subnormals become fp16 subnormals with the same relation); the fp16 multiply by 2^8
// gives the code's value, exact (at most 4 significant bits, at most 448).
template <uint32_t kSel>
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t w) {
  uint32_t t, r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(t) : "r"(w), "r"(0u), "r"(kSel));
  t = (t << 7) & 0xBF80BF80u;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(t), "r"(0x5C005C00u), "r"(0x80008000u));
  return r;
}

template <bool F16, uint32_t kSel>
__device__ __forceinline__ uint32_t widen8(uint32_t w) {
  return F16 ? e4m3x2_to_f16x2<kSel>(w) : e4m3x2_to_bf16x2<kSel>(w);
}

template <bool F16>
__global__ void __launch_bounds__(kThreads8, 1)
tc8_down_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_a_sh,
                const __grid_constant__ TokenMaps8 tm_b, const Tc8Args a8) {
  using C = Cfg8<F16>;
  const TcArgs& args = a8.a;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* aring = smem + C::kSlots * C::kSlotBytes;
  Shared8& S = *reinterpret_cast<Shared8*>(aring + kARing * C::kAStage);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = args.E;

  const PlanView pv = plan_view(const_cast<int*>(args.plan), E);
  const int* tpg = pv.tp2;
  for (int g = threadIdx.x; g < E + 2; g += blockDim.x) {
    S.tp[g] = tpg[g];
    S.row0[g] = pv.row0[g];
  }
  const int total = tpg[E + 1];
  const int R = pv.row0[E];

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kSlots; ++s) {
      ptx::mbar_init(&S.sfull[s], 1);
      ptx::mbar_init(&S.sempty[s], 1);
    }
    for (int c = 0; c < kARing; ++c) {
      ptx::mbar_init(&S.aready[c], kConvWarps);
      ptx::mbar_init(&S.afree[c], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&S.tmem_full[b], 1);
      ptx::mbar_init(&S.tmem_empty[b], 32 * kEpiWarps8);
    }
    for (int i = 0; i < kQueue8; ++i) {
      ptx::mbar_init(&S.q_full[i], 1);
      ptx::mbar_init(&S.q_empty[i], 1 + kConvWarps + kEpiWarps8);
    }
    ptx::mbar_init(&S.drain, 1);
    S.abort = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tm_q);
    ptx::prefetch_tmap(&tm_a_sh);
    for (int i = 0; i < kBoxHeights8; ++i) ptx::prefetch_tmap(&tm_b.m[i]);
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
    int js = 0;  // staging stage sequence (every stage of every tile)
    int armed[C::kSlots];
#pragma unroll
    for (int s = 0; s < C::kSlots; ++s) armed[s] = -1;
    bool aborted = false;
    const int plane_rows = (int)(args.h_plane / (size_t)args.ldh);
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
      const Geom8 G = geom8(args, S, tile, total, R);
      // token piece of this lane (lanes 2..): plane, first row and box height
      const CUtensorMap* bmap = nullptr;
      uint32_t boff = 0;
      int brow = 0;
      if (lane >= 2) {
        int np = 0, r, h;
        while (token_piece8(G.t.N, np, r, h)) ++np;
        const int j = lane - 2;
        if (j < np * C::kBTiles) {
          const int plane = j / np;
          token_piece8(G.t.N, j - plane * np, r, h);
          bmap = &tm_b.m[h];
          boff = kQBytes + (uint32_t)(plane * G.t.N + r) * kRowB;
          brow = G.b_row0 + r + plane * plane_rows;
        }
      }
      const uint32_t bytes = kQBytes + (uint32_t)C::kBTiles * G.t.N * kRowB;
      for (int ks = 0; ks < G.nk; ++ks, ++js) {
        const int s = js % C::kSlots;
        const uint32_t ph = (uint32_t)(js / C::kSlots) & 1u;
        bool ok = true;
        if (lane == 0) {
          ok = wait_phase(&S.sempty[s], ph ^ 1u, S, args.status);
          if (ok) {
            ptx::mbar_arrive_expect_tx(&S.sfull[s], bytes);
            armed[s] = (int)ph;
          }
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) {
          aborted = true;
          break;
        }
        uint8_t* st = smem + s * C::kSlotBytes;
        const int kb = G.shared ? (ks >> 1) : ks;  // 64-wide K block of this stage
        if (!G.shared) {
          if (lane < 2)
            ptx::tma_load_2d(st + lane * (kQBytes / 2), &tm_q, &S.sfull[s], kb * kBK8,
                             lane ? G.a_row1 : G.a_row0);
        } else if (lane == 0) {
          ptx::tma_load_2d(st, &tm_a_sh, &S.sfull[s], kb * kBK8, (ks & 1) ? G.a_row1 : G.a_row0);
        }
        if (bmap) ptx::tma_load_2d(st + boff, bmap, &S.sfull[s], kb * kBK8, brow);
      }
    }
    if (aborted && lane == 0) {
      for (int s = 0; s < C::kSlots; ++s)
        if (armed[s] >= 0) drain_phase(&S.sfull[s], (uint32_t)armed[s]);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int js = 0, ja = 0;
      Slots8 sl;
      bool aborted = false;
      const uint64_t dst0 = ptx::smem_desc_kmajor<128>(smem);   // staging slot 0
      const uint64_t dar0 = ptx::smem_desc_kmajor<128>(aring);  // operand slot 0
      for (int qi = 0; !aborted; ++qi) {
        const int slot = qi % kQueue8;
        if (!wait_phase(&S.q_full[slot], (uint32_t)(qi / kQueue8) & 1u, S, args.status)) {
          aborted = true;
          break;
        }
        const int tile = S.q[slot];
        ptx::mbar_arrive(&S.q_empty[slot]);
        if (tile < 0) break;
        const Geom8 G = geom8(args, S, tile, total, R);
        // bf16: columns [0, N) W h_hi, [N, 2N) W h_lo; fp16: columns [0, N) W h'
        const int cols = F16 ? G.t.N : 2 * G.t.N;
        const uint32_t idesc = F16 ? ptx::idesc_f16_f32(128, cols) : ptx::idesc_bf16_f32(128, cols);
        int first, count;
        sl.take(cols, first, count);
        for (int i = 0; i < count && !aborted; ++i) {
          const int sidx = (first + i) & 1;
          if (!wait_phase(&S.tmem_empty[sidx], (sl.uses[sidx] & 1u) ^ 1u, S, args.status))
            aborted = true;
        }
        if (aborted) break;
        ptx::tc_fence_after();
        const uint32_t d0 = tmem + first * kSlotCols8;
        const uint32_t d1 = d0 + (count == 2 ? kSlotCols8 : 128u);
        for (int ks = 0; ks < G.nk; ++ks, ++js) {
          const int s = js % C::kSlots;
          const uint32_t ph = (uint32_t)(js / C::kSlots) & 1u;
          if (!wait_phase(&S.sfull[s], ph, S, args.status)) {
            aborted = true;
            break;
          }
          const uint64_t sd = dst0 + (uint64_t)s * (C::kSlotBytes >> 4);
          const uint64_t bd = sd + (kQBytes >> 4);
          if (!G.shared) {
            const int c = ja & 1;
            const uint32_t pa = (uint32_t)(ja >> 1) & 1u;
            if (!wait_phase(&S.aready[c], pa, S, args.status)) {
              aborted = true;
              break;
            }
            ptx::tc_fence_after();
            const uint64_t ad = dar0 + (uint64_t)c * (C::kAStage >> 4);
            const uint32_t acc = ks > 0 ? 1u : 0u;
            ptx::umma_bf16_x4(d0, ad, bd, idesc, acc);
            ptx::umma_bf16_x4(d1, ad + (kAccBytes >> 4), bd, idesc, acc);
            ptx::umma_commit(&S.afree[c]);
            ++ja;
          } else {
            ptx::umma_bf16_x4((ks & 1) ? d1 : d0, sd, bd, idesc, ks >= 2 ? 1u : 0u);
          }
          ptx::umma_commit(&S.sempty[s]);
        }
        if (aborted) break;
        for (int i = 0; i < count; ++i) ptx::umma_commit(&S.tmem_full[(first + i) & 1]);
        sl.done(first, count);
      }
      if (aborted) {
        ptx::umma_commit(&S.drain);
        drain_phase(&S.drain, 0);
      }
    }
    __syncwarp();
  } else if (warp < 2 + kConvWarps) {
    // ------------------------------------------------------------ converters
    const int ct = threadIdx.x - 64;  // 0 .. 32 * kConvWarps - 1
    int js = 0, ja = 0;
    for (int qi = 0;; ++qi) {
      const int slot = qi % kQueue8;
      const bool got = wait_phase(&S.q_full[slot], (uint32_t)(qi / kQueue8) & 1u, S, args.status);
      if (!__all_sync(0xffffffffu, got)) break;
      const int tile = S.q[slot];
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&S.q_empty[slot]);
      if (tile < 0) break;
      const Geom8 G = geom8(args, S, tile, total, R);
      if (G.shared) {
        js += G.nk;  // 16-bit weights: nothing to widen
        continue;
      }
      bool ok = true;
      for (int ks = 0; ks < G.nk; ++ks, ++js, ++ja) {
        const int s = js % C::kSlots;
        const int c = ja & 1;
        ok = wait_phase(&S.sfull[s], (uint32_t)(js / C::kSlots) & 1u, S, args.status) &&
             wait_phase(&S.afree[c], ((uint32_t)(ja >> 1) & 1u) ^ 1u, S, args.status);
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
        const uint8_t* src = smem + s * C::kSlotBytes;
        uint8_t* dst = aring + c * C::kAStage;
        // 256 rows x 4 sixteen-byte chunks of codes; a warp's loads cover 512 consecutive
        // bytes, and its stores land in 8 rows whose swizzled chunks are all distinct
#pragma unroll 4
        for (int i = 0; i < (256 * 4) / (32 * kConvWarps); ++i) {
          const int q = i * (32 * kConvWarps) + ct;
          const int row = q >> 2, ch = q & 3;
          const uint4 v = *reinterpret_cast<const uint4*>(src + row * kQRowB + ch * 16);
          const uint4 o0 = make_uint4(widen8<F16, 0x9180>(v.x), widen8<F16, 0xB3A2>(v.x),
                                      widen8<F16, 0x9180>(v.y), widen8<F16, 0xB3A2>(v.y));
          const uint4 o1 = make_uint4(widen8<F16, 0x9180>(v.z), widen8<F16, 0xB3A2>(v.z),
                                      widen8<F16, 0x9180>(v.w), widen8<F16, 0xB3A2>(v.w));
          const int r = row & 127;
          uint8_t* base = dst + (row >> 7) * kAccBytes + r * kRowB;
          *reinterpret_cast<uint4*>(base + (((2 * ch) ^ (r & 7)) << 4)) = o0;
          *reinterpret_cast<uint4*>(base + (((2 * ch + 1) ^ (r & 7)) << 4)) = o1;
        }
        fence_proxy_async_smem();  // make the generic-proxy stores visible to the MMA
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&S.aready[c]);
      }
      if (!ok) break;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2 - kConvWarps;  // 0 .. kEpiWarps8 - 1
    const int qd = warp & 3;               // TMEM lanes 32*qd .. +31 (warp % 4 rule)
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
    constexpr int kChunks = Cfg8<F16>::kMaxTile / 32;
    Slots8 sl;
    for (int qi = 0;; ++qi) {
      const int slot = qi % kQueue8;
      const bool got = wait_phase(&S.q_full[slot], (uint32_t)(qi / kQueue8) & 1u, S, args.status);
      if (!__all_sync(0xffffffffu, got)) break;
      const int tile = S.q[slot];
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&S.q_empty[slot]);
      if (tile < 0) break;
      const Geom8 G = geom8(args, S, tile, total, R);
      const Tile& tl = G.t;
      int first, count;
      sl.take(F16 ? tl.N : 2 * tl.N, first, count);
      const uint32_t b0 = tmem + lane_off + first * kSlotCols8;
      const uint32_t b1 = b0 + (count == 2 ? kSlotCols8 : 128u);
      // row scales of this lane's two accumulator rows (1 for the bf16 shared expert), and
      // the token and routing weight of each column this warp stores
      float sc0 = 1.f, sc1 = 1.f;
      int col_tok[kChunks];
      float col_w[kChunks];
      if (!G.shared) {
        // fp16 operands: h' = h 2^-8, so the row scale takes the 2^8 back
        const float* s = a8.scale + (size_t)tl.g * args.H + tl.m * 256 + qd * 32 + lane;
        sc0 = __ldg(s) * (F16 ? 256.f : 1.f);
        sc1 = __ldg(s + 128) * (F16 ? 256.f : 1.f);
      }
#pragma unroll
      for (int ci = 0; ci < kChunks; ++ci) {
        const int c = ci * 32 + lane;
        col_tok[ci] = 0;
        col_w[ci] = 0.f;
        if (c < tl.nvalid) {
          const int p = tl.p0 + c;
          col_tok[ci] = token_of_row(args, p, R);
          if (args.out) col_w[ci] = p < R ? args.sorted_w[p] : args.sgate[col_tok[ci]];
        }
      }
      bool ok = true;
      for (int i = 0; i < count; ++i) {
        const int sidx = (first + i) & 1;
        ok = ok && wait_phase(&S.tmem_full[sidx], sl.uses[sidx] & 1u, S, args.status);
      }
      if (!__all_sync(0xffffffffu, ok)) break;
      ptx::tc_fence_after();
#pragma unroll
      for (int ci = 0; ci < kChunks; ++ci) {
        const int c0 = ci * 32;
        if (c0 >= tl.nvalid) break;
        uint32_t r0[32], r1[32];
        ptx::tmem_ld32(b0 + c0, r0);
        ptx::tmem_ld32(b1 + c0, r1);
        if (!F16) {
          // lo half of h in columns N + c0 (inside the accumulator's region: N <= 128)
          uint32_t l0[32], l1[32];
          ptx::tmem_ld32(b0 + tl.N + c0, l0);
          ptx::tmem_ld32(b1 + tl.N + c0, l1);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            r0[j] = __float_as_uint((__uint_as_float(r0[j]) + __uint_as_float(l0[j])) * sc0);
            r1[j] = __float_as_uint((__uint_as_float(r1[j]) + __uint_as_float(l1[j])) * sc1);
          }
        } else {
          ptx::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            r0[j] = __float_as_uint(__uint_as_float(r0[j]) * sc0);
            r1[j] = __float_as_uint(__uint_as_float(r1[j]) * sc1);
          }
        }
        {
          // 32 channels (lanes) x 32 tokens (registers) per accumulator, regrouped through
          // shared memory 8 tokens at a time so that each 16-byte atomic add of a warp
          // lands in whole 128-byte lines of one token's output row
          const int mrow = tl.m * 256 + qd * 32 + 4 * (lane & 7);
          const int H = args.H;
          float4(&xp)[8][8] = S.xpose[ew];
#pragma unroll
          for (int acc = 0; acc < 2; ++acc) {
            const uint32_t* r = acc ? r1 : r0;
#pragma unroll
            for (int sb = 0; sb < 4; ++sb) {
              __syncwarp();
              float* xs = reinterpret_cast<float*>(&xp[0][0]);
#pragma unroll
              for (int q = 0; q < 8; ++q) xs[q * 32 + lane] = __uint_as_float(r[sb * 8 + q]);
              __syncwarp();
#pragma unroll
              for (int hq = 0; hq < 2; ++hq) {
                const int q = hq * 4 + (lane >> 3);
                const float4 v = xp[q][lane & 7];
                const int col = c0 + sb * 8 + q;
                const int t = __shfl_sync(0xffffffffu, col_tok[ci], sb * 8 + q);
                const float w = __shfl_sync(0xffffffffu, col_w[ci], sb * 8 + q);
                if (col < tl.nvalid) {
                  const int p = tl.p0 + col;
                  const int m = mrow + acc * 128;
                  if (args.out) {
                    atomicAdd(reinterpret_cast<float4*>(args.out + (size_t)t * H + m),
                              make_float4(w * v.x, w * v.y, w * v.z, w * v.w));
                  } else {
                    float* row =
                        p < R ? args.y + (size_t)p * H : args.y_shared + (size_t)(p - R) * H;
                    *reinterpret_cast<float4*>(row + m) = v;
                  }
                }
              }
            }
          }
        }
      }
      ptx::tc_fence_before();
      for (int i = 0; i < count; ++i) ptx::mbar_arrive(&S.tmem_empty[(first + i) & 1]);
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
constexpr int kMaxTileQ = kTcChunkSmall;                    // 64 token rows per tile
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
    S.tp[g] = pv.tp1[g];
    S.row0[g] = pv.row0[g];
  }
  const int total = pv.tp1[E + 1];
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
            // SiLU(g) = g / (1 + e^-g), fast exponential and division (h carries 16 or,
            // for fp16 down operands, 11 significant bits)
            const float hv = __fdividef(gv, 1.f + __expf(-gv)) * __uint_as_float(r1[j]);
            const size_t at = (size_t)(tl.p0 + c0 + j) * args.ldh + ch;
            store_h(args.h, args.h_plane, at, hv, args.h_f16, args.status);
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

// ---------------------------------------------------------------- host side

// 2-D E4M3 tensor [outer][inner] (inner contiguous), boxes of 128 rows x 64 codes, no swizzle.
bool make_map_e4m3(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner};
  cuuint32_t box[2] = {(cuuint32_t)kBK8, 128};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

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
    if (!make_map(&b->m[i], base, inner, outer, kBK8, (uint32_t)(128 >> i))) return false;
  return true;
}

template <bool F16>
cudaError_t launch8_down(const CUtensorMap& q, const CUtensorMap& a_sh, const TokenMaps8& b,
                         const Tc8Args& args, cudaStream_t st) {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(tc8_down_kernel<F16>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)smem8_bytes<F16>());
  });
  if (attr_err != cudaSuccess) return attr_err;
  tc8_down_kernel<F16><<<sm_count(), kThreads8, smem8_bytes<F16>(), st>>>(q, a_sh, b, args);
  return cudaGetLastError();
}

}  // namespace

bool tc8_supported(const moe_shape& s) {
  return tc_supported(s) && (int64_t)s.T * s.k < 16 * (int64_t)s.E &&
         tc_gate_up_chunk(s.T, s.k, s.E) == kTcChunkSmall;
}

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
  args.a.h_f16 = w.ws_down_f16 ? 1 : 0;  // fp16 down operands: h as fp16(h 2^-8)
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
                            const moe_weights& w, const moe_fp8_experts& q, float* y,
                            float* y_shared, float* out, cudaStream_t st) {
  CUtensorMap qm, a_sh;
  TokenMaps8 b;
  const bool f16 = w.ws_down_f16 != nullptr;  // then the gate|up kernel stored h as fp16
  if (!make_map_e4m3(&qm, q.q_down, s.I, (uint64_t)s.E * s.H) ||
      !make_map(&a_sh, f16 ? w.ws_down_f16 : w.ws_down, s.Is, (uint64_t)s.H, kBK8, 128,
                f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) ||
      !make_token_maps8(&b, ws + L.h, L.ldh, 2 * (L.h_plane / L.ldh)))
    return cudaErrorInvalidValue;
  Tc8Args args{};
  args.a = base_args(s, L, ws);
  args.a.sorted_token = sorted_token;
  args.a.sorted_w = sorted_w;
  args.a.sgate = sgate;
  args.a.y = y;
  args.a.y_shared = y_shared;
  args.a.out = out;
  args.a.counter = reinterpret_cast<int*>(ws + L.sched) + 1;
  args.scale = q.s_down;
  LaunchScope scope(MOE_K_DOWN, st);
  return f16 ? launch8_down<true>(qm, a_sh, b, args, st) : launch8_down<false>(qm, a_sh, b, args, st);
}

}  // namespace moe
