// tc2_gemm.cu -- stage 4, "Grouped expert GEMMs" (Qwen3.8-Flash-Next architecture study,
// MoE pipeline diagram; expert(x) = W_down(SiLU(W_gate x) * W_up x)) on CTA pairs: one
// tcgen05.mma.cta_group::2 (M = 256) per 16-wide K step spans two SMs, each holding 128
// rows of the weight tile and HALF of the token tile in its own shared memory. Used for the
// down GEMM at every batch size and for the gate|up GEMM at prefill sizes.
//
// Why pairs: a pair halves each SM's share of the token operand and of the MMA issue work,
// and the down GEMM folds the hi and lo halves of h into the N dimension of one MMA, so its
// weight tile is read from shared memory once instead of twice. Measured on B200, this is
// faster than one CTA per tile for the down GEMM at every size and for gate|up from about
// 16 rows per expert. What paces both kernels is the single MMA-issuing thread: the tensor
// core queues only one or two MMAs, so the hand-off work between stages (barrier test,
// commit) is idle time for it. The issue loop is therefore kept minimal.
//
//   gate|up (pair tile: 128 channels x up to 256 tokens of one expert). CTA r holds gate rows
//     [c + 64r, c + 64r + 64) and the up rows of the same channels as its 128 A rows, and
//     token rows [N/2 r, N/2 (r + 1)) of the tile as its B half. Tensor-memory lanes 0-63
//     then hold gate and lanes 64-127 up for the same 64 channels; the epilogue pairs a
//     gate warp with an up warp through shared memory and stores h = SiLU(gate) * up as
//     the bf16 pair hi = bf16(h), lo = bf16(h - hi).
//   down (pair tile: 256 output channels x up to 128 packed rows). CTA r holds W_down rows
//     [m + 128r, m + 128r + 128) and plane r of h (r = 0: hi, r = 1: lo) for the tile's
//     rows, so the MMA's N = 2 x rows: columns [0, N) are W h_hi, [N, 2N) are W h_lo, and
//     the epilogue adds the two before scaling by the routing weight and adding into out.
//
// Roles in each 320-thread CTA (one CTA per SM, persistent; pair p takes tiles p, p + P,
// p + 2P, ... of the plan's order, so neighbouring tiles run at the same time):
//   warp 0      TMA producer over a ring of stages (6 of 32 KB holding 64 K, or 3 of 64 KB
//               holding 128 K: 128 A rows + up to 128 B rows each); both CTAs count their
//               copies on the leader's full barrier;
//   warp 1      tensor memory (512 columns, two 256-column slots, allocated for the pair);
//               in the leader CTA lane 0 issues the pair MMAs and commits them to both CTAs;
//   warps 2..9  epilogue; warp w reads TMEM lanes 32*(w%4) .. +31; the first four warps
//               take even 32-column chunks, the last four odd ones.
// Every mbarrier wait is bounded (2 s); on expiry the kernel records the timeout flag and
// every role leaves; the pair meets at a final cluster barrier before freeing TMEM.
#include <algorithm>

#include "tc_common.cuh"
#include "tc_gemm.h"

namespace moe {
namespace {

constexpr int kEpi = 8;
constexpr int kThreads2 = 64 + 32 * kEpi;
// A stage holds KSUB sub-tiles of 64 K of both operands (128-byte rows, 128-byte swizzle,
// the widest a TMA box may be). With KSUB = 2, eight MMAs share one hand-off (wait, commit)
// between the producer and the MMA issuer, which paid off on long K loops (hidden 8192;
// inter 2048) and cost on short ones (inter 640: 5 stages per tile), where KSUB = 1 keeps a
// 6-deep ring.
constexpr int kBK = 64;                   // K per sub-tile
constexpr uint32_t kRowB = kBK * 2;       // bytes per sub-tile row
constexpr uint32_t kASub = 128u * kRowB;  // 128 weight rows of one sub-tile: 16 KB
constexpr uint32_t kBSub = 128u * kRowB;  // up to 128 token rows of one sub-tile

template <int KSUB>
struct Ring {
  static constexpr int kStageK = kBK * KSUB;                   // K per stage
  static constexpr uint32_t kABytes = KSUB * kASub;            // this CTA's weight rows
  static constexpr uint32_t kBBytes = KSUB * kBSub;            // this CTA's token half
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;   // 32 or 64 KB
  static constexpr int kStages = KSUB == 1 ? 6 : 3;
};
constexpr int kMaxStages = 6;
constexpr int kSlotCols = 256;
// Each operand of a stage arrives in one TMA instruction (measured: an instruction costs
// the issuing thread ~90 cycles whatever its size, and the time from a freed stage to its
// last copy request lies on the pipeline's critical path). Weights: one 5-D (gate|up: K,
// channel row, gate/up, K block, expert) or 3-D (down: K, row, K block) box. Token rows:
// one 3-D box (K, row, K block) whose height is the CTA's row count rounded up to 16 (the
// rows past it are neighbours' or zero fill, and no MMA reads them): 8 tensor maps.
constexpr int kBHeights = 8;
__host__ __device__ constexpr int box_h(int i) { return 16 * (i + 1); }
__device__ __forceinline__ int box_index(int nb) { return (nb + 15) / 16 - 1; }

// kPairDownF16: the down GEMM on fp16 operands (W' = W * 2^8 from the weight pre-pass,
// h' = h * 2^-8 in plane 0): tiles of up to 256 rows, MMA N = rows, each CTA holding half of
// the tile's rows; one MMA per K step where the bf16 pair needs hi and lo columns.
enum PairMode { kPairGateUp = 0, kPairDown = 1, kPairDownF16 = 2 };

struct PairShared {
  uint64_t full[kMaxStages];   // leader: both CTAs' copies of a stage have landed
  uint64_t empty[kMaxStages];  // each CTA: the MMAs reading its copy of a stage are done
  uint64_t tmem_full[2];    // each CTA: the accumulator slot holds a finished tile
  uint64_t tmem_empty[2];   // leader: both CTAs' epilogues have drained the slot
  uint64_t drain;
  uint32_t tmem_base;
  volatile int abort;
  int tp[kMaxE + 2];
  int row0[kMaxE + 2];
  union {
    float4 xpose[kEpi][8][8];  // down: per warp, 8 tokens x 32 channels
    float up[4][32][32];       // gate|up: per warp pair, 32 tokens x 32 channels of up
  };
};

template <int KSUB>
constexpr size_t pair_smem_bytes() {
  return 1024 + (size_t)Ring<KSUB>::kStages * Ring<KSUB>::kStageBytes + sizeof(PairShared);
}
static_assert(pair_smem_bytes<1>() <= 232448 && pair_smem_bytes<2>() <= 232448,
              "over the 227 KB of shared memory a CTA may use");

struct PairMaps {
  CUtensorMap m[kBHeights];  // token boxes of 16, 32, ..., 128 rows
};

struct PairGeom {
  Tile t;
  int a_row0;          // gate|up: first of the 64 channels within the gate (and up) half;
                       // down: first of the 128 weight rows
  int a_e;             // gate|up: expert of the 5-D weight box (0 for the shared expert)
  int b_row;           // first row of this CTA's token half in its tensor map
  int nb;              // rows of this CTA's token half
  int nbb;             // rows of its token box (nb rounded up to 16)
  int n_mma;           // MMA N
  int nk;              // K stages
  bool shared;
};

template <int MODE, int KSUB>
__device__ __forceinline__ PairGeom pair_geom(const TcArgs& a, const PairShared& S, int tile,
                                              int R, int rank, int plane_rows) {
  constexpr int kStageK = Ring<KSUB>::kStageK;
  PairGeom G;
  G.t = decode_tile(S.row0, S.tp, a.E, tile,
                    MODE == kPairGateUp ? tc_gate_up_chunk(a.T, a.k, a.E)
                                        : (MODE == kPairDown ? kTcChunkDown : kTcChunkDownF16));
  G.shared = G.t.g == a.E;
  if (MODE == kPairGateUp) {
    G.a_row0 = G.t.m * 128 + rank * 64;
    G.a_e = G.shared ? 0 : G.t.g;
    G.nb = G.t.N / 2;
    G.b_row = (G.shared ? G.t.p0 - R : G.t.p0) + rank * G.nb;
    G.n_mma = G.t.N;
    G.nk = a.H / kStageK;
    G.nbb = (G.nb + 15) & ~15;
  } else if (MODE == kPairDown) {
    const int base = G.shared ? 0 : G.t.g * a.H;
    G.a_row0 = base + G.t.m * 256 + rank * 128;
    G.a_e = 0;
    G.nb = G.t.N;
    G.b_row = G.t.p0 + rank * plane_rows;
    G.n_mma = 2 * G.t.N;
    G.nk = (G.shared ? a.Is : a.I) / kStageK;
    G.nbb = (G.nb + 15) & ~15;
  } else {  // kPairDownF16: rows [0, N/2) of plane 0 in CTA 0, [N/2, N) in CTA 1
    const int base = G.shared ? 0 : G.t.g * a.H;
    G.a_row0 = base + G.t.m * 256 + rank * 128;
    G.a_e = 0;
    G.nb = G.t.N / 2;
    G.b_row = G.t.p0 + rank * G.nb;
    G.n_mma = G.t.N;
    G.nk = (G.shared ? a.Is : a.I) / kStageK;
    G.nbb = (G.nb + 15) & ~15;
  }
  return G;
}

template <int MODE, int KSUB>
__global__ void __launch_bounds__(kThreads2, 1)
tc2_grouped_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_a_sh,
                   const __grid_constant__ PairMaps tm_b, const __grid_constant__ PairMaps tm_b_sh,
                   const TcArgs args) {
  using RG = Ring<KSUB>;
  constexpr int kStages = RG::kStages, kStageK = RG::kStageK;
  constexpr uint32_t kABytes = RG::kABytes, kStageBytes = RG::kStageBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  PairShared& S = *reinterpret_cast<PairShared*>(smem + kStages * kStageBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = (int)ptx::cluster_ctarank();  // 0: the leader, which issues the MMAs
  const int pair = (int)ptx::cluster_id_x(), npairs = (int)ptx::cluster_count_x();
  const int E = args.E;
  const PlanView pv = plan_view(const_cast<int*>(args.plan), E);
  const int* tp = (MODE == kPairGateUp) ? pv.tp1 : (MODE == kPairDown ? pv.tp2 : pv.tp3);
  for (int g = threadIdx.x; g < E + 2; g += blockDim.x) {
    S.tp[g] = tp[g];
    S.row0[g] = pv.row0[g];
  }
  const int total = tp[E + 1];
  const int R = pv.row0[E];
  const int plane_rows = (MODE == kPairDown) ? (int)(args.h_plane / (size_t)args.ldh) : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(&S.full[s], 1);
      ptx::mbar_init(&S.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&S.tmem_full[b], 1);
      ptx::mbar_init(&S.tmem_empty[b], 2 * kEpi);  // one lane per epilogue warp of both CTAs
    }
    ptx::mbar_init(&S.drain, 1);
    S.abort = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tm_a);
    ptx::prefetch_tmap(&tm_a_sh);
    for (int i = 0; i < kBHeights; ++i) {
      ptx::prefetch_tmap(&tm_b.m[i]);
      ptx::prefetch_tmap(&tm_b_sh.m[i]);
    }
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(&S.tmem_base, 512);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();  // the peer's barriers exist before anyone signals them
  ptx::tc_fence_after();
  const uint32_t tmem = S.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    // Lane 0 waits for this CTA's copy of a stage to be free (and in the leader arms the
    // full barrier with both CTAs' bytes); then lane 0 issues the weight box and lane 1 the
    // box of this CTA's token rows, each covering all KSUB K blocks of the stage.
    const uint32_t full0 = ptx::mapa_shared(ptx::smem_u32(&S.full[0]), 0);
    const uint64_t evict_first = ptx::l2_policy_evict_first();
    int it = 0;
    bool aborted = false;
    for (int tile = pair; tile < total && !aborted; tile += npairs) {
      const PairGeom G = pair_geom<MODE, KSUB>(args, S, tile, R, rank, plane_rows);
      const CUtensorMap* a_map = G.shared ? &tm_a_sh : &tm_a;
      const CUtensorMap* b_map =
          &((MODE == kPairGateUp && G.shared) ? tm_b_sh : tm_b).m[box_index(G.nb)];
      const uint32_t bytes = 2u * KSUB * (kASub + (uint32_t)G.nbb * kRowB);  // both CTAs
      for (int ks = 0; ks < G.nk; ++ks, ++it) {
        const int s = it % kStages;
        const uint32_t ph = (uint32_t)(it / kStages) & 1u;
        bool ok = true;
        if (lane == 0) {
          ok = wait_phase(&S.empty[s], ph ^ 1u, S, args.status);
          if (ok && rank == 0) ptx::mbar_arrive_expect_tx(&S.full[s], bytes);
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) {
          aborted = true;
          break;
        }
        uint8_t* st = smem + s * kStageBytes;
        const uint32_t bar = full0 + (uint32_t)(s * sizeof(uint64_t));
        if (lane == 0) {
          if (MODE == kPairGateUp)  // [K block][gate, up][64 channels][64 K]
            ptx::tma_load_5d_pair(st, a_map, bar, 0, G.a_row0, 0, ks * KSUB, G.a_e);
          else if (G.shared)  // [K block][128 rows][64 K]; re-read by every token chunk
            ptx::tma_load_3d_pair(st, a_map, bar, 0, G.a_row0, ks * KSUB);
          else  // routed weights are read once: evicted first, so out rows and h stay in L2
            ptx::tma_load_3d_pair_hint(st, a_map, bar, 0, G.a_row0, ks * KSUB, evict_first);
        } else if (lane == 1) {  // [K block][nbb token rows][64 K]
          ptx::tma_load_3d_pair(st + kABytes, b_map, bar, 0, G.b_row, ks * KSUB);
        }
      }
    }
    // wait until the MMAs have released every stage this CTA filled, so that no commit
    // from the leader is still on its way to this CTA's barriers when the pair leaves
    if (lane == 0 && !aborted) {
      for (int j = 0; j < kStages && j < it; ++j) {
        const int u = it - 1 - j;
        if (!wait_phase(&S.empty[u % kStages], (uint32_t)(u / kStages) & 1u, S, args.status))
          break;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ pair MMA issuer (leader)
    if (rank == 0 && lane == 0) {
      // Kept short on purpose: the tensor core takes an MMA only about when it can start
      // it, so every instruction between a stage's MMAs and the next stage's is idle time
      // for it (running ring position instead of division, one asm block per stage).
      int s = 0, nt = 0;
      uint32_t ph = 0;
      bool aborted = false;
      const uint64_t desc0 = ptx::smem_desc_kmajor<kRowB>(smem);  // stage 0, A operand
      // readiness of the next stage, tested while the current stage's MMAs are queued
      bool ready = ptx::mbar_test_wait(&S.full[0], 0);
      for (int tile = pair; tile < total && !aborted; tile += npairs, ++nt) {
        const PairGeom G = pair_geom<MODE, KSUB>(args, S, tile, R, rank, plane_rows);
        const int slot = nt & 1;
        const uint32_t use = (uint32_t)(nt >> 1);
        if (!wait_phase(&S.tmem_empty[slot], (use & 1u) ^ 1u, S, args.status)) {
          aborted = true;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(slot * kSlotCols);
        const uint32_t idesc = MODE == kPairDownF16 ? ptx::idesc_f16_f32(256, G.n_mma)
                                                    : ptx::idesc_bf16_f32(256, G.n_mma);
        for (int ks = 0; ks < G.nk; ++ks) {
          // The copies' completion on the full barrier orders them before the MMAs that
          // read the stage; no tcgen05 fence is needed here.
          if (!ready && !wait_phase(&S.full[s], ph, S, args.status)) {
            aborted = true;
            break;
          }
          const int s2 = (s + 1 == kStages) ? 0 : s + 1;
          const uint32_t ph2 = (s2 == 0) ? (ph ^ 1u) : ph;
          const uint64_t ad = desc0 + (uint64_t)s * (kStageBytes >> 4);
          const uint64_t bd = ad + (kABytes >> 4);
          if (KSUB == 2) {
            ptx::umma_bf16_pair_x4(d, ad, bd, idesc, ks > 0 ? 1u : 0u);
            ready = ptx::mbar_test_wait(&S.full[s2], ph2);
            ptx::umma_bf16_pair_x4(d, ad + (kASub >> 4), bd + ((G.nbb * kRowB) >> 4), idesc, 1u);
          } else {
            ptx::umma_bf16_pair_x2(d, ad, bd, idesc, ks > 0 ? 1u : 0u);
            ready = ptx::mbar_test_wait(&S.full[s2], ph2);
            ptx::umma_bf16_pair_x2(d, ad + 4, bd + 4, idesc, 1u);
          }
          ptx::umma_commit_pair(&S.empty[s], 0x3);
          s = s2;
          ph = ph2;
        }
        if (aborted) break;
        ptx::umma_commit_pair(&S.tmem_full[slot], 0x3);
      }
      if (aborted) {
        ptx::umma_commit_pair(&S.drain, 0x1);  // completes once every MMA issued so far is done
        drain_phase(&S.drain, 0);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;  // which 32-column chunks this warp drains
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const uint32_t tmem_empty0 = ptx::mapa_shared(ptx::smem_u32(&S.tmem_empty[0]), 0);
    // out rows take k + 1 atomic adds each, from experts far apart in the tile order: keep
    // their lines in L2 (evicted last) rather than fetch them from DRAM for every add
    const uint64_t keep = ptx::l2_policy_evict_last();
    // gate|up: warps q = 0, 1 hold gate and q = 2, 3 up of the same 32 channels
    const int xp = half * 2 + (q & 1);  // warp pair index, 0..3
    // named barriers of the pair: its per-tile decision, "buffer free", "buffer full"
    const int bar_dec = 1 + 3 * xp, bar_free = 2 + 3 * xp, bar_full = 3 + 3 * xp;
    int nt = 0;
    for (int tile = pair; tile < total; tile += npairs, ++nt) {
      const PairGeom G = pair_geom<MODE, KSUB>(args, S, tile, R, rank, plane_rows);
      const Tile& tl = G.t;
      const int slot = nt & 1;
      const uint32_t use = (uint32_t)(nt >> 1);
      const uint32_t base = tmem + lane_off + (uint32_t)(slot * kSlotCols);
      // down: token and weight of this warp's columns, requested before waiting for the
      // accumulator so that the loads overlap the tile's MMAs
      // down: 32-column chunks per warp half (N <= 128 with the bf16 pair, <= 256 with fp16)
      constexpr int kDownChunks = MODE == kPairDownF16 ? 4 : 2;
      int col_tok[kDownChunks];
      float col_w[kDownChunks];
#pragma unroll
      for (int ci = 0; ci < kDownChunks; ++ci) {
        col_tok[ci] = 0;
        col_w[ci] = 0.f;
      }
      if (MODE != kPairGateUp) {
#pragma unroll
        for (int ci = 0; ci < kDownChunks; ++ci) {
          const int c = (2 * ci + half) * 32 + lane;
          if (c < tl.nvalid) {
            const int p = tl.p0 + c;
            col_tok[ci] = token_of_row(args, p, R);
            if (args.out) col_w[ci] = p < R ? args.sorted_w[p] : args.sgate[col_tok[ci]];
          }
        }
      }
      bool ok = wait_phase(&S.tmem_full[slot], use & 1u, S, args.status);
      // the gate and up warps of a pair decide together (they meet at named barriers below)
      ok = (MODE == kPairGateUp) ? ptx::bar_and(bar_dec, 64, ok) : __all_sync(0xffffffffu, ok);
      if (!ok) break;
      ptx::tc_fence_after();
      if (MODE == kPairGateUp) {
        const int ch = tl.m * 128 + rank * 64 + (q & 1) * 32 + lane;  // this lane's channel
        float(&xu)[32][32] = S.up[xp];
#pragma unroll 1
        for (int ci = 0; ci < 4; ++ci) {
          const int c0 = (2 * ci + half) * 32;
          if (c0 >= tl.nvalid) break;
          uint32_t r[32];
          ptx::tmem_ld32(base + (uint32_t)c0, r);
          ptx::tmem_ld_wait();
          if (q >= 2) {  // up warp: hand its 32 x 32 values to the gate warp
            ptx::bar_sync(bar_free, 64);
#pragma unroll
            for (int j = 0; j < 32; ++j) xu[j][lane] = __uint_as_float(r[j]);
            ptx::bar_arrive(bar_full, 64);
          } else {
            ptx::bar_arrive(bar_free, 64);
            ptx::bar_sync(bar_full, 64);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (c0 + j < tl.nvalid) {
                const float gv = __uint_as_float(r[j]);
                // SiLU(g) = g / (1 + e^-g) with the fast exponential and division (a few
                // ulp; h is carried with 16 or, for fp16 down operands, 11 significant bits)
                const float hv = __fdividef(gv, 1.f + __expf(-gv)) * xu[j][lane];
                const size_t at = (size_t)(tl.p0 + c0 + j) * args.ldh + ch;
                store_h(args.h, args.h_plane, at, hv, args.h_f16, args.status);
              }
            }
          }
        }
      } else {
        // bf16 pair: columns [0, N) hold W h_hi and [N, 2N) W h_lo of the same rows;
        // fp16 operands: columns [0, N) hold W h
        const int mrow = tl.m * 256 + rank * 128 + q * 32 + 4 * (lane & 7);  // this lane's channels
        const int H = args.H;
        float4(&xpz)[8][8] = S.xpose[warp - 2];
#pragma unroll
        for (int ci = 0; ci < kDownChunks; ++ci) {
          const int c0 = (2 * ci + half) * 32;
          if (c0 >= tl.nvalid) break;
          uint32_t r0[32], r1[32];
          ptx::tmem_ld32(base + (uint32_t)c0, r0);
          if (MODE == kPairDown) {
            ptx::tmem_ld32(base + (uint32_t)(tl.N + c0), r1);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) r1[j] = 0u;  // +0.0f
          }
          ptx::tmem_ld_wait();
          // 32 channels (lanes) x 32 tokens (registers); every 8 tokens go through shared
          // memory so that eight lanes own the 32 channels (128 bytes) of one token and each
          // 16-byte atomic add of a warp lands in whole 128-byte lines
#pragma unroll
          for (int sb = 0; sb < 4; ++sb) {
            __syncwarp();
            float* xs = reinterpret_cast<float*>(&xpz[0][0]);
#pragma unroll
            for (int k = 0; k < 8; ++k)
              xs[k * 32 + lane] = __uint_as_float(r0[sb * 8 + k]) + __uint_as_float(r1[sb * 8 + k]);
            __syncwarp();
#pragma unroll
            for (int hq = 0; hq < 2; ++hq) {
              const int k = hq * 4 + (lane >> 3);  // this lane's token within the 8
              const float4 v = xpz[k][lane & 7];
              const int col = c0 + sb * 8 + k;
              const int t = __shfl_sync(0xffffffffu, col_tok[ci], sb * 8 + k);
              const float w = __shfl_sync(0xffffffffu, col_w[ci], sb * 8 + k);
              if (col < tl.nvalid) {
                const int p = tl.p0 + col;
                if (args.out) {
                  ptx::red_add_v4_f32_hint(args.out + (size_t)t * H + mrow,
                                           make_float4(w * v.x, w * v.y, w * v.z, w * v.w), keep);
                } else {
                  float* row =
                      p < R ? args.y + (size_t)p * H : args.y_shared + (size_t)(p - R) * H;
                  *reinterpret_cast<float4*>(row + mrow) = v;
                }
              }
            }
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive_cluster(tmem_empty0 + (uint32_t)(slot * sizeof(uint64_t)));
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (S.abort) {
    // copies or commits aimed at the pair's barriers may still be in flight: give them time
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 2000000ull) {
    }
  }
  ptx::cluster_sync();  // neither CTA frees TMEM or leaves while its peer may signal it
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem, 512);
  }
}

// ---------------------------------------------------------------- host side

// Token rows [rows][ld] (2-byte elements) as 3-D boxes {64 K, h rows, KSUB K blocks} for the
// eight box heights.
template <int KSUB>
bool make_token_maps(PairMaps* b, const void* base, uint64_t ld, uint64_t rows,
                     CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  const uint64_t dims[3] = {(uint64_t)kBK, rows, ld / kBK};
  const uint64_t strides[2] = {ld * 2, kRowB};
  for (int i = 0; i < kBHeights; ++i) {
    const uint32_t box[3] = {(uint32_t)kBK, (uint32_t)box_h(i), (uint32_t)KSUB};
    if (!make_map_nd(&b->m[i], base, 3, dims, strides, box, dt)) return false;
  }
  return true;
}

// Gate|up weights [E][2I][H] as 5-D boxes {64 K, 64 channels, gate and up, KSUB K blocks, 1}.
bool make_gate_up_map(CUtensorMap* m, const void* base, uint64_t E, uint64_t I, uint64_t H) {
  const uint64_t dims[5] = {(uint64_t)kBK, I, 2, H / kBK, E};
  const uint64_t strides[4] = {H * 2, I * H * 2, kRowB, 2 * I * H * 2};
  const uint32_t box[5] = {(uint32_t)kBK, 64, 2, 2, 1};
  return make_map_nd(m, base, 5, dims, strides, box);
}

// Down weights [rows][I] as 3-D boxes {64 K, 128 rows, KSUB K blocks}.
template <int KSUB>
bool make_down_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t I,
                   CUtensorMapDataType dt) {
  const uint64_t dims[3] = {(uint64_t)kBK, rows, I / kBK};
  const uint64_t strides[2] = {I * 2, kRowB};
  const uint32_t box[3] = {(uint32_t)kBK, 128, (uint32_t)KSUB};
  return make_map_nd(m, base, 3, dims, strides, box, dt);
}

template <int MODE, int KSUB>
cudaError_t launch_pair(const CUtensorMap& a, const CUtensorMap& a_sh, const PairMaps& b,
                        const PairMaps& b_sh, const TcArgs& args, cudaStream_t st) {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  static int max_pairs = 0;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(tc2_grouped_kernel<MODE, KSUB>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)pair_smem_bytes<KSUB>());
    if (attr_err != cudaSuccess) return;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * (unsigned)sm_count(), 1, 1);
    cfg.blockDim = dim3(kThreads2, 1, 1);
    cfg.dynamicSmemBytes = pair_smem_bytes<KSUB>();
    cfg.attrs = at;
    cfg.numAttrs = 1;
    attr_err = cudaOccupancyMaxActiveClusters(&max_pairs, tc2_grouped_kernel<MODE, KSUB>, &cfg);
    if (attr_err == cudaSuccess && max_pairs < 1) attr_err = cudaErrorInvalidConfiguration;
  });
  if (attr_err != cudaSuccess) return attr_err;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2 * (unsigned)max_pairs, 1, 1);
  cfg.blockDim = dim3(kThreads2, 1, 1);
  cfg.dynamicSmemBytes = pair_smem_bytes<KSUB>();
  cfg.stream = st;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, tc2_grouped_kernel<MODE, KSUB>, a, a_sh, b, b_sh, args);
}

}  // namespace

cudaError_t launch_tc2_gate_up(const moe_shape& s, const Layout& L, char* ws, const uint16_t* x,
                               const int32_t* sorted_token, const moe_weights& w, int h_f16,
                               cudaStream_t st) {
  uint16_t* xs = reinterpret_cast<uint16_t*>(ws + L.xs);
  cudaError_t e = launch_gather_rows(s, L, ws, x, sorted_token, st);
  if (e != cudaSuccess) return e;
  CUtensorMap a, a_sh;
  PairMaps b, b_sh;
  if (!make_gate_up_map(&a, w.w_gate_up, s.E, s.I, s.H) ||
      !make_gate_up_map(&a_sh, w.ws_gate_up, 1, s.Is, s.H) ||
      !make_token_maps<2>(&b, xs, s.H, (uint64_t)s.T * s.k) ||
      !make_token_maps<2>(&b_sh, x, s.H, (uint64_t)s.T))
    return cudaErrorInvalidValue;
  TcArgs args = base_args(s, L, ws);
  args.sorted_token = sorted_token;
  args.h_f16 = h_f16;
  LaunchScope scope(MOE_K_GATE_UP, st);
  return launch_pair<kPairGateUp, 2>(a, a_sh, b, b_sh, args, st);
}

template <int MODE, int KSUB>
cudaError_t launch_down_mode(const moe_shape& s, const Layout& L, char* ws, const void* wd,
                             const void* wsd, CUtensorMapDataType dt, const TcArgs& args,
                             cudaStream_t st) {
  CUtensorMap a, a_sh;
  PairMaps b;
  const uint64_t rows = (MODE == kPairDown ? 2 : 1) * (L.h_plane / L.ldh);  // h planes used
  if (!make_down_map<KSUB>(&a, wd, (uint64_t)s.E * s.H, s.I, dt) ||
      !make_down_map<KSUB>(&a_sh, wsd, (uint64_t)s.H, s.Is, dt) ||
      !make_token_maps<KSUB>(&b, ws + L.h, L.ldh, rows, dt))
    return cudaErrorInvalidValue;
  return launch_pair<MODE, KSUB>(a, a_sh, b, b, args, st);
}

TcArgs down_args(const moe_shape& s, const Layout& L, char* ws, const int32_t* sorted_token,
                 const float* sorted_w, const float* sgate, float* y, float* y_shared, float* out) {
  TcArgs args = base_args(s, L, ws);
  args.sorted_token = sorted_token;
  args.sorted_w = sorted_w;
  args.sgate = sgate;
  args.y = y;
  args.y_shared = y_shared;
  args.out = out;
  return args;
}

cudaError_t launch_tc2_down(const moe_shape& s, const Layout& L, char* ws,
                            const int32_t* sorted_token, const float* sorted_w, const float* sgate,
                            const moe_weights& w, float* y, float* y_shared, float* out,
                            cudaStream_t st) {
  const TcArgs args = down_args(s, L, ws, sorted_token, sorted_w, sgate, y, y_shared, out);
  LaunchScope scope(MOE_K_DOWN, st);
  // 128-K stages (eight MMAs per producer/issuer hand-off) for long down loops (I >= 1024)
  // and for decode-size batches, whose tiny MMAs (N = 2 x a few rows) leave the issuing
  // thread as the bound with the copies landing far ahead; 64-K stages and a 6-deep ring
  // for short loops at prefill sizes (inter 640: 5 stages per tile)
  const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if ((s.I >= 1024 && s.Is >= 1024) || (int64_t)s.T * s.k < 16 * (int64_t)s.E)
    return launch_down_mode<kPairDown, 2>(s, L, ws, w.w_down, w.ws_down, bf, args, st);
  return launch_down_mode<kPairDown, 1>(s, L, ws, w.w_down, w.ws_down, bf, args, st);
}

cudaError_t launch_tc2_down_f16(const moe_shape& s, const Layout& L, char* ws,
                                const int32_t* sorted_token, const float* sorted_w,
                                const float* sgate, const moe_weights& w, float* y,
                                float* y_shared, float* out, cudaStream_t st) {
  const TcArgs args = down_args(s, L, ws, sorted_token, sorted_w, sgate, y, y_shared, out);
  LaunchScope scope(MOE_K_DOWN, st);
  return launch_down_mode<kPairDownF16, 2>(s, L, ws, w.w_down_f16, w.ws_down_f16,
                                           CU_TENSOR_MAP_DATA_TYPE_FLOAT16, args, st);
}

}  // namespace moe
