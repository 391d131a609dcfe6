// tc_gemm.cu -- stage 4, "Grouped expert GEMMs" (Qwen3.8-Flash-Next architecture study,
// MoE pipeline diagram; expert(x) = W_down(SiLU(W_gate x) * W_up x)), and the router GEMM
// of stage 1, on the 5th-generation tensor cores: TMA-fed shared-memory ring,
// tcgen05.mma with fp32 accumulators in tensor memory, fused epilogues.
//
// Orientation ("swap AB"): weight rows are the MMA's M side (two 128-row accumulators per
// tile = 256 weight rows sharing one token tile), the tokens of one expert are the N side
// (multiples of 16; up to 256 per gate|up tile, so a prefill expert is one tile and its
// gate|up weights pass through shared memory once; up to 128 per down and router tile),
// K is the hidden (gate|up, router) or intermediate (down) dimension.
//
//   gate|up: gate rows [c, c+128) and up rows [I+c, I+c+128) of one expert against its
//     token rows, copied beforehand in dispatch order (gather_rows_kernel) so that a token
//     tile is a few plain 2-D TMA boxes. Epilogue: h = SiLU(gate) * up stored as the bf16
//     pair hi = bf16(h), lo = bf16(h - hi).
//   down: 256 rows of one expert's W_down against its packed rows. The tile's h_lo rows
//     follow its h_hi rows in shared memory, so one MMA per accumulator with N = 2 x rows
//     yields W h_hi in columns [0, N) and W h_lo in [N, 2N), added in the epilogue (half
//     the MMA instructions of two N-wide MMAs; at decode sizes the issuing thread is the
//     bound). Epilogue: y rows (staged path) or routing-weight-scaled fp32 atomic adds
//     into out[token] ("Weighted combine + gated shared expert").
//   router: 256 experts x 128 tokens of logits = x . (hi + mid + lo)^T, K = 3H over the
//     exact bf16 split of the fp32 router matrix.
//
// Roles in a 320-thread CTA (one CTA per SM, persistent; tiles handed out in order by an
// atomic counter through a shared-memory queue):
//   warp 0      TMA producer over a ring of kStages stages (lane 0 takes tiles and arms
//               the barriers; each box of a stage is issued by its own lane);
//   warp 1      TMEM owner (all 512 columns, two slots of 256) and MMA issuer (lane 0);
//               a tile of at most 128 tokens takes one slot (its two accumulators are
//               128 columns each) and the next tile's MMAs fill the other slot while the
//               epilogue drains it; a larger tile takes both slots;
//   warps 2..9  epilogue; warp w reads TMEM lanes 32*(w%4) .. +31, the first four warps
//               even 32-column chunks, the last four odd ones.
// Every mbarrier wait is bounded (2 s); on expiry the kernel records the timeout flag,
// lets every role leave its loop, drains its own copies and MMAs and frees TMEM.
#include <algorithm>

#include "tc_common.cuh"
#include "tc_gemm.h"

namespace moe {
namespace {

constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
// A token tile of N rows (a multiple of 16) is loaded as at most five TMA boxes of 128, 64,
// 32 or 16 rows (128-row boxes first, then the binary digits of the rest): a TMA
// instruction costs about as much as moving 60-70 rows, so sixteen-row boxes alone made
// the token loads the slowest part of a prefill stage.
constexpr int kBoxHeights = 4;
__host__ __device__ constexpr int box_rows_of(int i) { return 128 >> i; }
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSlotCols = 256;
constexpr int kQueue = 4;  // tile ids handed from the producer to the MMA and epilogue roles

// kGateUpSmall: the gate|up GEMM for decode-size batches (T*k < 16*E), whose tiles are
// chunked at 64 token rows: its stages reserve room for 64 rows instead of 256, so five of
// them fit and about 170 KB of weights are in flight per SM instead of about 100 KB.
enum Mode { kGateUp = 0, kDown = 1, kRouter = 2, kGateUpSmall = 3 };
__host__ __device__ constexpr bool is_gate_up(int mode) {
  return mode == kGateUp || mode == kGateUpSmall;
}

// Per-mode pipeline geometry. The down GEMM keeps tiles of at most 128 tokens: its K loop
// is short (K = I), so its epilogue must overlap the next tile's MMAs (one TMEM slot per
// tile); a 256-token down tile measured 1.36x slower on the Flash-Next prefill layer.
template <int MODE>
struct Cfg {
  static constexpr int kBK = 64;                                  // K per stage
  static constexpr int kRowBytes = kBK * 2;                       // 128 (= swizzle)
  static constexpr int kMaxTile =  // tokens per tile
      MODE == kGateUp ? kTcChunk : (MODE == kGateUpSmall ? kTcChunkSmall : 128);
  static constexpr uint32_t kATileBytes = 128u * kRowBytes;
  static constexpr uint32_t kBTileBytes = (uint32_t)kMaxTile * kRowBytes;
  static constexpr int kBTiles = (MODE == kDown) ? 2 : 1;  // down: hi and lo rows of h
  static constexpr uint32_t kStageBytes = 2 * kATileBytes + kBTiles * kBTileBytes;
  static constexpr int kStages = MODE == kGateUpSmall ? 5 : 3;
  static constexpr int kKK = kBK / 16;  // MMAs (K = 16) per stage and accumulator
};

struct SharedState {
  uint64_t full[5];
  uint64_t empty[5];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t q_full[kQueue];
  uint64_t q_empty[kQueue];
  uint64_t drain;
  uint32_t tmem_base;
  volatile int abort;
  int q[kQueue];
  int tp[kMaxE + 2];    // tile prefix of the grouped GEMM (copied from the plan)
  int row0[kMaxE + 2];  // first packed row of each group (copied from the plan)
  float4 xpose[kEpiWarps][8][8];  // down epilogue: per warp, 8 tokens x 32 channels
};

template <int MODE>
constexpr size_t smem_bytes() {
  return 1024 + (size_t)Cfg<MODE>::kStages * Cfg<MODE>::kStageBytes + sizeof(SharedState);
}
static_assert(smem_bytes<kGateUp>() <= 232448 && smem_bytes<kDown>() <= 232448 &&
                  smem_bytes<kRouter>() <= 232448 && smem_bytes<kGateUpSmall>() <= 232448,
              "over the 227 KB of shared memory a CTA may use");

// The token operand's tensor map in each box height (index i: 128 >> i rows).
struct BMaps {
  CUtensorMap m[kBoxHeights];
};

// Piece `j` of an N-row token tile: its first row and box-height index; false past the
// last piece.
__device__ __forceinline__ bool token_piece(int N, int j, int& row, int& hidx) {
  const int n128 = N >> 7;
  if (j < n128) {
    row = j * 128;
    hidx = 0;
    return true;
  }
  j -= n128;
  int r = n128 * 128;
#pragma unroll
  for (int h = 1; h < kBoxHeights; ++h) {
    if (N & box_rows_of(h)) {
      if (j == 0) {
        row = r;
        hidx = h;
        return true;
      }
      --j;
      r += box_rows_of(h);
    }
  }
  return false;
}

// Everything the three roles need to know about one tile.
struct Geom {
  Tile t;
  int a_row0, a_row1;  // A-operand rows of the two accumulators
  int b_row0;          // first row of the token tile in its tensor map
  int nk;              // K stages
  bool shared;         // shared-expert group (its own weight / token tensor maps)
};

template <int MODE>
__device__ __forceinline__ Geom tile_geom(const TcArgs& a, const SharedState& S, int tile,
                                          int R) {
  using C = Cfg<MODE>;
  Geom G;
  if (MODE == kRouter) {
    const int mt = (a.E + 255) / 256;
    const int m = tile % mt, c = tile / mt;
    G.t.g = 0;
    G.t.m = m;
    G.t.p0 = c * C::kMaxTile;
    G.t.nvalid = min(C::kMaxTile, a.T - G.t.p0);
    G.t.N = (G.t.nvalid + 15) & ~15;
    G.a_row0 = m * 256;
    G.a_row1 = m * 256 + 128;
    G.b_row0 = G.t.p0;
    G.nk = 3 * a.H / C::kBK;
    G.shared = false;
    return G;
  }
  G.t = decode_tile(S.row0, S.tp, a.E, tile, C::kMaxTile);
  G.shared = G.t.g == a.E;
  if (is_gate_up(MODE)) {
    const int Ig = G.shared ? a.Is : a.I;
    const int base = G.shared ? 0 : G.t.g * 2 * a.I;
    G.a_row0 = base + G.t.m * 128;
    G.a_row1 = base + Ig + G.t.m * 128;
    G.b_row0 = G.shared ? G.t.p0 - R : G.t.p0;  // x rows for the shared expert
    G.nk = a.H / C::kBK;
  } else {
    const int base = G.shared ? 0 : G.t.g * a.H;
    G.a_row0 = base + G.t.m * 256;
    G.a_row1 = G.a_row0 + 128;
    G.b_row0 = G.t.p0;
    G.nk = (G.shared ? a.Is : a.I) / C::kBK;
  }
  return G;
}

// TMEM slot bookkeeping shared by the MMA issuer and the epilogue (both walk the same tile
// sequence): a tile of at most 128 tokens takes the next slot, a larger one both slots.
struct Slots {
  int next = 0;
  uint32_t uses[2] = {0u, 0u};
  // cols: TMEM columns one accumulator of the tile needs (N; 2N for the down GEMM, whose
  // hi and lo halves of h share one MMA)
  __device__ __forceinline__ void take(int cols, int& first, int& count) const {
    count = cols > 128 ? 2 : 1;
    first = count == 2 ? 0 : next;
  }
  __device__ __forceinline__ void done(int first, int count) {
    for (int i = 0; i < count; ++i) uses[(first + i) & 1]++;
    next = count == 2 ? 0 : (first ^ 1);
  }
};

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
tc_grouped_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_a_sh,
                  const __grid_constant__ BMaps tm_b, const __grid_constant__ BMaps tm_b_sh,
                  const TcArgs args) {
  using C = Cfg<MODE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  SharedState& S = *reinterpret_cast<SharedState*>(smem + C::kStages * C::kStageBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = args.E;
  int total, R = 0;
  if (MODE == kRouter) {
    total = args.ntiles;
  } else {
    // the plan is read on every tile by every role: keep it in shared memory
    const PlanView pv = plan_view(const_cast<int*>(args.plan), E);
    const int* tp = (is_gate_up(MODE)) ? pv.tp1 : pv.tp2;
    for (int g = threadIdx.x; g < E + 2; g += blockDim.x) {
      S.tp[g] = tp[g];
      S.row0[g] = pv.row0[g];
    }
    total = tp[E + 1];
    R = pv.row0[E];
  }

  if (is_gate_up(MODE) && blockIdx.x == 0 && threadIdx.x == 0) *args.counter_next = 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      ptx::mbar_init(&S.full[s], 1);
      ptx::mbar_init(&S.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&S.tmem_full[b], 1);
      ptx::mbar_init(&S.tmem_empty[b], 32 * kEpiWarps);
    }
    for (int i = 0; i < kQueue; ++i) {
      ptx::mbar_init(&S.q_full[i], 1);
      ptx::mbar_init(&S.q_empty[i], 1 + kEpiWarps);  // the MMA lane, one lane per epilogue warp
    }
    ptx::mbar_init(&S.drain, 1);
    S.abort = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tm_a);
    ptx::prefetch_tmap(&tm_a_sh);
    for (int i = 0; i < kBoxHeights; ++i) {
      ptx::prefetch_tmap(&tm_b.m[i]);
      ptx::prefetch_tmap(&tm_b_sh.m[i]);
    }
  }
  if (warp == 1) {
    ptx::tmem_alloc(&S.tmem_base, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = S.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // Lane 0 takes tiles, waits for free stages and arms the full barriers; then every
    // lane with a box of the stage issues it (lanes 0-1: the two weight boxes, lanes 2..:
    // the token pieces, hi plane then lo plane for down), so the copies start together.
    int it = 0;
    int armed[C::kStages];
#pragma unroll
    for (int s = 0; s < C::kStages; ++s) armed[s] = -1;
    bool aborted = false;
    const int plane_rows = (MODE == kDown) ? (int)(args.h_plane / (size_t)args.ldh) : 0;
    // tiles are handed out in order by one counter: neighbouring tiles (the chunks of one
    // weight tile, the M tiles of one expert) run at the same time on neighbouring SMs.
    // Lane 0 asks for the next tile one tile ahead, so the counter's round trip to L2 hides
    // behind the current tile's copies instead of stalling them (short decode tiles paid
    // it once per tile).
    int ahead = (lane == 0) ? atomicAdd(args.counter, 1) : 0;
    for (int qi = 0; !aborted; ++qi) {
      const int slot = qi % kQueue;
      int tile = 0;
      if (lane == 0) {
        if (!wait_phase(&S.q_empty[slot], ((uint32_t)(qi / kQueue) & 1u) ^ 1u, S, args.status)) {
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
      const Geom G = tile_geom<MODE>(args, S, tile, R);
      // this lane's box: weight rows (lanes 0, 1) or one token piece of one plane
      const CUtensorMap* my_map = nullptr;
      uint32_t my_off = 0;
      int my_row = 0;
      if (lane < 2) {
        my_map = G.shared ? &tm_a_sh : &tm_a;
        my_off = lane * C::kATileBytes;
        my_row = lane ? G.a_row1 : G.a_row0;
      } else {
        int np = 0, r, h;
        while (token_piece(G.t.N, np, r, h)) ++np;
        const int j = lane - 2;
        if (j < np * C::kBTiles) {
          const int plane = j / np;
          token_piece(G.t.N, j - plane * np, r, h);
          const BMaps& bm = (is_gate_up(MODE) && G.shared) ? tm_b_sh : tm_b;
          my_map = &bm.m[h];
          // down: the lo rows follow the hi rows, so one MMA with N = 2 x rows reads both
          my_off = 2 * C::kATileBytes + (uint32_t)(plane * G.t.N + r) * C::kRowBytes;
          my_row = G.b_row0 + r + plane * plane_rows;
        }
      }
      const uint32_t bytes = 2 * C::kATileBytes + (uint32_t)C::kBTiles * G.t.N * C::kRowBytes;
      for (int ks = 0; ks < G.nk; ++ks, ++it) {
        const int s = it % C::kStages;
        const uint32_t ph = (uint32_t)(it / C::kStages) & 1u;
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
        if (my_map) {
          const int ka = ks * C::kBK;
          const int kx = (MODE == kRouter && lane >= 2) ? ka % args.H : ka;
          ptx::tma_load_2d(smem + s * C::kStageBytes + my_off, my_map, &S.full[s], kx, my_row);
        }
      }
    }
    if (aborted && lane == 0) {
      // let this CTA's copies in flight land before the shared memory is released
      for (int s = 0; s < C::kStages; ++s)
        if (armed[s] >= 0) drain_phase(&S.full[s], (uint32_t)armed[s]);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // Kept short on purpose: the tensor core takes an MMA only about when it can start
      // it, so every instruction between MMAs is idle time for it (running ring position,
      // four MMAs per asm block).
      int s = 0;
      uint32_t ph = 0;
      Slots sl;
      bool aborted = false;
      const uint64_t desc0 = ptx::smem_desc_kmajor<C::kRowBytes>(smem);  // stage 0, first A tile
      constexpr uint64_t kDA = C::kATileBytes >> 4;
      // readiness of the next stage, tested while the current stage's MMAs are queued
      bool ready = ptx::mbar_test_wait(&S.full[0], 0);
      for (int qi = 0; !aborted; ++qi) {
        const int slot = qi % kQueue;
        if (!wait_phase(&S.q_full[slot], (uint32_t)(qi / kQueue) & 1u, S, args.status)) {
          aborted = true;
          break;
        }
        const int tile = S.q[slot];
        ptx::mbar_arrive(&S.q_empty[slot]);
        if (tile < 0) break;
        const Geom G = tile_geom<MODE>(args, S, tile, R);
        const int cols = MODE == kDown ? 2 * G.t.N : G.t.N;  // down: columns [0,N) hi, [N,2N) lo
        const uint32_t idesc = ptx::idesc_bf16_f32(128, cols);
        int first, count;
        sl.take(cols, first, count);
        for (int i = 0; i < count && !aborted; ++i) {
          const int sidx = (first + i) & 1;
          if (!wait_phase(&S.tmem_empty[sidx], (sl.uses[sidx] & 1u) ^ 1u, S, args.status))
            aborted = true;
        }
        if (aborted) break;
        ptx::tc_fence_after();
        const uint32_t d0 = tmem + first * kSlotCols;
        const uint32_t d1 = d0 + (count == 2 ? kSlotCols : 128u);
        for (int ks = 0; ks < G.nk; ++ks) {
          // The copies' completion on the full barrier orders them before the MMAs that
          // read the stage; no tcgen05 fence is needed here.
          if (!ready && !wait_phase(&S.full[s], ph, S, args.status)) {
            aborted = true;
            break;
          }
          const int s2 = (s + 1 == C::kStages) ? 0 : s + 1;
          const uint32_t ph2 = (s2 == 0) ? (ph ^ 1u) : ph;
          const uint64_t a0 = desc0 + (uint64_t)s * (C::kStageBytes >> 4);
          const uint64_t bd = a0 + 2 * kDA;
          const uint32_t acc = ks > 0 ? 1u : 0u;
          ptx::umma_bf16_x4(d0, a0, bd, idesc, acc);
          ready = ptx::mbar_test_wait(&S.full[s2], ph2);
          ptx::umma_bf16_x4(d1, a0 + kDA, bd, idesc, acc);
          ptx::umma_commit(&S.empty[s]);
          s = s2;
          ph = ph2;
        }
        if (aborted) break;
        for (int i = 0; i < count; ++i) ptx::umma_commit(&S.tmem_full[(first + i) & 1]);
        sl.done(first, count);
      }
      if (aborted) {
        ptx::umma_commit(&S.drain);  // completes once every MMA issued so far is done
        drain_phase(&S.drain, 0);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int qd = warp & 3;
    const int half = (warp - 2) / 4;  // which 32-column chunks this warp drains
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
    constexpr int kChunks = Cfg<MODE>::kMaxTile / 64;  // chunks per warp
    Slots sl;
    for (int qi = 0;; ++qi) {
      const int slot = qi % kQueue;
      const bool got = wait_phase(&S.q_full[slot], (uint32_t)(qi / kQueue) & 1u, S, args.status);
      if (!__all_sync(0xffffffffu, got)) break;
      const int tile = S.q[slot];
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&S.q_empty[slot]);
      if (tile < 0) break;
      const Geom G = tile_geom<MODE>(args, S, tile, R);
      const Tile& tl = G.t;
      int first, count;
      sl.take(MODE == kDown ? 2 * tl.N : tl.N, first, count);
      const uint32_t b0 = tmem + lane_off + first * kSlotCols;
      const uint32_t b1 = b0 + (count == 2 ? kSlotCols : 128u);
      // down: token and weight of this warp's columns, requested before waiting for the
      // accumulators so that the loads overlap the tile's MMAs
      int col_tok[kChunks];
      float col_w[kChunks];
      if (MODE == kDown) {
#pragma unroll
        for (int ci = 0; ci < kChunks; ++ci) {
          const int c = (2 * ci + half) * 32 + lane;
          col_tok[ci] = 0;
          col_w[ci] = 0.f;
          if (c < tl.nvalid) {
            const int p = tl.p0 + c;
            col_tok[ci] = token_of_row(args, p, R);
            if (args.out) col_w[ci] = p < R ? args.sorted_w[p] : args.sgate[col_tok[ci]];
          }
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
        const int c0 = (2 * ci + half) * 32;
        if (c0 >= tl.nvalid) break;
        uint32_t r0[32], r1[32];
        ptx::tmem_ld32(b0 + c0, r0);
        ptx::tmem_ld32(b1 + c0, r1);
        if (MODE == kDown) {
          // add the lo half (columns N + c0 ..; they stay inside this accumulator's region:
          // c0 < N, so N + c0 + 31 < 128 for N <= 64 and < 256 for N <= 128)
          uint32_t l0[32], l1[32];
          ptx::tmem_ld32(b0 + tl.N + c0, l0);
          ptx::tmem_ld32(b1 + tl.N + c0, l1);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            r0[j] = __float_as_uint(__uint_as_float(r0[j]) + __uint_as_float(l0[j]));
            r1[j] = __float_as_uint(__uint_as_float(r1[j]) + __uint_as_float(l1[j]));
          }
        } else {
          ptx::tmem_ld_wait();
        }
        if (is_gate_up(MODE)) {
          const int ch = tl.m * 128 + qd * 32 + lane;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            if (c0 + j < tl.nvalid) {
              const float gv = __uint_as_float(r0[j]);
              // SiLU(g) = g / (1 + e^-g) with the fast exponential and division (a few ulp;
              // h is carried with 16 or, for fp16 down operands, 11 significant bits)
              const float hv = __fdividef(gv, 1.f + __expf(-gv)) * __uint_as_float(r1[j]);
              const size_t at = (size_t)(tl.p0 + c0 + j) * args.ldh + ch;
              store_h(args.h, args.h_plane, at, hv, args.h_f16, args.status);
            }
          }
        } else if (MODE == kRouter) {
          const int e0 = tl.m * 256 + qd * 32 + lane;  // experts e0 and e0 + 128
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            if (c0 + j < tl.nvalid) {
              float* row = args.logits + (size_t)(tl.p0 + c0 + j) * E;
              if (e0 < E) row[e0] = __uint_as_float(r0[j]);
              if (e0 + 128 < E) row[e0 + 128] = __uint_as_float(r1[j]);
            }
          }
        } else {
          // 32 channels (lanes) x 32 tokens (registers) per accumulator; every 8 tokens go
          // through shared memory so that eight lanes own the 32 channels (128 bytes) of one
          // token, four tokens per instruction: every 16-byte atomic add or store of a
          // warp lands in whole 128-byte lines (a lane-per-channel order, or two 16-byte
          // pieces 32 bytes apart, cut the reduction throughput by a third)
          const int mrow = tl.m * 256 + qd * 32 + 4 * (lane & 7);  // this lane's channels
          const int H = args.H;
          float4(&xp)[8][8] = S.xpose[warp - 2];
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
                const int q = hq * 4 + (lane >> 3);  // this lane's token within the 8
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
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

// Token rows in dispatch order: xs[p] = x[sorted_token[p]] for the R routed rows, so that
// a tile's tokens are consecutive rows of one tensor. One warp per row, 16-byte copies.
__global__ void __launch_bounds__(256)
gather_rows_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ sorted_token,
                   const int* __restrict__ plan, int E, int T, int H, uint16_t* __restrict__ xs,
                   uint32_t* __restrict__ status, int* __restrict__ counter) {
  if (blockIdx.x == 0 && threadIdx.x == 0) *counter = 0;  // tile counter of the gate|up GEMM
  const int R = plan_view(const_cast<int*>(plan), E).row0[E];
  const int lane = threadIdx.x & 31;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  for (int p = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; p < R; p += nwarps) {
    int t = sorted_token[p];
    if ((unsigned)t >= (unsigned)T) {
      set_flag(status, kFlagBounds);
      t = 0;
    }
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * H);
    uint4* dst = reinterpret_cast<uint4*>(xs + (size_t)p * H);
    for (int c = lane; c < H / 8; c += 32) dst[c] = __ldg(src + c);
  }
}

// Router matrix fp32 [E][H] -> bf16 pieces [E][3H] = hi | mid | lo with
// w = hi + mid + lo exactly (each piece takes the next 8 significant bits), so every
// product with a bf16 activation is exact.
__global__ void router_split_kernel(const float* __restrict__ wr, uint16_t* __restrict__ out,
                                    int E, int H, int* __restrict__ counter) {
  if (blockIdx.x == 0 && threadIdx.x == 0) *counter = 0;  // tile counter of the router GEMM
  const size_t n = (size_t)E * H;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    const size_t e = i / H, h = i % H;
    const float w = wr[i];
    const uint16_t hi = f32_to_bf16_rn(w);
    const float r1 = w - bf16lo(hi);
    const uint16_t mid = f32_to_bf16_rn(r1);
    const float r2 = r1 - bf16lo(mid);
    uint16_t* row = out + e * 3 * (size_t)H;
    row[h] = hi;
    row[H + h] = mid;
    row[2 * H + h] = f32_to_bf16_rn(r2);
  }
}

// ---------------------------------------------------------------- host side

// The token tensor [outer][inner] in every box height of a token tile.
bool make_bmaps(BMaps* b, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner) {
  for (int i = 0; i < kBoxHeights; ++i)
    if (!make_map(&b->m[i], base, inner, outer, box_inner, (uint32_t)box_rows_of(i))) return false;
  return true;
}

template <int MODE>
cudaError_t launch_mode(const CUtensorMap& a, const CUtensorMap& a_sh, const BMaps& b,
                        const BMaps& b_sh, const TcArgs& args, int grid, cudaStream_t st) {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(tc_grouped_kernel<MODE>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)smem_bytes<MODE>());
  });
  if (attr_err != cudaSuccess) return attr_err;
  tc_grouped_kernel<MODE><<<grid, kThreads, smem_bytes<MODE>(), st>>>(a, a_sh, b, b_sh, args);
  return cudaGetLastError();
}

}  // namespace

bool tc_router_supported(const moe_shape& s) {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return false;
  return major == 10 && encode_fn() != nullptr && s.H % 64 == 0;
}

cudaError_t launch_tc_router(const moe_shape& s, const Layout& L, char* ws, const uint16_t* x,
                             const float* wr, float* logits, cudaStream_t st) {
  using C = Cfg<kRouter>;
  uint16_t* split = reinterpret_cast<uint16_t*>(ws + L.wr_split);
  {
    LaunchScope scope(MOE_K_OTHER, st);
    const size_t n = (size_t)s.E * s.H;
    const int blocks = (int)std::min<size_t>((n + 255) / 256, (size_t)sm_count() * 8);
    router_split_kernel<<<blocks, 256, 0, st>>>(wr, split, s.E, s.H,
                                                reinterpret_cast<int*>(ws + L.sched) + 2);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  CUtensorMap a;
  BMaps b;
  if (!make_map(&a, split, 3ull * s.H, (uint64_t)s.E, C::kBK, 128) ||
      !make_bmaps(&b, x, s.H, (uint64_t)s.T, C::kBK))
    return cudaErrorInvalidValue;
  TcArgs args = base_args(s, L, ws);
  args.logits = logits;
  args.ntiles = ((s.E + 255) / 256) * ((s.T + C::kMaxTile - 1) / C::kMaxTile);
  args.counter = reinterpret_cast<int*>(ws + L.sched) + 2;
  LaunchScope scope(MOE_K_ROUTER_LOGITS, st);
  return launch_mode<kRouter>(a, a, b, b, args, std::min(args.ntiles, sm_count()), st);
}

bool tc_supported(const moe_shape& s) {
  if (s.I % 128 || s.Is % 128 || s.H % 256) return false;
  return tc_router_supported(s);
}

cudaError_t launch_gather_rows(const moe_shape& s, const Layout& L, char* ws, const uint16_t* x,
                               const int32_t* sorted_token, cudaStream_t st) {
  LaunchScope scope(MOE_K_OTHER, st);
  gather_rows_kernel<<<sm_count() * 8, 256, 0, st>>>(
      x, sorted_token, reinterpret_cast<const int*>(ws + L.plan), s.E, s.T, s.H,
      reinterpret_cast<uint16_t*>(ws + L.xs), reinterpret_cast<uint32_t*>(ws + L.status),
      reinterpret_cast<int*>(ws + L.sched) + 0);
  return cudaGetLastError();
}

cudaError_t launch_tc_gate_up(const moe_shape& s, const Layout& L, char* ws, const uint16_t* x,
                              const int32_t* sorted_token, const moe_weights& w, int h_f16,
                              cudaStream_t st) {
  using C = Cfg<kGateUp>;  // kBK and box shapes are the same for kGateUpSmall
  uint16_t* xs = reinterpret_cast<uint16_t*>(ws + L.xs);
  {
    cudaError_t e = launch_gather_rows(s, L, ws, x, sorted_token, st);
    if (e != cudaSuccess) return e;
  }
  CUtensorMap a, a_sh;
  BMaps b, b_sh;
  if (!make_map(&a, w.w_gate_up, s.H, (uint64_t)s.E * 2 * s.I, C::kBK, 128) ||
      !make_map(&a_sh, w.ws_gate_up, s.H, 2ull * s.Is, C::kBK, 128) ||
      !make_bmaps(&b, xs, s.H, (uint64_t)s.T * s.k, C::kBK) ||
      !make_bmaps(&b_sh, x, s.H, (uint64_t)s.T, C::kBK))
    return cudaErrorInvalidValue;
  TcArgs args = base_args(s, L, ws);
  args.sorted_token = sorted_token;
  args.counter = reinterpret_cast<int*>(ws + L.sched) + 0;
  args.counter_next = reinterpret_cast<int*>(ws + L.sched) + 1;
  args.h_f16 = h_f16;
  LaunchScope scope(MOE_K_GATE_UP, st);
  if (tc_gate_up_chunk(s.T, s.k, s.E) == kTcChunkSmall)
    return launch_mode<kGateUpSmall>(a, a_sh, b, b_sh, args, sm_count(), st);
  return launch_mode<kGateUp>(a, a_sh, b, b_sh, args, sm_count(), st);
}

cudaError_t launch_tc_down(const moe_shape& s, const Layout& L, char* ws,
                           const int32_t* sorted_token, const float* sorted_w, const float* sgate,
                           const moe_weights& w, float* y, float* y_shared, float* out,
                           cudaStream_t st) {
  using C = Cfg<kDown>;
  CUtensorMap a, a_sh;
  BMaps b;
  if (!make_map(&a, w.w_down, s.I, (uint64_t)s.E * s.H, C::kBK, 128) ||
      !make_map(&a_sh, w.ws_down, s.Is, (uint64_t)s.H, C::kBK, 128) ||
      !make_bmaps(&b, ws + L.h, L.ldh, 2 * (L.h_plane / L.ldh), C::kBK))
    return cudaErrorInvalidValue;
  TcArgs args = base_args(s, L, ws);
  args.sorted_token = sorted_token;
  args.sorted_w = sorted_w;
  args.sgate = sgate;
  args.y = y;
  args.y_shared = y_shared;
  args.out = out;
  args.counter = reinterpret_cast<int*>(ws + L.sched) + 1;
  LaunchScope scope(MOE_K_DOWN, st);
  return launch_mode<kDown>(a, a_sh, b, b, args, sm_count(), st);
}

}  // namespace moe
