// tc_gemm.cu -- stage 4, "Grouped expert GEMMs" (Qwen3.8-Flash-Next architecture study,
// MoE pipeline diagram; expert(x) = W_down(SiLU(W_gate x) * W_up x)) on the 5th-generation
// tensor cores: TMA-fed shared-memory ring, tcgen05.mma with fp32 accumulators in tensor
// memory, and fused epilogues.
//
// Orientation ("swap AB"): expert weight rows are the MMA's M side (128 rows per
// accumulator), the tokens of one expert are the N side (16..256 per tile), K is the
// hidden (gate|up) or intermediate (down) dimension. Every weight byte is read from HBM
// once per token chunk; token rows come from L2.
//
//   gate|up kernel: per tile, gate rows [c, c+128) and up rows [I+c, I+c+128) of one expert
//     against up to 256 of its tokens, gathered from x by TMA (tile::gather4) through the
//     dispatch order. Two accumulators (gate, up) share the token tile. Epilogue:
//     h = SiLU(gate) * up, stored as the bf16 pair hi = bf16(h), lo = bf16(h - hi).
//   down kernel: per tile, 256 output rows (two accumulators) of one expert's W_down
//     against up to 128 of its packed rows; the token tile holds the hi rows followed by
//     the lo rows, so one MMA with N' = 2N produces W h_hi and W h_lo side by side and the
//     epilogue adds them. Epilogue: y rows (staged path) or routing-weight-scaled fp32
//     atomic adds into out[token] ("Weighted combine + gated shared expert").
//
// Roles in a 192-thread CTA (one CTA per SM, persistent over the tile list):
//   warp 0      TMA producer (lane 0 issues), kStages-deep ring of 64 KB stages;
//   warp 1      TMEM owner (512 columns) and MMA issuer (lane 0);
//   warps 2..5  epilogue, warp w reads TMEM lanes 32*(w%4) .. +31.
// Every mbarrier wait is bounded (2 s); on expiry the kernel records the timeout flag,
// lets every role leave its loop, drains its own copies and MMAs and frees TMEM.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "device_common.cuh"
#include "sm100_ptx.cuh"
#include "tc_gemm.h"

namespace moe {
namespace {

constexpr int kStages = 3;
constexpr int kThreads = 192;
constexpr uint32_t kATileBytes = 128 * 128;      // 128 rows x 64 bf16
constexpr uint32_t kBTileMaxBytes = 256 * 128;   // 256 rows x 64 bf16
constexpr uint32_t kStageBytes = 2 * kATileBytes + kBTileMaxBytes;
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint64_t kDrainLimitNs = 200000000ull;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAcc1Col = 256;  // column of the second accumulator

enum Mode { kGateUp = 0, kDown = 1, kRouter = 2 };

struct SharedState {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t tmem_full;
  uint64_t tmem_empty;
  uint64_t drain;
  uint32_t tmem_base;
  volatile int abort;
  int tok[256];
};

constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kStageBytes + sizeof(SharedState);

struct TcArgs {
  const int* plan;
  int E, H, I, Is, T, ldh;
  size_t h_plane;
  const int32_t* sorted_token;
  const float* sorted_w;
  const float* sgate;
  uint16_t* h;
  float* y;
  float* y_shared;
  float* out;
  uint32_t* status;
  float* logits;  // router: [T][E]
  int ntiles;     // router: tile count (no plan)
};

struct Tile {
  int g, m, p0, nvalid, N;
};

// Tile -> (group, M tile, packed rows). Groups own consecutive tile ranges
// [tp[g], tp[g+1]); inside a group the token chunks of one M tile are adjacent, so the
// second chunk's weight tile is read from L2.
__device__ __forceinline__ Tile decode_tile(const PlanView& pv, const int* tp, int E, int tile,
                                            int chunk_max) {
  int lo = 0, hi = E + 1;  // tp[lo] <= tile < tp[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (tp[mid] <= tile) lo = mid;
    else hi = mid;
  }
  Tile t;
  t.g = lo;
  const int n = pv.row0[lo + 1] - pv.row0[lo];
  const int nch = (n + chunk_max - 1) / chunk_max;
  const int cs = (((n + nch - 1) / nch) + 15) & ~15;
  const int local = tile - tp[lo];
  t.m = local / nch;
  const int c = local - t.m * nch;
  const int start = c * cs;
  t.nvalid = min(cs, n - start);
  t.N = (t.nvalid + 15) & ~15;
  t.p0 = pv.row0[lo] + start;
  return t;
}

// Bounded wait on an mbarrier phase; false if it ran out (flag recorded) or another role
// already gave up.
__device__ __forceinline__ bool wait_phase(uint64_t* bar, uint32_t parity, SharedState& S,
                                           uint32_t* status) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
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

// Short bounded wait used while leaving after an abort.
__device__ __forceinline__ void drain_phase(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!ptx::mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kDrainLimitNs) return;
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

// Everything the three roles need to know about one tile.
struct Geom {
  Tile t;
  int a_row0, a_row1;  // A-operand rows of the two accumulators
  int nk;              // 64-wide K steps
  bool shared;         // shared-expert group (its own weight tensor map)
};

template <int MODE>
__device__ __forceinline__ Geom tile_geom(const TcArgs& a, const PlanView& pv, int tile) {
  Geom G;
  if (MODE == kRouter) {
    // 256 router rows (experts) x up to 256 tokens; K runs over the hi|mid|lo pieces
    const int mt = (a.E + 255) / 256;
    const int m = tile % mt, c = tile / mt;
    G.t.g = 0;
    G.t.m = m;
    G.t.p0 = c * 256;
    G.t.nvalid = min(256, a.T - G.t.p0);
    G.t.N = (G.t.nvalid + 15) & ~15;
    G.a_row0 = m * 256;
    G.a_row1 = m * 256 + 128;
    G.nk = 3 * a.H / 64;
    G.shared = false;
    return G;
  }
  const int* tp = (MODE == kGateUp) ? pv.tp1 : pv.tp2;
  G.t = decode_tile(pv, tp, a.E, tile, (MODE == kGateUp) ? kTcChunk : kTcChunkDown);
  G.shared = G.t.g == a.E;
  if (MODE == kGateUp) {
    const int Ig = G.shared ? a.Is : a.I;
    const int base = G.shared ? 0 : G.t.g * 2 * a.I;
    G.a_row0 = base + G.t.m * 128;
    G.a_row1 = base + Ig + G.t.m * 128;
    G.nk = a.H / 64;
  } else {
    const int base = G.shared ? 0 : G.t.g * a.H;
    G.a_row0 = base + G.t.m * 256;
    G.a_row1 = G.a_row0 + 128;
    G.nk = (G.shared ? a.Is : a.I) / 64;
  }
  return G;
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
tc_grouped_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_a_sh,
                  const __grid_constant__ CUtensorMap tm_b, const TcArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  SharedState& S = *reinterpret_cast<SharedState*>(smem + kStages * kStageBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = args.E;
  PlanView pv{};
  int total, R = 0;
  if (MODE == kRouter) {
    total = args.ntiles;
  } else {
    pv = plan_view(const_cast<int*>(args.plan), E);
    total = ((MODE == kGateUp) ? pv.tp1 : pv.tp2)[E + 1];
    R = pv.row0[E];
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(&S.full[s], 1);
      ptx::mbar_init(&S.empty[s], 1);
    }
    ptx::mbar_init(&S.tmem_full, 1);
    ptx::mbar_init(&S.tmem_empty, 128);
    ptx::mbar_init(&S.drain, 1);
    S.abort = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tm_a);
    ptx::prefetch_tmap(&tm_a_sh);
    ptx::prefetch_tmap(&tm_b);
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
    int it = 0;
    int armed[kStages];
#pragma unroll
    for (int s = 0; s < kStages; ++s) armed[s] = -1;
    int aborted = 0;
    const int plane_rows = (MODE == kDown) ? (int)(args.h_plane / (size_t)args.ldh) : 0;
    for (int tile = blockIdx.x; tile < total && !aborted; tile += gridDim.x) {
      const Geom G = tile_geom<MODE>(args, pv, tile);
      const Tile& tl = G.t;
      const CUtensorMap* ta = G.shared ? &tm_a_sh : &tm_a;
      if (MODE == kGateUp) {
        for (int j = lane; j < tl.N; j += 32) {
          const int q = j < tl.nvalid ? j : tl.nvalid - 1;  // pad with the last real row
          S.tok[j] = token_of_row(args, tl.p0 + q, R);
        }
        __syncwarp();
      }
      if (lane == 0) {
        const int brows = (MODE == kDown) ? 2 * tl.N : tl.N;
        const uint32_t bytes = 2 * kATileBytes + (uint32_t)brows * 128u;
        for (int ks = 0; ks < G.nk; ++ks, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (uint32_t)(it / kStages) & 1u;
          if (!wait_phase(&S.empty[s], ph ^ 1u, S, args.status)) {
            aborted = 1;
            break;
          }
          ptx::mbar_arrive_expect_tx(&S.full[s], bytes);
          armed[s] = (int)ph;
          uint8_t* st = smem + s * kStageBytes;
          ptx::tma_load_2d(st, ta, &S.full[s], ks * 64, G.a_row0);
          ptx::tma_load_2d(st + kATileBytes, ta, &S.full[s], ks * 64, G.a_row1);
          uint8_t* b = st + 2 * kATileBytes;
          if (MODE == kGateUp) {
            for (int j = 0; j < tl.N; j += 4)
              ptx::tma_gather4(b + j * 128, &tm_b, &S.full[s], ks * 64, S.tok[j], S.tok[j + 1],
                               S.tok[j + 2], S.tok[j + 3]);
          } else if (MODE == kDown) {
            for (int j = 0; j < tl.N; j += 16) {
              ptx::tma_load_2d(b + j * 128, &tm_b, &S.full[s], ks * 64, tl.p0 + j);
              ptx::tma_load_2d(b + (tl.N + j) * 128, &tm_b, &S.full[s], ks * 64,
                               plane_rows + tl.p0 + j);
            }
          } else {
            const int kx = (ks * 64) % args.H;  // the same x columns for each router piece
            for (int j = 0; j < tl.N; j += 16)
              ptx::tma_load_2d(b + j * 128, &tm_b, &S.full[s], kx, tl.p0 + j);
          }
        }
      }
      aborted = __shfl_sync(0xffffffffu, aborted, 0);
      __syncwarp();
    }
    if (aborted && lane == 0) {
      // let this CTA's copies in flight land before the shared memory is released
      for (int s = 0; s < kStages; ++s)
        if (armed[s] >= 0) drain_phase(&S.full[s], (uint32_t)armed[s]);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int it = 0, tcount = 0;
      bool aborted = false;
      for (int tile = blockIdx.x; tile < total && !aborted; tile += gridDim.x, ++tcount) {
        const Geom G = tile_geom<MODE>(args, pv, tile);
        const int nmma = (MODE == kDown) ? 2 * G.t.N : G.t.N;
        const uint32_t idesc = ptx::idesc_bf16_f32(128, nmma);
        if (!wait_phase(&S.tmem_empty, ((uint32_t)tcount & 1u) ^ 1u, S, args.status)) {
          aborted = true;
          break;
        }
        ptx::tc_fence_after();
        for (int ks = 0; ks < G.nk; ++ks, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (uint32_t)(it / kStages) & 1u;
          if (!wait_phase(&S.full[s], ph, S, args.status)) {
            aborted = true;
            break;
          }
          ptx::tc_fence_after();
          const uint8_t* st = smem + s * kStageBytes;
          const uint64_t a0 = ptx::smem_desc_sw128(st);
          const uint64_t a1 = ptx::smem_desc_sw128(st + kATileBytes);
          const uint64_t bd = ptx::smem_desc_sw128(st + 2 * kATileBytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t acc = (ks > 0 || kk > 0) ? 1u : 0u;
            // +32 bytes along K inside the 128-byte swizzle atom = +2 in the address field
            ptx::umma_bf16(tmem, a0 + 2 * kk, bd + 2 * kk, idesc, acc);
            ptx::umma_bf16(tmem + kAcc1Col, a1 + 2 * kk, bd + 2 * kk, idesc, acc);
          }
          ptx::umma_commit(&S.empty[s]);
        }
        if (aborted) break;
        ptx::umma_commit(&S.tmem_full);
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
    const uint32_t lane_base = tmem + ((uint32_t)(qd * 32) << 16);
    int tcount = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++tcount) {
      const Geom G = tile_geom<MODE>(args, pv, tile);
      const Tile& tl = G.t;
      const bool ok = wait_phase(&S.tmem_full, (uint32_t)tcount & 1u, S, args.status);
      if (!__all_sync(0xffffffffu, ok)) break;
      ptx::tc_fence_after();
      if (MODE == kGateUp) {
        const int ch = tl.m * 128 + qd * 32 + lane;
        for (int c0 = 0; c0 < tl.nvalid; c0 += 32) {
          uint32_t g[32], u[32];
          ptx::tmem_ld32(lane_base + c0, g);
          ptx::tmem_ld32(lane_base + kAcc1Col + c0, u);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            if (c0 + j < tl.nvalid) {
              const float gv = __uint_as_float(g[j]);
              const float hv = gv / (1.f + expf(-gv)) * __uint_as_float(u[j]);
              const uint16_t hi = f32_to_bf16_rn(hv);
              const size_t at = (size_t)(tl.p0 + c0 + j) * args.ldh + ch;
              args.h[at] = hi;
              args.h[args.h_plane + at] = f32_to_bf16_rn(hv - bf16lo(hi));
            }
          }
        }
      } else if (MODE == kRouter) {
        const int e0 = tl.m * 256 + qd * 32 + lane;  // experts e0 and e0 + 128
        for (int c0 = 0; c0 < tl.nvalid; c0 += 32) {
          uint32_t l0[32], l1[32];
          ptx::tmem_ld32(lane_base + c0, l0);
          ptx::tmem_ld32(lane_base + kAcc1Col + c0, l1);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            if (c0 + j < tl.nvalid) {
              float* row = args.logits + (size_t)(tl.p0 + c0 + j) * E;
              if (e0 < E) row[e0] = __uint_as_float(l0[j]);
              if (e0 + 128 < E) row[e0 + 128] = __uint_as_float(l1[j]);
            }
          }
        }
      } else {
        const int m = tl.m * 256 + qd * 32 + lane;  // rows m (first accumulator), m + 128
        const int H = args.H;
        for (int c0 = 0; c0 < tl.nvalid; c0 += 32) {
          uint32_t ra[32], rb[32];
          float y0[32], y1[32];
          ptx::tmem_ld32(lane_base + c0, ra);
          ptx::tmem_ld32(lane_base + tl.N + c0, rb);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) y0[j] = __uint_as_float(ra[j]) + __uint_as_float(rb[j]);
          ptx::tmem_ld32(lane_base + kAcc1Col + c0, ra);
          ptx::tmem_ld32(lane_base + kAcc1Col + tl.N + c0, rb);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) y1[j] = __uint_as_float(ra[j]) + __uint_as_float(rb[j]);
          // token and weight of column c0 + lane
          const int colp = tl.p0 + c0 + lane;
          int tok = 0;
          float wgt = 0.f;
          if (c0 + lane < tl.nvalid) {
            tok = token_of_row(args, colp, R);
            if (args.out) wgt = colp < R ? args.sorted_w[colp] : args.sgate[tok];
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            if (c0 + j < tl.nvalid) {
              const int t = __shfl_sync(0xffffffffu, tok, j);
              const float w = __shfl_sync(0xffffffffu, wgt, j);
              const int p = tl.p0 + c0 + j;
              if (args.out) {
                float* o = args.out + (size_t)t * H + m;
                atomicAdd(o, w * y0[j]);
                atomicAdd(o + 128, w * y1[j]);
              } else if (p < R) {
                float* o = args.y + (size_t)p * H + m;
                o[0] = y0[j];
                o[128] = y1[j];
              } else {
                float* o = args.y_shared + (size_t)(p - R) * H + m;
                o[0] = y0[j];
                o[128] = y1[j];
              }
            }
          }
        }
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(&S.tmem_empty);
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

// Router matrix fp32 [E][H] -> bf16 pieces [E][3H] = hi | mid | lo with
// w = hi + mid + lo exactly (each piece takes the next 8 significant bits), so every
// product with a bf16 activation is exact and the tensor-core sum is an fp32 dot product.
__global__ void router_split_kernel(const float* __restrict__ wr, uint16_t* __restrict__ out,
                                    int E, int H) {
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

// 2-D bf16 tensor [outer][inner] (inner contiguous), box [box_outer][box_inner],
// 128-byte swizzle (box_inner = 64 elements = 128 bytes).
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
              uint32_t box_inner, uint32_t box_outer) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * sizeof(uint16_t)};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

template <int MODE>
cudaError_t launch_mode(const CUtensorMap& a, const CUtensorMap& a_sh, const CUtensorMap& b,
                        const TcArgs& args, cudaStream_t st) {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(tc_grouped_kernel<MODE>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  });
  if (attr_err != cudaSuccess) return attr_err;
  tc_grouped_kernel<MODE><<<sm_count(), kThreads, kSmemBytes, st>>>(a, a_sh, b, args);
  return cudaGetLastError();
}

TcArgs base_args(const moe_shape& s, const Layout& L, char* ws) {
  TcArgs a{};
  a.plan = reinterpret_cast<const int*>(ws + L.plan);
  a.E = s.E;
  a.H = s.H;
  a.I = s.I;
  a.Is = s.Is;
  a.T = s.T;
  a.ldh = L.ldh;
  a.h_plane = L.h_plane;
  a.h = reinterpret_cast<uint16_t*>(ws + L.h);
  a.status = reinterpret_cast<uint32_t*>(ws + L.status);
  return a;
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
  uint16_t* split = reinterpret_cast<uint16_t*>(ws + L.wr_split);
  {
    LaunchScope scope(MOE_K_OTHER, st);
    const size_t n = (size_t)s.E * s.H;
    const int blocks = (int)std::min<size_t>((n + 255) / 256, (size_t)sm_count() * 8);
    router_split_kernel<<<blocks, 256, 0, st>>>(wr, split, s.E, s.H);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  CUtensorMap a, b;
  if (!make_map(&a, split, 3ull * s.H, (uint64_t)s.E, 64, 128) ||
      !make_map(&b, x, s.H, (uint64_t)s.T, 64, 16))
    return cudaErrorInvalidValue;
  TcArgs args = base_args(s, L, ws);
  args.logits = logits;
  args.ntiles = ((s.E + 255) / 256) * ((s.T + 255) / 256);
  LaunchScope scope(MOE_K_ROUTER_LOGITS, st);
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(tc_grouped_kernel<kRouter>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const int grid = std::min(args.ntiles, sm_count());
  tc_grouped_kernel<kRouter><<<grid, kThreads, kSmemBytes, st>>>(a, a, b, args);
  return cudaGetLastError();
}

bool tc_supported(const moe_shape& s) {
  if (s.I % 128 || s.Is % 128 || s.H % 256) return false;
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return false;
  return major == 10 && encode_fn() != nullptr;
}

cudaError_t launch_tc_gate_up(const moe_shape& s, const Layout& L, char* ws, const uint16_t* x,
                              const int32_t* sorted_token, const moe_weights& w, cudaStream_t st) {
  CUtensorMap a, a_sh, b;
  if (!make_map(&a, w.w_gate_up, s.H, (uint64_t)s.E * 2 * s.I, 64, 128) ||
      !make_map(&a_sh, w.ws_gate_up, s.H, 2ull * s.Is, 64, 128) ||
      !make_map(&b, x, s.H, (uint64_t)s.T, 64, 1))
    return cudaErrorInvalidValue;
  TcArgs args = base_args(s, L, ws);
  args.sorted_token = sorted_token;
  LaunchScope scope(MOE_K_GATE_UP, st);
  return launch_mode<kGateUp>(a, a_sh, b, args, st);
}

cudaError_t launch_tc_down(const moe_shape& s, const Layout& L, char* ws,
                           const int32_t* sorted_token, const float* sorted_w, const float* sgate,
                           const moe_weights& w, float* y, float* y_shared, float* out,
                           cudaStream_t st) {
  CUtensorMap a, a_sh, b;
  if (!make_map(&a, w.w_down, s.I, (uint64_t)s.E * s.H, 64, 128) ||
      !make_map(&a_sh, w.ws_down, s.Is, (uint64_t)s.H, 64, 128) ||
      !make_map(&b, ws + L.h, L.ldh, 2 * (L.h_plane / L.ldh), 64, 16))
    return cudaErrorInvalidValue;
  TcArgs args = base_args(s, L, ws);
  args.sorted_token = sorted_token;
  args.sorted_w = sorted_w;
  args.sgate = sgate;
  args.y = y;
  args.y_shared = y_shared;
  args.out = out;
  LaunchScope scope(MOE_K_DOWN, st);
  return launch_mode<kDown>(a, a_sh, b, args, st);
}

}  // namespace moe
