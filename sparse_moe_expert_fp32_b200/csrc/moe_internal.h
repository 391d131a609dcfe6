// moe_internal.h -- workspace layout, dispatch plan and launch declarations shared by the
// translation units of libmoe_b200.so. Not part of the public ABI (include/moe.h is).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

constexpr int kMaxE = 1024;
constexpr int kMaxK = 32;
constexpr int kPermBlock = 256;  // tokens per dispatch block (one bit per token in a mask)
constexpr int kTcChunk = 256;    // max tokens (MMA N) per tensor-core tile
constexpr uint32_t kFlagBounds = 1u;
constexpr uint32_t kFlagTimeout = 2u;
constexpr uint32_t kFlagRange = 4u;  // a value saturated to fit fp16 (down operands)

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Byte offsets of the workspace regions (all 256-byte aligned).
struct Layout {
  size_t status;        // uint32 [64]: [0] = error flags, [1..] = diagnostics
  size_t logits;        // fp32 [8][T][E] partial router logits for T < 512, else [T][E]
                        // (at least 8 x 511 x E entries from T = 512 on: sizes grow with T)
  size_t wr_split;      // bf16 [E][3H]: router matrix as hi|mid|lo bf16 pieces (tensor-core router)
  size_t ids;           // int32 [T][k]
  size_t w;             // fp32 [T][k]
  size_t sgate;         // fp32 [T]
  size_t gap;           // fp32 [T]
  size_t blk_mask;      // uint32 [nblk][E][8]: token bitmask per dispatch block and expert
  size_t blk_base;      // int32 [nblk][E]: first packed row of (block, expert)
  size_t offsets;       // int32 [E+2]
  size_t sorted_token;  // int32 [T*k]
  size_t sorted_w;      // fp32 [T*k]: routing weight of each packed row
  size_t assign_row;    // int32 [T*k]
  size_t plan;          // int32 plan arrays (see PlanView)
  size_t sched;         // int32 [4] tile counters of the tensor-core kernels (gate|up, down,
                        // router), zeroed by the kernel that runs before each of them
  size_t xs;            // bf16 [T*k][H]: token rows in dispatch order (tensor-core gate|up)
  size_t h;             // bf16 [2][T*k + T][ldh]: SwiGLU intermediate as a hi|lo pair of planes
                        // (h = hi + lo), routed rows then shared rows
  size_t h_plane;       // elements per plane: (T*k + T) * ldh
  size_t total;
  int nblk;
  int ldh;              // max(I, Is)
};

Layout layout(const moe_shape& s);

// Dispatch plan: groups 0..E-1 are the routed experts, group E the shared expert
// (all T tokens in order). Group g owns packed rows [row0[g], row0[g+1]) of h.
struct PlanView {
  int* n_active;  // [1]
  int* active;    // [E+1] group ids with >= 1 row, ascending
  int* row0;      // [E+2]
  int* tp1;       // [E+2] tile prefix of the tensor-core gate|up GEMM
  int* tp2;       // [E+2] tile prefix of the tensor-core down GEMM (bf16 h pair, 128 rows)
  int* tp3;       // [E+2] tile prefix of the down GEMM on fp16 operands (256 rows)
  int* tp4;       // [E+2] tile prefix of the FP8 gate|up GEMM (64 rows at every batch size)
  int* tp5;       // [E+2] tile prefix of the FP8 down GEMM (32 rows)
};

__host__ __device__ inline size_t plan_ints(int E) { return 1 + (size_t)(E + 1) + 6 * (size_t)(E + 2); }

__host__ __device__ inline PlanView plan_view(void* base, int E) {
  int* p = static_cast<int*>(base);
  PlanView v;
  v.n_active = p;
  v.active = p + 1;
  v.row0 = v.active + (E + 1);
  v.tp1 = v.row0 + (E + 2);
  v.tp2 = v.tp1 + (E + 2);
  v.tp3 = v.tp2 + (E + 2);
  v.tp4 = v.tp3 + (E + 2);
  v.tp5 = v.tp4 + (E + 2);
  return v;
}

// Tensor-core tiling of a group with n rows into ceil(n / max) token chunks of nearly equal
// size (multiples of 16 rows): max 256 rows for the gate|up GEMM, 128 for the down GEMM on
// the bf16 h pair (its MMA N is twice the rows), 256 for the down GEMM on fp16 operands.
constexpr int kTcChunkDown = 128;
constexpr int kTcChunkDownF16 = 256;
// Rows per gate|up tile: decode-size batches (T*k < 16*E, a few rows per expert) chunk at
// kTcChunkSmall, so that the one-CTA gate|up kernel's stages can be small and more of them
// fit; larger batches at kTcChunk. The plan builder and both gate|up kernels call this with
// the same T, k, E.
constexpr int kTcChunkSmall = 64;
// Rows per tile of the FP8 kernels, whatever the batch size: gate|up 64 (the token operand
// is two E4M3 pieces, MMA N = 2 x rows), down 32 (h is four pieces, MMA N = 4 x rows; both
// accumulators of a tile then fit in one 256-column TMEM slot).
constexpr int kTcChunkGateUp8 = 64;
constexpr int kTcChunkDown8 = 32;
__host__ __device__ inline int tc_gate_up_chunk(int T, int k, int E) {
  return (long long)T * k < 16LL * E ? kTcChunkSmall : kTcChunk;
}
__host__ __device__ inline int tc_nchunks(int n, int max_rows) {
  return (n + max_rows - 1) / max_rows;
}

// Hidden-dimension slices of the small-batch router's partial logits.
constexpr int kRouterSplits = 8;

// Bytes of the FP8 down GEMM's token operand: four E4M3 pieces of every routed row of h
// (T*k rows of I codes), 256-byte aligned; the fp32 row scales follow.
inline size_t fp8_h_pieces_bytes(const moe_shape& s) {
  return align_up((size_t)4 * s.T * s.k * s.I, 256);
}

// ---------------------------------------------------------------- launch bookkeeping

// RAII: counts a launch and, while profiling is on, brackets it with CUDA events.
struct LaunchScope {
  LaunchScope(moe_kernel id, cudaStream_t s, int nkernels = 1);
  ~LaunchScope();
  int slot;
  cudaStream_t stream;
};

// ---------------------------------------------------------------- kernel launches
// Every launcher enqueues on `st` and returns cudaGetLastError().

// Router logits by the best kernel for the shape (uses the workspace). Small batches
// (T < 512) leave router_slices(s) = kRouterSplits partial sums [slices][T][E] that
// launch_router_topk adds up in order.
cudaError_t launch_router_logits(const moe_shape& s, const Layout& L, char* ws, const uint16_t* x,
                                 const float* wr, float* logits, cudaStream_t st);
int router_slices(const moe_shape& s);
cudaError_t launch_router_topk(const moe_shape& s, const float* logits, const float* wr,
                               const float* bias, const uint16_t* x, const uint16_t* wsg,
                               int32_t* ids, float* w,
                               float* sgate, float* gap, float* out_zero, cudaStream_t st);
cudaError_t launch_permute(const moe_shape& s, const Layout& L, char* ws, const int32_t* ids,
                           const float* topk_w, int32_t* offsets, int32_t* sorted_token,
                           float* sorted_w, int32_t* assign_row, cudaStream_t st);
// Plan from caller-supplied offsets; shared_rows = T with the shared expert, 0 without.
cudaError_t launch_plan_from_offsets(const moe_shape& s, const Layout& L, char* ws,
                                     const int32_t* offsets, int shared_rows, cudaStream_t st);
// Expert-parallel row movement (ep.cu).
cudaError_t launch_gather_rows_bf16(const uint16_t* x, const int32_t* index, int64_t rows,
                                    int64_t n_src, int H, uint16_t* out, uint32_t* status,
                                    int sms, cudaStream_t st);
cudaError_t launch_scatter_rows_f32(const float* y, const int32_t* index, int64_t rows,
                                    int64_t n_dst, int H, float* out, uint32_t* status, int sms,
                                    cudaStream_t st);
cudaError_t launch_ep_regroup(const int32_t* counts, int G, int El, int64_t capacity,
                              int32_t* offsets, int32_t* src_index, int32_t* src_rows,
                              uint32_t* status, cudaStream_t st);
cudaError_t launch_ep_counts(const int32_t* offsets, int G, int El, int32_t* counts,
                             int32_t* rows, cudaStream_t st);
cudaError_t launch_stream_gate_up(const moe_shape& s, const Layout& L, char* ws, const uint16_t* x,
                                  const int32_t* sorted_token, const moe_weights& w,
                                  cudaStream_t st);
cudaError_t launch_stream_down(const moe_shape& s, const Layout& L, char* ws,
                               const int32_t* sorted_token, const float* sorted_w,
                               const float* sgate, const moe_weights& w, float* y,
                               float* y_shared, float* out, cudaStream_t st);
cudaError_t launch_combine(const moe_shape& s, const float* y, const float* y_shared,
                           const int32_t* assign_row, const float* topk_w, const float* sgate,
                           float* out, cudaStream_t st);
// Zero-channel compaction (a weight pre-pass; compact.cu).
size_t compact_workspace_bytes(const moe_shape& s);
cudaError_t launch_zero_channel_map(const moe_shape& s, const uint16_t* w_gate_up, int Ic,
                                    char* ws, int32_t** src, int32_t** count, cudaStream_t st);
cudaError_t launch_compact_banks(const moe_shape& s, const uint16_t* w_gate_up,
                                 const uint16_t* w_down, const int32_t* src, int Ic,
                                 uint16_t* gate_up_c, uint16_t* down_c, cudaStream_t st);
// FP8 expert pre-pass (fp8_quant.cu): rows of n bf16 -> E4M3 codes and fp32 row scales.
cudaError_t launch_quantize_fp8_rows(const uint16_t* w, size_t rows, int n, uint8_t* q,
                                     float* scale, int sms, cudaStream_t st);
// Down-projection weights re-encoded as fp16(W * 2^8) (down_f16.cu); n a multiple of 8.
cudaError_t launch_down_to_f16(const uint16_t* w, size_t n, uint16_t* out, uint32_t* status,
                               int sms, cudaStream_t st);
cudaError_t launch_wait_flag(const int32_t* flag, uint64_t timeout_ns, uint32_t* status,
                             cudaStream_t st);

}  // namespace moe
