// moe_api.cu -- the C ABI declared in include/moe.h: argument validation, workspace layout,
// variant choice and the order of kernel launches for each stage of the layer
// (Qwen3.8-Flash-Next architecture study, MoE pipeline "Router -> Top 10 + normalize ->
// Dispatch R tokens -> Grouped expert GEMMs -> Weighted combine + gated shared expert").
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "moe_internal.h"
#include "tc_gemm.h"

namespace moe {

Layout layout(const moe_shape& s) {
  Layout L{};
  const size_t T = (size_t)s.T, E = (size_t)s.E, k = (size_t)s.k, H = (size_t)s.H;
  const size_t R = T * k;
  L.nblk = (int)((T + kPermBlock - 1) / kPermBlock);
  if (L.nblk < 1) L.nblk = 1;
  L.ldh = s.I > s.Is ? s.I : s.Is;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    size_t at = o;
    o = align_up(o + (bytes ? bytes : 1), 256);
    return at;
  };
  L.status = take(64 * sizeof(uint32_t));
  // below 512 tokens the router keeps kRouterSplits partial sums per logit; the region is
  // sized so that the workspace never shrinks as T grows (a workspace for T serves every
  // T' <= T)
  const size_t small_max = (size_t)kRouterSplits * 511;
  const size_t logit_rows = T < 512 ? kRouterSplits * T : (T > small_max ? T : small_max);
  L.logits = take(logit_rows * E * sizeof(float));
  L.wr_split = take(E * 3 * H * sizeof(uint16_t));
  L.ids = take(R * sizeof(int32_t));
  L.w = take(R * sizeof(float));
  L.sgate = take(T * sizeof(float));
  L.gap = take(T * sizeof(float));
  L.blk_mask = take((size_t)L.nblk * E * 8 * sizeof(uint32_t));
  L.blk_base = take((size_t)L.nblk * E * sizeof(int32_t));
  L.offsets = take((E + 2) * sizeof(int32_t));
  L.sorted_token = take(R * sizeof(int32_t));
  L.sorted_w = take(R * sizeof(float));
  L.assign_row = take(R * sizeof(int32_t));
  L.plan = take(plan_ints(s.E) * sizeof(int32_t));
  L.sched = take(4 * sizeof(int32_t));
  // the FP8 layer reuses it for h's E4M3 pieces and their row scales once gate|up has run
  L.xs = take(std::max(R * H * sizeof(uint16_t), fp8_h_pieces_bytes(s) + R * sizeof(float)));
  L.h_plane = (R + T) * (size_t)L.ldh;
  L.h = take(2 * L.h_plane * sizeof(uint16_t));
  L.total = o;
  return L;
}

// ---------------------------------------------------------------- launch bookkeeping

namespace {

std::atomic<uint64_t> g_launches{0};
std::atomic<int> g_variant{MOE_VARIANT_AUTO};  // process-wide default
// per-workspace choices (moe_workspace_set_variant), keyed by the workspace's address
std::mutex g_ws_variant_mu;
std::unordered_map<const void*, int> g_ws_variant;
std::mutex g_prof_mu;
bool g_prof_on = false;
struct ProfRec {
  int kid;
  cudaEvent_t a, b;
};
std::vector<ProfRec> g_recs;
std::vector<cudaEvent_t> g_pool;
constexpr size_t kMaxProfRecs = 65536;

cudaEvent_t pool_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

}  // namespace

// NVTX range names per moe_kernel id (host ranges around each launch: they show the layer's
// stages on a profiler's timeline and cost a few nanoseconds when no tool is attached)
const char* const kKernelNames[MOE_K_COUNT] = {"moe.router_logits", "moe.router_topk",
                                               "moe.permute",       "moe.gate_up",
                                               "moe.down",          "moe.combine",
                                               "moe.other"};

LaunchScope::LaunchScope(moe_kernel id, cudaStream_t s, int nkernels) : slot(-1), stream(s) {
  g_launches.fetch_add((uint64_t)nkernels, std::memory_order_relaxed);
  nvtxRangePushA(kKernelNames[(int)id < MOE_K_COUNT ? (int)id : MOE_K_OTHER]);
  if (!g_prof_on) return;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (!g_prof_on || g_recs.size() >= kMaxProfRecs) return;
  cudaEvent_t a = pool_event(), b = pool_event();
  if (!a || !b) return;
  cudaEventRecord(a, s);
  slot = (int)g_recs.size();
  g_recs.push_back({(int)id, a, b});
}

LaunchScope::~LaunchScope() {
  nvtxRangePop();
  if (slot < 0) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (slot < (int)g_recs.size()) cudaEventRecord(g_recs[slot].b, stream);
}

}  // namespace moe

using namespace moe;

namespace {

bool aligned16(const void* p) { return p && ((uintptr_t)p & 15u) == 0; }

moe_status check_shape(const moe_shape* s) {
  if (!s) return MOE_ERR_INVALID_ARG;
  if (s->T < 0 || s->H <= 0 || s->E <= 0 || s->k <= 0 || s->I <= 0 || s->Is <= 0)
    return MOE_ERR_INVALID_ARG;
  if (s->E > kMaxE || s->k > kMaxK || s->k > s->E) return MOE_ERR_UNSUPPORTED;
  if (s->H % 64 || s->I % 64 || s->Is % 64) return MOE_ERR_UNSUPPORTED;
  if (s->T > (1 << 20) || (int64_t)s->T * s->k >= ((int64_t)1 << 31)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status check_ws(const moe_shape& s, const void* ws, size_t ws_bytes, size_t extra = 0) {
  if (!aligned16(ws)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < layout(s).total + extra) return MOE_ERR_WORKSPACE_TOO_SMALL;
  return MOE_OK;
}

moe_status check_router_weights(const moe_weights* w) {
  if (!w || !aligned16(w->w_router) || !aligned16(w->w_shared_gate)) return MOE_ERR_INVALID_ARG;
  if (w->router_bias && !aligned16(w->router_bias)) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

moe_status check_expert_weights(const moe_weights* w) {
  if (!w || !aligned16(w->w_gate_up) || !aligned16(w->w_down) || !aligned16(w->ws_gate_up) ||
      !aligned16(w->ws_down))
    return MOE_ERR_INVALID_ARG;
  // the fp16 down operands: both or neither
  if ((w->w_down_f16 || w->ws_down_f16) && (!aligned16(w->w_down_f16) || !aligned16(w->ws_down_f16)))
    return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

int sm_count_host() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

#define MOE_TRY(expr)                     \
  do {                                    \
    moe_status _st = (expr);              \
    if (_st != MOE_OK) return _st;        \
  } while (0)
#define MOE_CUDA(expr) MOE_TRY(cuda_status(expr))

// The variant for calls on workspace `ws`: its own choice if one was set, else the
// process-wide default.
int variant_of(const void* ws) {
  {
    std::lock_guard<std::mutex> lk(g_ws_variant_mu);
    auto it = g_ws_variant.find(ws);
    if (it != g_ws_variant.end()) return it->second;
  }
  return g_variant.load();
}

// Tensor-core variant for this shape? AUTO takes it wherever the shape allows: on B200 it
// streams the activated experts' weights faster than the CUDA-core kernels even at
// decode sizes (a 16-token MMA tile costs nothing next to the weight bytes).
bool use_tc(const moe_shape& s, int v) {
  if (v == MOE_VARIANT_STREAM) return false;
  return tc_supported(s);
}

// CTA-pair kernels for this shape, per GEMM? Measured on B200 (µs per launch, one-CTA /
// pair): the down GEMM is faster on pairs at every size (Flash-Next decode 234 / 220,
// 2.4T-shaped prefill 8001 / 6941); the gate|up GEMM only once the token tiles are wide
// (decode 384 / 393; 2.4T-shaped prefill 6986 / 6921; Flash-Next prefill 780 / 709), which
// AUTO takes as an average of at least 16 routed rows per expert.
bool use_tc2_gate_up(const moe_shape& s, int v) {
  if (v == MOE_VARIANT_TC2) return true;
  return v == MOE_VARIANT_AUTO && (int64_t)s.T * s.k >= 16 * (int64_t)s.E;
}

bool use_tc2_down(int v) { return v == MOE_VARIANT_TC2 || v == MOE_VARIANT_AUTO; }

// Stage 4 on the plan in the workspace: fused (out != NULL) or per-row y / y_shared.
moe_status run_grouped(const moe_shape& s, const Layout& L, char* ws, const uint16_t* x,
                       const int32_t* sorted_token, const float* sorted_w, const float* sgate,
                       const moe_weights& w, float* y, float* y_shared, float* out,
                       cudaStream_t st) {
  const int v = variant_of(ws);
  if (use_tc(s, v)) {
    // fp16 down operands given: h is stored as fp16(h 2^-8) and the down GEMM runs on CTA
    // pairs with one MMA per K step (any tensor-core variant)
    const int f16 = (w.w_down_f16 && w.ws_down_f16) ? 1 : 0;
    if (use_tc2_gate_up(s, v)) MOE_CUDA(launch_tc2_gate_up(s, L, ws, x, sorted_token, w, f16, st));
    else MOE_CUDA(launch_tc_gate_up(s, L, ws, x, sorted_token, w, f16, st));
    if (f16)
      MOE_CUDA(launch_tc2_down_f16(s, L, ws, sorted_token, sorted_w, sgate, w, y, y_shared, out, st));
    else if (use_tc2_down(v))
      MOE_CUDA(launch_tc2_down(s, L, ws, sorted_token, sorted_w, sgate, w, y, y_shared, out, st));
    else
      MOE_CUDA(launch_tc_down(s, L, ws, sorted_token, sorted_w, sgate, w, y, y_shared, out, st));
  } else {
    MOE_CUDA(launch_stream_gate_up(s, L, ws, x, sorted_token, w, st));
    MOE_CUDA(launch_stream_down(s, L, ws, sorted_token, sorted_w, sgate, w, y, y_shared, out, st));
  }
  return MOE_OK;
}

}  // namespace

extern "C" {

size_t moe_workspace_bytes(const moe_shape* shape) {
  if (check_shape(shape) != MOE_OK) return 0;
  return layout(*shape).total;
}

size_t moe_host_staging_bytes(const moe_shape* shape) {
  if (check_shape(shape) != MOE_OK) return 0;
  const size_t n = (size_t)shape->T * shape->H;
  return align_up(n * sizeof(uint16_t), 256) + align_up(n * sizeof(float), 256);
}

moe_status moe_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (!aligned16(ws) || ws_bytes < 256) return MOE_ERR_INVALID_ARG;
  {
    std::lock_guard<std::mutex> lk(g_ws_variant_mu);
    g_ws_variant.erase(ws);
  }
  MOE_CUDA(cudaMemsetAsync(ws, 0, 256, (cudaStream_t)stream));
  return MOE_OK;
}

moe_status moe_router_topk(const moe_shape* shape, const void* x, const moe_weights* weights,
                           int32_t* topk_ids, float* topk_w, float* shared_gate, float* gap,
                           void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check_shape(shape));
  const moe_shape& s = *shape;
  MOE_TRY(check_router_weights(weights));
  if (!aligned16(x) || !aligned16(topk_ids) || !aligned16(topk_w) || !aligned16(shared_gate))
    return MOE_ERR_INVALID_ARG;
  if (gap && !aligned16(gap)) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ws(s, ws, ws_bytes));
  if (s.T == 0) return MOE_OK;
  const Layout L = layout(s);
  char* w = static_cast<char*>(ws);
  cudaStream_t st = (cudaStream_t)stream;
  float* logits = reinterpret_cast<float*>(w + L.logits);
  MOE_CUDA(launch_router_logits(s, L, w, static_cast<const uint16_t*>(x), weights->w_router,
                                logits, st));
  MOE_CUDA(launch_router_topk(s, logits, weights->w_router, weights->router_bias,
                              static_cast<const uint16_t*>(x),
                              static_cast<const uint16_t*>(weights->w_shared_gate), topk_ids,
                              topk_w, shared_gate, gap, nullptr, st));
  return MOE_OK;
}

moe_status moe_permute(const moe_shape* shape, const int32_t* topk_ids, int32_t* offsets,
                       int32_t* sorted_token, int32_t* assign_row, void* ws, size_t ws_bytes,
                       void* stream) {
  MOE_TRY(check_shape(shape));
  const moe_shape& s = *shape;
  if (!aligned16(topk_ids) || !aligned16(offsets) || !aligned16(sorted_token) ||
      !aligned16(assign_row))
    return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ws(s, ws, ws_bytes));
  if (s.T == 0) return MOE_OK;
  const Layout L = layout(s);
  MOE_CUDA(launch_permute(s, L, static_cast<char*>(ws), topk_ids, nullptr, offsets, sorted_token,
                          nullptr, assign_row, (cudaStream_t)stream));
  return MOE_OK;
}

moe_status moe_grouped_swiglu(const moe_shape* shape, const void* x, const int32_t* sorted_token,
                              const int32_t* offsets, const moe_weights* weights, float* y,
                              float* y_shared, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check_shape(shape));
  if (!weights) return MOE_ERR_INVALID_ARG;
  // both shared-expert matrices NULL: routed experts only (y_shared is not written)
  const bool shared = weights->ws_gate_up || weights->ws_down;
  moe_weights wv = *weights;
  moe_shape s = *shape;
  if (!shared) {
    // no tile reads the shared expert's matrices; its tensor maps still need a valid base
    wv.ws_gate_up = wv.w_gate_up;
    wv.ws_down = wv.w_down;
    if (wv.w_down_f16) wv.ws_down_f16 = wv.w_down_f16;
    s.Is = s.I;  // the workspace layout for Is = I is no larger than the caller's
  }
  MOE_TRY(check_expert_weights(&wv));
  if (!aligned16(x) || !aligned16(sorted_token) || !aligned16(offsets) || !aligned16(y) ||
      (shared && !aligned16(y_shared)))
    return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ws(*shape, ws, ws_bytes));
  if (s.T == 0) return MOE_OK;
  const Layout L = layout(s);
  char* w = static_cast<char*>(ws);
  cudaStream_t st = (cudaStream_t)stream;
  MOE_CUDA(launch_plan_from_offsets(s, L, w, offsets, shared ? s.T : 0, st));
  return run_grouped(s, L, w, static_cast<const uint16_t*>(x), sorted_token, nullptr, nullptr, wv,
                     y, shared ? y_shared : nullptr, nullptr, st);
}

moe_status moe_unpermute_combine(const moe_shape* shape, const float* y, const float* y_shared,
                                 const int32_t* assign_row, const float* topk_w,
                                 const float* shared_gate, float* out, void* stream) {
  MOE_TRY(check_shape(shape));
  const moe_shape& s = *shape;
  if (!aligned16(y) || !aligned16(y_shared) || !aligned16(assign_row) || !aligned16(topk_w) ||
      !aligned16(shared_gate) || !aligned16(out))
    return MOE_ERR_INVALID_ARG;
  if (s.T == 0) return MOE_OK;
  MOE_CUDA(launch_combine(s, y, y_shared, assign_row, topk_w, shared_gate, out,
                          (cudaStream_t)stream));
  return MOE_OK;
}

moe_status moe_layer_forward(const moe_shape* shape, const void* x, const moe_weights* weights,
                             float* out, int32_t* topk_ids, float* topk_w, float* gap, void* ws,
                             size_t ws_bytes, void* stream) {
  MOE_TRY(check_shape(shape));
  const moe_shape& s = *shape;
  MOE_TRY(check_router_weights(weights));
  MOE_TRY(check_expert_weights(weights));
  if (!aligned16(x) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  if ((topk_ids && !aligned16(topk_ids)) || (topk_w && !aligned16(topk_w)) ||
      (gap && !aligned16(gap)))
    return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ws(s, ws, ws_bytes));
  if (s.T == 0) return MOE_OK;
  const Layout L = layout(s);
  char* w = static_cast<char*>(ws);
  cudaStream_t st = (cudaStream_t)stream;
  const uint16_t* xb = static_cast<const uint16_t*>(x);
  int32_t* ids = topk_ids ? topk_ids : reinterpret_cast<int32_t*>(w + L.ids);
  float* tw = topk_w ? topk_w : reinterpret_cast<float*>(w + L.w);
  float* sg = reinterpret_cast<float*>(w + L.sgate);
  float* logits = reinterpret_cast<float*>(w + L.logits);
  int32_t* sorted_token = reinterpret_cast<int32_t*>(w + L.sorted_token);
  float* sorted_w = reinterpret_cast<float*>(w + L.sorted_w);

  MOE_CUDA(launch_router_logits(s, L, w, xb, weights->w_router, logits, st));
  MOE_CUDA(launch_router_topk(s, logits, weights->w_router, weights->router_bias, xb,
                              static_cast<const uint16_t*>(weights->w_shared_gate), ids, tw, sg,
                              gap, out /* rows zeroed here, accumulated by the down GEMM */, st));
  MOE_CUDA(launch_permute(s, L, w, ids, tw, reinterpret_cast<int32_t*>(w + L.offsets),
                          sorted_token, sorted_w, reinterpret_cast<int32_t*>(w + L.assign_row),
                          st));
  return run_grouped(s, L, w, xb, sorted_token, sorted_w, sg, *weights, nullptr, nullptr, out, st);
}

moe_status moe_layer_forward_host(const moe_shape* shape, const void* x_host,
                                  const moe_weights* weights, float* out_host, void* ws,
                                  size_t ws_bytes, void* stream) {
  MOE_TRY(check_shape(shape));
  const moe_shape& s = *shape;
  if (!x_host || !out_host) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ws(s, ws, ws_bytes, moe_host_staging_bytes(shape)));
  if (s.T == 0) return MOE_OK;
  const Layout L = layout(s);
  char* w = static_cast<char*>(ws);
  cudaStream_t st = (cudaStream_t)stream;
  const size_t n = (size_t)s.T * s.H;
  void* x_dev = w + L.total;
  float* out_dev = reinterpret_cast<float*>(w + L.total + align_up(n * sizeof(uint16_t), 256));
  MOE_CUDA(cudaMemcpyAsync(x_dev, x_host, n * sizeof(uint16_t), cudaMemcpyHostToDevice, st));
  MOE_TRY(moe_layer_forward(shape, x_dev, weights, out_dev, nullptr, nullptr, nullptr, ws,
                            L.total, stream));
  MOE_CUDA(cudaMemcpyAsync(out_host, out_dev, n * sizeof(float), cudaMemcpyDeviceToHost, st));
  return MOE_OK;
}

size_t moe_compact_workspace_bytes(const moe_shape* shape) {
  if (check_shape(shape) != MOE_OK) return 0;
  return compact_workspace_bytes(*shape);
}

moe_status moe_zero_channel_count(const moe_shape* shape, const void* w_gate_up,
                                  int32_t* max_live, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check_shape(shape));
  const moe_shape& s = *shape;
  if (!aligned16(w_gate_up) || !max_live || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < compact_workspace_bytes(s)) return MOE_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = (cudaStream_t)stream;
  char* w = static_cast<char*>(ws);
  MOE_CUDA(cudaMemsetAsync(w, 0, 256, st));
  int32_t *src = nullptr, *count = nullptr;
  MOE_CUDA(launch_zero_channel_map(s, static_cast<const uint16_t*>(w_gate_up), s.I, w, &src,
                                   &count, st));
  std::vector<int32_t> counts((size_t)s.E);
  MOE_CUDA(cudaMemcpyAsync(counts.data(), count, counts.size() * sizeof(int32_t),
                           cudaMemcpyDeviceToHost, st));
  MOE_CUDA(cudaStreamSynchronize(st));
  int32_t m = 0;
  for (int32_t c : counts) m = c > m ? c : m;
  *max_live = m;
  return MOE_OK;
}

moe_status moe_compact_zero_channels(const moe_shape* shape, const void* w_gate_up,
                                     const void* w_down, int32_t I_c, void* gate_up_c,
                                     void* down_c, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check_shape(shape));
  const moe_shape& s = *shape;
  if (!aligned16(w_gate_up) || !aligned16(w_down) || !aligned16(gate_up_c) ||
      !aligned16(down_c) || !aligned16(ws))
    return MOE_ERR_INVALID_ARG;
  if (I_c <= 0 || I_c % 64 || I_c > s.I) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < compact_workspace_bytes(s)) return MOE_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = (cudaStream_t)stream;
  char* w = static_cast<char*>(ws);
  MOE_CUDA(cudaMemsetAsync(w, 0, 256, st));
  int32_t *src = nullptr, *count = nullptr;
  MOE_CUDA(launch_zero_channel_map(s, static_cast<const uint16_t*>(w_gate_up), I_c, w, &src,
                                   &count, st));
  MOE_CUDA(launch_compact_banks(s, static_cast<const uint16_t*>(w_gate_up),
                                static_cast<const uint16_t*>(w_down), src, I_c,
                                static_cast<uint16_t*>(gate_up_c), static_cast<uint16_t*>(down_c),
                                st));
  return MOE_OK;
}

moe_status moe_prepare_down_f16(const moe_shape* shape, const void* w_down, const void* ws_down,
                                void* w_down_f16, void* ws_down_f16, void* ws, size_t ws_bytes,
                                void* stream) {
  MOE_TRY(check_shape(shape));
  const moe_shape& s = *shape;
  // the routed pair may be left out (both NULL): the FP8 layer needs only the shared one
  const bool routed = w_down || w_down_f16;
  if ((routed && (!aligned16(w_down) || !aligned16(w_down_f16))) || !aligned16(ws_down) ||
      !aligned16(ws_down_f16))
    return MOE_ERR_INVALID_ARG;
  if (ws && (!aligned16(ws) || ws_bytes < 256)) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  uint32_t* status = static_cast<uint32_t*>(ws);
  const int sms = sm_count_host();
  if (routed)
    MOE_CUDA(launch_down_to_f16(static_cast<const uint16_t*>(w_down), (size_t)s.E * s.H * s.I,
                                static_cast<uint16_t*>(w_down_f16), status, sms, st));
  MOE_CUDA(launch_down_to_f16(static_cast<const uint16_t*>(ws_down), (size_t)s.H * s.Is,
                              static_cast<uint16_t*>(ws_down_f16), status, sms, st));
  return MOE_OK;
}

moe_status moe_quantize_fp8_experts(const moe_shape* shape, const void* w_gate_up,
                                    const void* w_down, void* q_gate_up, float* s_gate_up,
                                    void* q_down, float* s_down, void* stream) {
  MOE_TRY(check_shape(shape));
  const moe_shape& s = *shape;
  if (!aligned16(w_gate_up) || !aligned16(w_down) || !aligned16(q_gate_up) ||
      !aligned16(s_gate_up) || !aligned16(q_down) || !aligned16(s_down))
    return MOE_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  int dev = 0, sms = 148;
  MOE_CUDA(cudaGetDevice(&dev));
  MOE_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  MOE_CUDA(launch_quantize_fp8_rows(static_cast<const uint16_t*>(w_gate_up),
                                    (size_t)s.E * 2 * s.I, s.H, static_cast<uint8_t*>(q_gate_up),
                                    s_gate_up, sms, st));
  MOE_CUDA(launch_quantize_fp8_rows(static_cast<const uint16_t*>(w_down), (size_t)s.E * s.H, s.I,
                                    static_cast<uint8_t*>(q_down), s_down, sms, st));
  return MOE_OK;
}

moe_status moe_layer_forward_fp8(const moe_shape* shape, const void* x, const moe_weights* weights,
                                 const moe_fp8_experts* experts, float* out, int32_t* topk_ids,
                                 float* topk_w, float* gap, void* ws, size_t ws_bytes,
                                 void* stream) {
  MOE_TRY(check_shape(shape));
  const moe_shape& s = *shape;
  MOE_TRY(check_router_weights(weights));
  if (!aligned16(weights->ws_gate_up) || !aligned16(weights->ws_down)) return MOE_ERR_INVALID_ARG;
  if (weights->ws_down_f16 && !aligned16(weights->ws_down_f16)) return MOE_ERR_INVALID_ARG;
  if (!experts || !aligned16(experts->q_gate_up) || !aligned16(experts->s_gate_up) ||
      !aligned16(experts->q_down) || !aligned16(experts->s_down))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  if ((topk_ids && !aligned16(topk_ids)) || (topk_w && !aligned16(topk_w)) ||
      (gap && !aligned16(gap)))
    return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ws(s, ws, ws_bytes));
  if (s.T == 0) return MOE_OK;
  if (!tc8_supported(s)) return MOE_ERR_UNSUPPORTED;
  const Layout L = layout(s);
  char* w = static_cast<char*>(ws);
  cudaStream_t st = (cudaStream_t)stream;
  const uint16_t* xb = static_cast<const uint16_t*>(x);
  int32_t* ids = topk_ids ? topk_ids : reinterpret_cast<int32_t*>(w + L.ids);
  float* tw = topk_w ? topk_w : reinterpret_cast<float*>(w + L.w);
  float* sg = reinterpret_cast<float*>(w + L.sgate);
  float* logits = reinterpret_cast<float*>(w + L.logits);
  int32_t* sorted_token = reinterpret_cast<int32_t*>(w + L.sorted_token);
  float* sorted_w = reinterpret_cast<float*>(w + L.sorted_w);

  MOE_CUDA(launch_router_logits(s, L, w, xb, weights->w_router, logits, st));
  MOE_CUDA(launch_router_topk(s, logits, weights->w_router, weights->router_bias, xb,
                              static_cast<const uint16_t*>(weights->w_shared_gate), ids, tw, sg,
                              gap, out /* rows zeroed here, accumulated by the down GEMM */, st));
  MOE_CUDA(launch_permute(s, L, w, ids, tw, reinterpret_cast<int32_t*>(w + L.offsets),
                          sorted_token, sorted_w, reinterpret_cast<int32_t*>(w + L.assign_row),
                          st));
  MOE_CUDA(launch_tc8_gate_up(s, L, w, xb, sorted_token, *weights, *experts, st));
  MOE_CUDA(launch_tc8_down(s, L, w, sorted_token, sorted_w, sg, *weights, *experts, out, st));
  return MOE_OK;
}

static bool valid_variant(moe_variant v) {
  return v == MOE_VARIANT_AUTO || v == MOE_VARIANT_STREAM || v == MOE_VARIANT_TC ||
         v == MOE_VARIANT_TC2;
}

moe_status moe_gather_rows(int64_t rows, int32_t H, const void* x, int64_t n_src,
                           const int32_t* index, void* out, void* ws, size_t ws_bytes,
                           void* stream) {
  if (rows < 0 || n_src < 0 || H <= 0 || H % 8) return MOE_ERR_INVALID_ARG;
  if (ws && (!aligned16(ws) || ws_bytes < 256)) return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  if (!aligned16(x) || !aligned16(index) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  MOE_CUDA(launch_gather_rows_bf16(static_cast<const uint16_t*>(x), index, rows, n_src, H,
                                   static_cast<uint16_t*>(out), static_cast<uint32_t*>(ws),
                                   sm_count_host(), (cudaStream_t)stream));
  return MOE_OK;
}

moe_status moe_scatter_rows(int64_t rows, int32_t H, const float* y, int64_t n_dst,
                            const int32_t* index, float* out, void* ws, size_t ws_bytes,
                            void* stream) {
  if (rows < 0 || n_dst < 0 || H <= 0 || H % 4) return MOE_ERR_INVALID_ARG;
  if (ws && (!aligned16(ws) || ws_bytes < 256)) return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  if (!aligned16(y) || !aligned16(index) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  MOE_CUDA(launch_scatter_rows_f32(y, index, rows, n_dst, H, out, static_cast<uint32_t*>(ws),
                                   sm_count_host(), (cudaStream_t)stream));
  return MOE_OK;
}

moe_status moe_ep_counts(int32_t G, int32_t E_local, const int32_t* offsets, int32_t* counts,
                         int32_t* rows, void* stream) {
  if (G <= 0 || E_local <= 0) return MOE_ERR_INVALID_ARG;
  if ((int64_t)G * E_local > kMaxE) return MOE_ERR_UNSUPPORTED;
  if (!aligned16(offsets) || !aligned16(counts) || !aligned16(rows)) return MOE_ERR_INVALID_ARG;
  MOE_CUDA(launch_ep_counts(offsets, G, E_local, counts, rows, (cudaStream_t)stream));
  return MOE_OK;
}

moe_status moe_ep_regroup(int32_t G, int32_t E_local, const int32_t* recv_counts,
                          int64_t capacity, int32_t* offsets, int32_t* src_index,
                          int32_t* src_rows, void* ws, size_t ws_bytes, void* stream) {
  if (G <= 0 || E_local <= 0 || capacity < 0) return MOE_ERR_INVALID_ARG;
  if ((int64_t)G * E_local > kMaxE || capacity >= ((int64_t)1 << 31)) return MOE_ERR_UNSUPPORTED;
  if (!aligned16(recv_counts) || !aligned16(offsets) || (capacity > 0 && !aligned16(src_index)) ||
      (src_rows && !aligned16(src_rows)))
    return MOE_ERR_INVALID_ARG;
  if (ws && (!aligned16(ws) || ws_bytes < 256)) return MOE_ERR_INVALID_ARG;
  MOE_CUDA(launch_ep_regroup(recv_counts, G, E_local, capacity, offsets, src_index, src_rows,
                             static_cast<uint32_t*>(ws), (cudaStream_t)stream));
  return MOE_OK;
}

moe_status moe_set_variant(moe_variant variant) {
  if (!valid_variant(variant)) return MOE_ERR_INVALID_ARG;
  g_variant.store((int)variant);
  return MOE_OK;
}

moe_status moe_workspace_set_variant(void* ws, size_t ws_bytes, moe_variant variant) {
  if (!aligned16(ws) || ws_bytes < 256 || !valid_variant(variant)) return MOE_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_ws_variant_mu);
  g_ws_variant[ws] = (int)variant;
  return MOE_OK;
}

moe_status moe_device_status(void* ws, size_t ws_bytes, void* stream, uint32_t* detail) {
  if (!aligned16(ws) || ws_bytes < 256) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  MOE_CUDA(cudaStreamSynchronize(st));
  uint32_t flags = 0;
  MOE_CUDA(cudaMemcpyAsync(&flags, ws, sizeof(flags), cudaMemcpyDeviceToHost, st));
  MOE_CUDA(cudaStreamSynchronize(st));
  MOE_CUDA(cudaMemsetAsync(ws, 0, sizeof(uint32_t), st));
  MOE_CUDA(cudaStreamSynchronize(st));
  if (detail) *detail = flags;
  if (flags & kFlagTimeout) return MOE_ERR_DEVICE_TIMEOUT;
  if (flags & kFlagBounds) return MOE_ERR_DEVICE_BOUNDS;
  if (flags & kFlagRange) return MOE_ERR_DEVICE_RANGE;
  return MOE_OK;
}

moe_status moe_debug_wait_flag(const int32_t* flag, uint64_t timeout_ns, void* ws,
                               size_t ws_bytes, void* stream) {
  if (!flag || ((uintptr_t)flag & 3u) || !aligned16(ws) || ws_bytes < 256)
    return MOE_ERR_INVALID_ARG;
  if (timeout_ns > 10000000000ull) timeout_ns = 10000000000ull;  // never wait beyond 10 s
  MOE_CUDA(launch_wait_flag(flag, timeout_ns, static_cast<uint32_t*>(ws), (cudaStream_t)stream));
  return MOE_OK;
}

moe_status moe_profile_enable(int32_t on) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_on = on != 0;
  return MOE_OK;
}

moe_status moe_profile_collect(float* total_ms, int32_t* launches) {
  if (!total_ms || !launches) return MOE_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (int i = 0; i < MOE_K_COUNT; ++i) {
    total_ms[i] = 0.f;
    launches[i] = 0;
  }
  moe_status st = MOE_OK;
  for (const ProfRec& r : g_recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess)
      st = MOE_ERR_CUDA;
    total_ms[r.kid] += ms;
    launches[r.kid] += 1;
    g_pool.push_back(r.a);
    g_pool.push_back(r.b);
  }
  g_recs.clear();
  return st;
}

uint64_t moe_launch_count(void) { return g_launches.load(); }

const char* moe_status_string(moe_status status) {
  switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, bad value)";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape";
    case MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA runtime or launch error";
    case MOE_ERR_DEVICE_TIMEOUT: return "a bounded device wait timed out";
    case MOE_ERR_DEVICE_BOUNDS: return "expert id out of range";
    case MOE_ERR_DEVICE_RANGE:
      return "a value saturated to fit fp16 (down operands) or h held inf/NaN";
  }
  return "unknown status";
}

}  // extern "C"
