/*
 * moe.h -- C ABI of the routed Mixture-of-Experts FFN layer for NVIDIA B200 (sm_100a).
 *
 * The layer (Qwen3.8-Flash-Next architecture study, section "MoE: 512 experts behind a
 * width-640 intermediate", layer formula and pipeline diagram):
 *
 *   expert(x) = W_down (SiLU(W_gate x) * W_up x)
 *   MoE(x)    = sum_{e in top-k} p_e expert_e(x) + sigmoid(w_shared . x) shared(x)
 *
 * computed in the page's five stages "Router [T, 512] -> Top 10 + normalize ->
 * Dispatch R tokens -> Grouped expert GEMMs -> Weighted combine + gated shared expert".
 * Each stage is one entry point below; moe_layer_forward runs all of them.
 *
 * Conventions shared by every call
 * --------------------------------
 * - Memory: every pointer argument is DEVICE memory unless its description says HOST.
 *   The caller allocates and owns every buffer, including the workspace; the library
 *   never allocates, frees or synchronises on these calls (moe_device_status and the
 *   profiling calls excepted, which synchronise the given stream).
 * - Types: "bf16" buffers hold IEEE bfloat16 bit patterns (2 bytes), "fp32" IEEE float.
 *   Every matrix is dense and row-major with the stated shape; no padding or strides.
 * - Alignment: every device pointer must be 16-byte aligned (MOE_ERR_INVALID_ARG
 *   otherwise).
 * - Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   Work is enqueued asynchronously; outputs are valid once the stream reaches that point.
 *   The calls make no host-device synchronisation and can be captured in a CUDA graph.
 * - Errors: a call returns a moe_status synchronously. Argument errors are reported
 *   before anything is enqueued. MOE_ERR_CUDA reports a launch error. Errors found by a
 *   kernel while it runs (an expert id out of range, a bounded wait that ran out) are
 *   recorded in the workspace's status word and reported by moe_device_status.
 *   No C++ exception crosses this boundary.
 * - Empty input: T == 0 is valid and enqueues nothing.
 * - Shape limits: 1 <= k <= min(E, 32), E <= 1024, H, I, Is multiples of 64,
 *   T <= 2^20, T*k < 2^31. Other shapes give MOE_ERR_UNSUPPORTED.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,         /* null/misaligned pointer, bad enum value       */
  MOE_ERR_UNSUPPORTED = 2,         /* shape outside the limits above                */
  MOE_ERR_WORKSPACE_TOO_SMALL = 3, /* ws_bytes < moe_workspace_bytes(shape)         */
  MOE_ERR_CUDA = 4,                /* a CUDA runtime call or launch failed          */
  MOE_ERR_DEVICE_TIMEOUT = 5,      /* a bounded device-side wait gave up            */
  MOE_ERR_DEVICE_BOUNDS = 6,       /* a kernel met an expert id outside [0, E)      */
  MOE_ERR_DEVICE_RANGE = 7         /* a value saturated to fit fp16 (down operands),
                                      or h held inf/NaN (FP8 layer)                 */
} moe_status;

/* Layer shape. T tokens, hidden size H, E routed experts, k experts per token,
 * routed-expert intermediate size I, shared-expert intermediate size Is. */
typedef struct moe_shape {
  int32_t T, H, E, k, I, Is;
} moe_shape;

/* Layer weights (device memory, owned by the caller, read only). */
typedef struct moe_weights {
  const float* w_router;    /* fp32 [E][H]   router matrix                                 */
  const float* router_bias; /* fp32 [E]      added to the logits, or NULL for none         */
  const void* w_gate_up;    /* bf16 [E][2I][H] per expert: rows 0..I-1 gate, I..2I-1 up   */
  const void* w_down;       /* bf16 [E][H][I]  per expert down projection                 */
  const void* ws_gate_up;   /* bf16 [2Is][H]   shared expert gate|up                      */
  const void* ws_down;      /* bf16 [H][Is]    shared expert down                          */
  const void* w_shared_gate;/* bf16 [H]        shared-expert output gate vector            */
  /* Optional fp16 down operands from moe_prepare_down_f16, or NULL (both or neither): */
  const void* w_down_f16;   /* fp16 [E][H][I]  fp16(w_down * 2^8)                          */
  const void* ws_down_f16;  /* fp16 [H][Is]    fp16(ws_down * 2^8)                         */
} moe_weights;

/* Grouped-GEMM variant used by moe_grouped_swiglu and moe_layer_forward. */
typedef enum moe_variant {
  MOE_VARIANT_AUTO = 0,   /* tensor-core kernels where the shape allows (I, Is multiples of
                             128, H of 256), else the streaming kernels: the down GEMM on
                             CTA pairs; the gate|up GEMM on CTA pairs when the batch
                             averages at least 16 routed rows per expert (T*k >= 16*E),
                             else one CTA per tile                                        */
  MOE_VARIANT_STREAM = 1, /* weight-streaming CUDA-core kernels                             */
  MOE_VARIANT_TC = 2,     /* tcgen05/TMEM grouped GEMMs fed by TMA, one CTA per tile (falls
                             back to streaming for shapes they do not support)             */
  MOE_VARIANT_TC2 = 3     /* the same GEMMs on CTA pairs (tcgen05.mma.cta_group::2, M = 256,
                             each SM holding half of the token tile; same fallback)        */
} moe_variant;

/* Kernel ids for the measurement calls below. */
typedef enum moe_kernel {
  MOE_K_ROUTER_LOGITS = 0, /* router logits                                   */
  MOE_K_ROUTER_TOPK = 1,   /* softmax / top-k / renormalise / shared gate     */
  MOE_K_PERMUTE = 2,       /* the three dispatch kernels, counted together    */
  MOE_K_GATE_UP = 3,       /* grouped gate|up GEMM with the SwiGLU epilogue    */
  MOE_K_DOWN = 4,          /* grouped down GEMM (+ fused weighted combine)     */
  MOE_K_COMBINE = 5,       /* unpermute + weighted combine (staged path)       */
  MOE_K_OTHER = 6,         /* helpers (router weight split, waits)             */
  MOE_K_COUNT = 7
} moe_kernel;

/* Bytes of device workspace the calls below need for `shape` (0 on a bad shape).
 * One workspace serves all calls; its first bytes hold the device status word.
 * The size never decreases as T grows, so a workspace sized for T serves every smaller
 * batch with the same H, E, k, I, Is. Calls that share a workspace must not overlap in
 * time on the GPU. */
size_t moe_workspace_bytes(const moe_shape* shape);

/* Extra bytes moe_layer_forward_host needs on top of moe_workspace_bytes
 * (device staging for x and out). */
size_t moe_host_staging_bytes(const moe_shape* shape);

/* Set the status word of a fresh workspace to zero (enqueued on `stream`).
 * Call once after allocating a workspace; moe_device_status clears it afterwards. */
moe_status moe_workspace_init(void* ws, size_t ws_bytes, void* stream);

/*
 * Stages 1-2: "Router [T, 512]" and "Top 10 + normalize" (MoE section, pipeline
 * diagram; "Selected router probabilities are normalized"; "Routing uses FP32 softmax").
 *   logits[t,e] = x[t,:] . w_router[e,:] (+ router_bias[e])    fp32
 *   topk_ids[t,:] = the k largest logits, larger first, equal logits -> lower index
 *   topk_w[t,j]   = softmax(logits[t])[id_j] / sum_j softmax(logits[t])[id_j]
 *   shared_gate[t]= sigmoid(x[t,:] . w_shared_gate)                fp32
 *   gap[t]        = (k-th largest logit) - ((k+1)-th largest), +inf when k == E
 * x: bf16 [T][H]. topk_ids: int32 [T][k]; topk_w: fp32 [T][k]; shared_gate: fp32 [T];
 * gap: fp32 [T] or NULL. Uses weights->w_router, router_bias, w_shared_gate only.
 */
moe_status moe_router_topk(const moe_shape* shape, const void* x, const moe_weights* weights,
                           int32_t* topk_ids, float* topk_w, float* shared_gate, float* gap,
                           void* ws, size_t ws_bytes, void* stream);

/*
 * Stage 3: "Dispatch R tokens" (MoE pipeline diagram; R = kT token-expert assignments,
 * section "Follow the kernels, one layer at a time"). A stable counting sort of the
 * T*k assignments by expert:
 *   offsets[e]..offsets[e+1]-1 are the packed rows of expert e   (int32 [E+1])
 *   sorted_token[p] = token of packed row p, ascending inside an expert (int32 [T*k])
 *   assign_row[t*k+j] = packed row of assignment (t, j)          (int32 [T*k])
 * topk_ids: int32 [T][k], each row k distinct ids in [0, E). An id outside [0, E) is
 * skipped and flagged (MOE_ERR_DEVICE_BOUNDS from moe_device_status); the outputs are
 * then unspecified. Also records the dispatch in the workspace for the grouped GEMMs.
 */
moe_status moe_permute(const moe_shape* shape, const int32_t* topk_ids, int32_t* offsets,
                       int32_t* sorted_token, int32_t* assign_row, void* ws, size_t ws_bytes,
                       void* stream);

/*
 * moe_permute without a workspace, for callers that cannot allocate device memory: code
 * that runs where an allocation would block or is not allowed (inside a real-time serving
 * loop that must not enter the allocator, a plugin host that hands a custom op only its
 * input and output buffers, a process whose memory pool is already fully reserved).
 * The pages have no counterpart; it computes exactly what moe_permute computes (same
 * offsets, sorted_token, assign_row), with the same argument meaning and layout.
 * Its scratch is a fixed 640 KB array inside this library, held on every GPU that loads
 * the library until the process exits; it allocates nothing and calls no allocating
 * routine. Limit: ceil(T/256) * E <= 16384 (for example T <= 8192 with E = 512); larger
 * shapes return MOE_ERR_UNSUPPORTED (use moe_permute with a workspace). The first call on
 * a device looks up the array's device address; make that first call before capturing a
 * stream into a CUDA graph. The address is kept until the process exits: do not call this
 * after a cudaDeviceReset (or another teardown of the device's primary context) in the
 * same process. All calls share the one array: calls that overlap on the GPU (different
 * streams, or several host threads) race and give wrong results. An id outside [0, E) is
 * skipped and not reported (the array's status word has no reader); offsets[E] then falls
 * short of T*k, which the caller can check.
 */
moe_status moe_permute_noalloc(const moe_shape* shape, const int32_t* topk_ids, int32_t* offsets,
                               int32_t* sorted_token, int32_t* assign_row, void* stream);

/*
 * Stage 4: "Grouped expert GEMMs" with the layer's expert formula
 * expert(x) = W_down(SiLU(W_gate x) * W_up x). Unweighted per-assignment outputs:
 *   y[p,:]        = expert_{e(p)}(x[sorted_token[p],:])   fp32 [T*k][H] (packed order)
 *   y_shared[t,:] = shared(x[t,:])                         fp32 [T][H]
 * sorted_token / offsets as produced by moe_permute. The intermediate
 * h = SiLU(gate) * up is carried as a pair of bf16 values (hi = bf16(h), lo = bf16(h - hi),
 * about 16 significant bits) into the down projection; accumulation is fp32.
 * With weights->ws_gate_up and weights->ws_down both NULL there is no shared expert in this
 * call (the routed experts of an expert-parallel owner, below): y_shared is not written and
 * may be NULL.
 */
moe_status moe_grouped_swiglu(const moe_shape* shape, const void* x, const int32_t* sorted_token,
                              const int32_t* offsets, const moe_weights* weights, float* y,
                              float* y_shared, void* ws, size_t ws_bytes, void* stream);

/*
 * Stage 5: "Weighted combine + gated shared expert" (layer formula):
 *   out[t,:] = sum_{j<k} topk_w[t,j] * y[assign_row[t*k+j],:] + shared_gate[t] * y_shared[t,:]
 * summed in that order, fp32. out: fp32 [T][H]. Needs no workspace.
 */
moe_status moe_unpermute_combine(const moe_shape* shape, const float* y, const float* y_shared,
                                 const int32_t* assign_row, const float* topk_w,
                                 const float* shared_gate, float* out, void* stream);

/*
 * The whole layer, MoE(x) for every token (all five stages). x: bf16 [T][H];
 * out: fp32 [T][H]. topk_ids / topk_w / gap: optional copies of the routing
 * (int32 [T][k], fp32 [T][k], fp32 [T]) or NULL. The down GEMM adds its weighted
 * output and the gated shared expert straight into `out` (fp32 atomic adds), so the
 * order of the k+1 additions per element is not fixed between runs.
 */
moe_status moe_layer_forward(const moe_shape* shape, const void* x, const moe_weights* weights,
                             float* out, int32_t* topk_ids, float* topk_w, float* gap, void* ws,
                             size_t ws_bytes, void* stream);

/*
 * moe_layer_forward with HOST activations: x_host (bf16 [T][H], HOST memory, pinned
 * for asynchronous copies) is copied to the device, the layer runs, and out_host
 * (fp32 [T][H], HOST memory) receives the result; all enqueued on `stream` (the host
 * buffers must stay valid until the stream reaches that point). The workspace must
 * hold moe_workspace_bytes + moe_host_staging_bytes.
 */
moe_status moe_layer_forward_host(const moe_shape* shape, const void* x_host,
                                  const moe_weights* weights, float* out_host, void* ws,
                                  size_t ws_bytes, void* stream);

/*
 * Expert parallelism ("Qwen3.8-Flash-Next" architecture study, section "Expert
 * parallelism": the routed experts are split across GPUs, and dispatch and combine
 * exchange token activations across expert owners). The E routed experts are split into G
 * contiguous slices of E_local = E / G, slice d owned by rank d. moe_permute's packed order
 * (experts ascending) is then already grouped by owner. The exchange itself, an all-to-all
 * of variable-size blocks of rows, belongs to the caller's collective library (NCCL through
 * torch.distributed in the Python binding); these calls move rows and plans on one GPU
 * around it. One layer step on rank r:
 *   holder:  moe_router_topk, moe_permute (all E experts), moe_ep_counts,
 *            moe_gather_rows(index = sorted_token)            -> send buffer
 *   exchange counts [G][E_local], then rows (sizes from the counts)
 *   owner:   moe_ep_regroup, moe_grouped_swiglu(T = received rows, k = 1, E = E_local,
 *            x = received rows, sorted_token = src_index, no shared expert),
 *            moe_scatter_rows(index = src_index)            -> rows back in received order
 *   exchange the output rows back (reverse sizes)
 *   holder:  shared expert (moe_grouped_swiglu with every routed group empty) and
 *            moe_unpermute_combine on the returned rows, which are in its packed order.
 *
 * moe_ep_counts: offsets int32 [G*E_local + 1] from moe_permute -> counts int32
 *   [G][E_local] (rows for owner d's local expert e) and rows int32 [G] (all rows for owner d).
 * moe_gather_rows: out[p] = x[index[p]] for p < rows; x, out bf16 rows of H elements (H a
 *   multiple of 8); index int32 in [0, n_src).
 * moe_ep_regroup: on an owner, recv_counts int32 [G][E_local] (rows source s sent for local
 *   expert e; the received buffer holds, source by source, each source's rows expert by
 *   expert). Writes offsets int32 [E_local + 1] of the expert-major order, src_index int32
 *   [capacity] (expert-major row p is received row src_index[p]) and, if not NULL,
 *   src_rows int32 [G] (rows received from each source). G * E_local <= 1024; more rows
 *   than capacity are dropped and flagged.
 * moe_scatter_rows: out[index[p]] = y[p] for p < rows; y, out fp32 rows of H elements (H a
 *   multiple of 4); index int32 in [0, n_dst).
 * ws (optional, may be NULL): a workspace whose status word records an index or count out
 * of range (moe_device_status then reports MOE_ERR_DEVICE_BOUNDS); such rows are skipped.
 * Errors: MOE_ERR_INVALID_ARG (bad size, null or misaligned pointer), MOE_ERR_UNSUPPORTED,
 * MOE_ERR_CUDA. All asynchronous on `stream`.
 */
moe_status moe_ep_counts(int32_t G, int32_t E_local, const int32_t* offsets, int32_t* counts,
                         int32_t* rows, void* stream);
moe_status moe_gather_rows(int64_t rows, int32_t H, const void* x, int64_t n_src,
                           const int32_t* index, void* out, void* ws, size_t ws_bytes,
                           void* stream);
moe_status moe_ep_regroup(int32_t G, int32_t E_local, const int32_t* recv_counts,
                          int64_t capacity, int32_t* offsets, int32_t* src_index,
                          int32_t* src_rows, void* ws, size_t ws_bytes, void* stream);
moe_status moe_scatter_rows(int64_t rows, int32_t H, const float* y, int64_t n_dst,
                            const int32_t* index, float* out, void* ws, size_t ws_bytes,
                            void* stream);

/*
 * Zero-channel compaction of structurally sparse routed experts: a weight pre-pass run once
 * when the weights are loaded, not a step of the layer.
 * Source: "Qwen3.8-2.4T-A95B" discussion #29, tensor table. The GGUF zero fractions show
 * 71.0 % of the ffn_gate_exps and ffn_up_exps rows of a 2.4T layer as exact zeros.
 * Channel c of routed expert e is dead when gate row W_gate,e[c,:] or up row W_up,e[c,:]
 * is all zero (every bf16 element +0 or -0). Then h_c = SiLU(g_c) * u_c = 0 exactly, and
 * down column c adds nothing to expert(x) = W_down (SiLU(W_gate x) * W_up x).
 * Compaction keeps each expert's live channels in their original order, packed to the
 * front of a common width I_c, with zeros after them. The layer then runs on the
 * compacted bank with moe_shape.I = I_c. Its outputs are those of the full bank up to
 * the order of fp32 additions. Gate/up/down bytes and FLOPs scale by I_c / I.
 * The shared expert is not touched.
 *
 * moe_compact_workspace_bytes: scratch size for the two calls below (caller-owned device
 *   memory, 16-byte aligned; about 5*E*I + 4*E bytes). 0 for an invalid shape.
 * moe_zero_channel_count: scans w_gate_up (bf16 [E][2I][H]) and writes to *max_live (host
 *   int32) the largest live-channel count of any expert. It SYNCHRONISES `stream` (the
 *   count is read back); do not call it inside a stream capture.
 * moe_compact_zero_channels: writes gate_up_c (bf16 [E][2*I_c][H], rows 0..I_c-1 gate,
 *   I_c..2*I_c-1 up) and down_c (bf16 [E][H][I_c]) from w_gate_up and w_down (bf16
 *   [E][H][I]); asynchronous on `stream`. I_c must be a multiple of 64, at most I, and at
 *   least the count from moe_zero_channel_count. The tensor-core layer kernels also need a
 *   multiple of 128, so round the count up to 128. If some expert has more live channels
 *   than I_c, its extra channels are dropped and the bounds flag is set in the
 *   workspace's status word; moe_device_status(ws, ...) reports it as
 *   MOE_ERR_DEVICE_BOUNDS. Errors: MOE_ERR_INVALID_ARG (null or misaligned pointer, bad
 *   I_c), MOE_ERR_WORKSPACE_TOO_SMALL, MOE_ERR_CUDA.
 */
size_t moe_compact_workspace_bytes(const moe_shape* shape);
moe_status moe_zero_channel_count(const moe_shape* shape, const void* w_gate_up,
                                  int32_t* max_live, void* ws, size_t ws_bytes, void* stream);
moe_status moe_compact_zero_channels(const moe_shape* shape, const void* w_gate_up,
                                     const void* w_down, int32_t I_c, void* gate_up_c,
                                     void* down_c, void* ws, size_t ws_bytes, void* stream);

/*
 * fp16 down operands: a weight pre-pass, run once when the weights are loaded. The down
 * projection y = W_down h can take h as one fp16 value per element (11 significant bits)
 * instead of the bf16 pair hi + lo (16 bits): one MMA per K step instead of two, and down
 * tiles of up to 256 token rows. The tensor core's f16 MMA needs both operands in one
 * format, so the down matrices are re-encoded as W' = fp16(W * 2^8); the layer then stores
 * h' = fp16(h * 2^-8), and W' h' = W h. A bf16 weight w with 2^-25 <= |w| < 256 (or 0) is
 * re-encoded exactly; smaller magnitudes round with an error of at most 2^-33; larger ones
 * saturate and set the range flag. An intermediate |h| above 65504 * 2^8 saturates and sets
 * the range flag too (moe_device_status: MOE_ERR_DEVICE_RANGE).
 * moe_prepare_down_f16: w_down bf16 [E][H][I] -> w_down_f16 fp16 [E][H][I]; ws_down bf16
 *   [H][Is] -> ws_down_f16 fp16 [H][Is]; asynchronous on `stream`. w_down and w_down_f16
 *   may both be NULL (only the shared expert's matrix is re-encoded, which is all the FP8
 *   layer can use). ws (optional, may be NULL) receives the range flag in its status word.
 * Pass the results as moe_weights.w_down_f16 / ws_down_f16: moe_layer_forward,
 * moe_layer_forward_host and moe_grouped_swiglu then use them whenever they take the
 * tensor-core kernels (the down GEMM then runs on CTA pairs); the weight-streaming variant
 * ignores them. Outputs stay fp32 with fp32 accumulation.
 */
moe_status moe_prepare_down_f16(const moe_shape* shape, const void* w_down, const void* ws_down,
                                void* w_down_f16, void* ws_down_f16, void* ws, size_t ws_bytes,
                                void* stream);

/*
 * FP8 routed experts. Source: "Qwen3.8, weights in hand: 98% of a 2.4T model is routed
 * experts", section "What FP8 actually quantizes". The FP8 checkpoint stores the routed
 * experts at one byte per parameter and keeps the router, the shared expert and the
 * shared-expert gate in bf16. The page does not name the 8-bit format or its scaling; this
 * library reads it as E4M3 codes (bias 7, largest finite 448, 0x7F/0xFF NaN) with one fp32
 * scale per weight row:
 *   scale = amax_row / 448 (fp32 division; 0 for an all-zero row)
 *   code  = E4M3 round-to-nearest-even of (w / scale) (fp32 division), clamped to +-448
 * and the weight the layer uses is decode(code) * scale. Both GEMMs run E4M3 MMAs on the
 * codes; the token operand goes in as exact E4M3 pieces with a power-of-two row scale: x as
 * two (its bf16 value exactly, for elements within 2^9 of the row's largest), h as four
 * (within 2^-16 of each element: the precision of the bf16 layer's hi + lo pair). fp32
 * accumulation and output.
 *
 * moe_fp8_experts: q_gate_up uint8 [E][2I][H] (rows 0..I-1 gate, I..2I-1 up), s_gate_up
 *   fp32 [E][2I], q_down uint8 [E][H][I], s_down fp32 [E][H]. Device pointers, 16-byte
 *   aligned, caller-owned.
 * moe_quantize_fp8_experts: the weight pre-pass (run once at load time), bf16 w_gate_up
 *   [E][2I][H] and w_down [E][H][I] -> the four arrays above; asynchronous on `stream`.
 *   Errors: MOE_ERR_INVALID_ARG (null or misaligned pointer), MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA.
 * moe_layer_forward_fp8: moe_layer_forward with the routed experts taken from `experts`
 *   (weights->w_gate_up and weights->w_down are not read and may be NULL). With
 *   weights->ws_down_f16 given (moe_prepare_down_f16 with no routed pair), the shared
 *   expert's down GEMM takes h's shared rows as one fp16 value (11 significant bits)
 *   instead of the pair. Any batch size, with I and Is multiples of 128 and H of 256 on
 *   sm_100; otherwise MOE_ERR_UNSUPPORTED. Same outputs, workspace and errors as
 *   moe_layer_forward.
 */
typedef struct moe_fp8_experts {
  const void* q_gate_up;
  const float* s_gate_up;
  const void* q_down;
  const float* s_down;
} moe_fp8_experts;

moe_status moe_quantize_fp8_experts(const moe_shape* shape, const void* w_gate_up,
                                    const void* w_down, void* q_gate_up, float* s_gate_up,
                                    void* q_down, float* s_down, void* stream);
moe_status moe_layer_forward_fp8(const moe_shape* shape, const void* x,
                                 const moe_weights* weights, const moe_fp8_experts* experts,
                                 float* out, int32_t* topk_ids, float* topk_w, float* gap,
                                 void* ws, size_t ws_bytes, void* stream);

/* Grouped-GEMM variant. moe_workspace_set_variant chooses it for the calls made with the
 * workspace `ws` (its address is the key; moe_workspace_init clears the choice, so a new
 * workspace allocated at a reused address starts from the default). moe_set_variant sets
 * the process-wide default, used by workspaces without a choice of their own (initially
 * AUTO). Both take effect at the next call; neither touches the GPU. */
moe_status moe_set_variant(moe_variant variant);
moe_status moe_workspace_set_variant(void* ws, size_t ws_bytes, moe_variant variant);

/* Synchronise `stream`, read the workspace status word (MOE_OK, MOE_ERR_DEVICE_BOUNDS,
 * MOE_ERR_DEVICE_TIMEOUT or MOE_ERR_DEVICE_RANGE), and clear it. `detail` (HOST, may be NULL) receives
 * the raw flag bits. */
moe_status moe_device_status(void* ws, size_t ws_bytes, void* stream, uint32_t* detail);

/* Failure-detection check: enqueue a kernel that waits for *flag != 0 (device int32)
 * for at most timeout_ns nanoseconds (capped at 10 s), then records MOE_ERR_DEVICE_TIMEOUT in the
 * workspace status word and returns. The wait is the same bounded wait the pipelined
 * kernels use. Never hangs. */
moe_status moe_debug_wait_flag(const int32_t* flag, uint64_t timeout_ns, void* ws,
                               size_t ws_bytes, void* stream);

/* Measurement: while enabled, every kernel launch records a CUDA event pair on its
 * stream (launches into a stream that is being captured into a CUDA graph are not
 * recorded). moe_profile_collect synchronises those events and returns, per moe_kernel
 * id, the summed device time in ms (HOST float[MOE_K_COUNT]) and the launch counts
 * (HOST int32[MOE_K_COUNT]), then forgets them. At most 65536 launches are recorded. */
moe_status moe_profile_enable(int32_t on);
moe_status moe_profile_collect(float* total_ms, int32_t* launches);

/* Number of kernels this library has launched since it was loaded. */
uint64_t moe_launch_count(void);

/* Short text for a status code (static storage). */
const char* moe_status_string(moe_status status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
