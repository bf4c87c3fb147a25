/*
 * moe.h -- C ABI of the B200 (sm_100a) MoE FFN layer library
 *          (libmoe_b200.so, built from sigmoid_top_routing_warp_b200/csrc).
 *
 * The layer is the dots-style fine-grained mixture-of-experts feed-forward
 * block.  Per token x (a row of H values) it computes
 *
 *   logits  L = x W_g^T                        (router, E experts)
 *   scores  s = sigmoid(L)
 *   choice  c = s + b  (b: per-expert bias, used only for choosing; optional
 *           group limit: keep the topk_group groups of E/n_group contiguous
 *           experts with the largest sum of their group_topn best keys)
 *   idx     = the k experts with the largest c (ties: lower expert first),
 *             listed in that order ("slot" order)
 *   w_j     = s[idx_j] / sum_j s[idx_j] (if norm_topk_prob) * rsf
 *   out     = SwiGLU_shared(x) + sum_j w_j * SwiGLU_{idx_j}(x)
 *   SwiGLU_e(x) = W2_e ( SiLU(W_gate,e x) * (W_up,e x) )
 *
 * Sources (web pages, cited by title and section):
 *   "dots3-note 架构深度解析：16B 激活参数的 280B MoE 如何实现高效推理" (mlqm.cn),
 *     section 稀疏激活：Top-8 路由: sigmoid scoring, noaux_tc routing,
 *     norm_topk_prob, 256 routed + 1 shared experts, top-8, hidden 5120,
 *     moe_intermediate_size 1536, BF16 / FP8 weights.
 *   "Xiaohongshu dots3 note Open Source Deep Dive: 280B MoE Multimodal Model"
 *     (happyrock.cloud), §3.1 Expert Routing Mechanism (gate, top-k,
 *     renormalise, shared + weighted routed sum), §3.3 layer diagram,
 *     §8.2 Ascend Adaptation Architecture (FUSED_MC2:
 *     dispatch -> gmm1 -> swiglu -> gmm2 -> combine).
 *   "🤗 Transformers 中的 dots.llm1（Dots1）模型" (blog.gitcode.com), table
 *     MoE 路由与专家相关字段 (n_group, topk_group, norm_topk_prob,
 *     routed_scaling_factor, moe_intermediate_size) and the parallel-plan
 *     paragraph (packed gate_up_proj, grouped_gemm experts).
 *
 * Conventions for every entry point:
 *   - Every data pointer is DEVICE memory owned by the caller.  The library
 *     never allocates, frees or keeps a pointer after the call returns.
 *   - Matrices are row-major and densely packed.  bf16 values are stored as
 *     IEEE bfloat16 (2 bytes); fp32 as IEEE binary32.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream) on the current CUDA device.  No call
 *     synchronises with the host except moe_check_device_status.
 *   - Argument and shape errors are detected on the host before anything is
 *     launched: the call returns a non-zero moe_status_t and
 *     moe_get_last_error() describes it.  Nothing is written in that case.
 *   - Errors the kernels detect (a bounded wait that ran out) are recorded in
 *     a status word inside the workspace; read it with
 *     moe_check_device_status.
 *   - Calls that share a workspace must not overlap on the GPU.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1, /* null pointer, bad shape or option            */
    MOE_ERR_UNSUPPORTED = 2, /* valid layer the kernels do not handle         */
    MOE_ERR_WORKSPACE = 3,   /* workspace smaller than moe_workspace_size()  */
    MOE_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed            */
    MOE_ERR_TIMEOUT = 5      /* a device-side bounded wait ran out           */
} moe_status_t;

typedef enum {
    MOE_DTYPE_BF16 = 0,              /* bf16 activations and weights, fp32 accumulation */
    MOE_DTYPE_FP8_E4M3_BLOCK128 = 1  /* expert weights e4m3 (OCP FP8, 1 byte) with one fp32
                                        scale per 128 x 128 block; expert-GEMM activations
                                        quantised to e4m3 per row and 128 columns
                                        (moe_quantize_act); router stays bf16           */
} moe_dtype_t;

/* Layer description.  Field names follow the Dots1 / DeepSeek-V3 config:
 *   T                      tokens in this call (rows of x), >= 0
 *   H                      hidden size (multiple of 128)
 *   E                      routed experts (n_routed_experts), 1..1024
 *   k                      experts per token (num_experts_per_tok), 1..min(E, 32)
 *   I                      expert intermediate size (moe_intermediate_size),
 *                          multiple of 128
 *   n_shared               shared experts (n_shared_experts) >= 0; they act as
 *                          one SwiGLU of width n_shared * I
 *   n_group, topk_group    group-limited choice (1, 1 = plain top-k)
 *   group_topn             keys summed into a group score (2)
 *   norm_topk_prob         non-zero: divide weights by their sum
 *   routed_scaling_factor  multiplies the routed weights (1.0)
 *   dtype                  moe_dtype_t
 *   flags                  0, or MOE_FLAG_TEST_STALL (tests only)           */
typedef struct {
    int32_t T, H, E, k, I, n_shared;
    int32_t n_group, topk_group, group_topn;
    int32_t norm_topk_prob;
    float routed_scaling_factor;
    int32_t dtype;
    uint32_t flags;
} moe_config_t;

/* Test of the device-side failure path, never set in normal use: the first
 * CTA of the router GEMM leaves its first pipeline stage unfilled, so its
 * bounded wait runs out (about one second), the kernel records a timeout in
 * the workspace status word and returns; moe_check_device_status then
 * reports MOE_ERR_TIMEOUT and the CUDA context stays usable. */
#define MOE_FLAG_TEST_STALL 0x1u

/* A cudaStream_t. */
typedef void* moe_stream_t;

/* Number of stage events moe_forward records when given an event array:
 * event i is recorded when stage i starts, the last one after the last
 * stage.  Stages: 0 router GEMM, 1 router selection, 2 dispatch (histogram,
 * scan, scatter, gather), 3 gate/up GEMM + SwiGLU, 4 down GEMM x weight,
 * 5 combine. */
#define MOE_NUM_STAGES 6

/* Message of the last failed call on this host thread ("" if none). */
const char* moe_get_last_error(void);

/* Bytes of device workspace the calls below need for this configuration
 * (0 if the configuration is invalid; see moe_get_last_error).  The
 * workspace holds logits, routing, the dispatch plan, the gathered
 * activations and the intermediate expert outputs; it must be 256-byte
 * aligned.  Its first 256 bytes hold the status word (word 0) and the
 * persistent GEMMs' tile-claim counters (words 16..63).  Every call that
 * launches a GEMM zeroes the counter words on its stream first, so the
 * workspace needs no zero-fill; the status word must start at zero (a
 * zero-filled buffer, or moe_check_device_status after an error). */
size_t moe_workspace_size(const moe_config_t* cfg);

/* Router: steps a1-a4.  Page: mlqm.cn 稀疏激活 (sigmoid, noaux_tc,
 * norm_topk_prob); Dots1 table (n_group, topk_group, routed_scaling_factor);
 * Deep Dive §3.1 (gate, top-k, renormalise).
 *   x        bf16 [T, H]        tokens
 *   w_router bf16 [E, H]        gate weight (no bias term)
 *   bias     fp32 [E]           noaux_tc selection bias
 *   logits   fp32 [T, E]  out   x W_g^T (fp32 accumulation)
 *   topk_idx int32 [T, k] out   chosen experts in slot order
 *   topk_w   fp32 [T, k]  out   routing weights
 *   ws       workspace (moe_workspace_size bytes)                          */
moe_status_t moe_route(const moe_config_t* cfg, const void* x, const void* w_router,
                       const float* bias, float* logits, int32_t* topk_idx, float* topk_w,
                       void* ws, size_t ws_bytes, moe_stream_t stream);

/* Router selection alone (steps a2-a4) from given fp32 logits [T, E]: the
 * same outputs as moe_route without the GEMM.  No workspace. */
moe_status_t moe_route_from_logits(const moe_config_t* cfg, const float* logits,
                                   const float* bias, int32_t* topk_idx, float* topk_w,
                                   moe_stream_t stream);

/* Dispatch order: step a5 (Deep Dive §8.2 "dispatch").  A counting sort of
 * the T*k (token, slot) pairs by expert, stable in t*k + j, so that the rows
 * of one expert are contiguous and in token order.
 *   topk_idx int32 [T, k]       from moe_route
 *   offsets  int32 [E + 1] out  first sorted row of each expert; offsets[E] = T*k
 *   rows     int32 [T*k]   out  source token of each sorted row
 *   pos      int32 [T*k]   out  sorted row of slot t*k + j                   */
moe_status_t moe_permute(const moe_config_t* cfg, const int32_t* topk_idx, int32_t* offsets,
                         int32_t* rows, int32_t* pos, void* ws, size_t ws_bytes,
                         moe_stream_t stream);

/* Dispatch order like moe_permute, for callers that cannot allocate device
 * memory at all (for example a plugin that its host framework hands only
 * input and output buffers, or a runtime whose memory planner owns the whole
 * HBM budget): no workspace argument.  The pages have no counterpart; this is
 * a convenience of this library.  Its scratch is a fixed array of
 * MOE_PERMUTE_NOALLOC_SCRATCH_INTS int32 values (256 KiB) in the library's
 * device image, held by every GPU that loads the library until exit.
 *   - Sizes whose multi-block pass needs more scratch than that
 *     (ceil(T*k / 2048) * E entries when T*k > 4096) are rejected with
 *     MOE_ERR_UNSUPPORTED before anything is launched.
 *   - The first call on a device looks up the array's device address with
 *     cudaGetSymbolAddress (a one-time set-up per device); make that first
 *     call before any stream capture.  The address belongs to the device's
 *     CUDA context: when that context is replaced (cudaDeviceReset), the next
 *     call sees a new context id and looks the address up again, so that call
 *     too should come before any capture.
 *   - T = 0 writes offsets[0..E] = 0, as moe_permute does.
 *   - Every call shares the one array: calls that overlap on the GPU race on
 *     it and must not be issued.
 *   - It calls no cudaMalloc, cudaFree or allocating library routine.
 * Arguments and outputs as for moe_permute.                                 */
#define MOE_PERMUTE_NOALLOC_SCRATCH_INTS 65536
moe_status_t moe_permute_noalloc(const moe_config_t* cfg, const int32_t* topk_idx,
                                 int32_t* offsets, int32_t* rows, int32_t* pos,
                                 moe_stream_t stream);

/* Expert FFNs: steps a6-a8 (Deep Dive §8.2 "gmm1 -> swiglu -> gmm2"; Dots1
 * packed gate_up_proj).  Gathers the sorted rows, runs every expert's
 * SwiGLU on its rows as one grouped GEMM pair on the tensor cores, and
 * scales each routed row by its routing weight.
 *   x, offsets, rows, pos, topk_w   as above
 *   w13   bf16 [E, 2I, H]   per expert: gate rows 0..I-1, up rows I..2I-1
 *   w2    bf16 [E, H, I]    per expert down projection
 *   w13s  bf16 [2 Is, H]    shared expert gate/up (Is = n_shared * I)
 *   w2s   bf16 [H, Is]      shared expert down
 *   y     bf16 [T*k, H] out w_j * SwiGLU_{idx_j}(x_t) at row pos[t*k + j];
 *         fp32 when k == 1: a token's only routed row is then not averaged
 *         with other experts', and its bf16 rounding alone would be the
 *         largest error term of the output
 *   y_shared fp32 [T, H] out  SwiGLU_shared(x) (may be NULL iff n_shared == 0);
 *            kept in fp32 because, with weight 1, it is the largest term of
 *            the combine and its rounding would dominate the output error
 * For MOE_DTYPE_FP8_E4M3_BLOCK128 the four weight matrices hold e4m3 codes
 * (same shapes, 1 byte each) and the *_scale arguments their fp32 block
 * scales, row-major over 128 x 128 blocks:
 *   w13_scale [E, 2I/128, H/128], w2_scale [E, H/128, I/128],
 *   w13s_scale [2Is/128, H/128], w2s_scale [H/128, Is/128];
 * weight value = code * scale of its block.  For MOE_DTYPE_BF16 the *_scale
 * arguments must be NULL.                                                   */
moe_status_t moe_expert_ffn(const moe_config_t* cfg, const void* x, const int32_t* offsets,
                            const int32_t* rows, const int32_t* pos, const float* topk_w,
                            const void* w13, const float* w13_scale, const void* w2,
                            const float* w2_scale, const void* w13s, const float* w13s_scale,
                            const void* w2s, const float* w2s_scale, void* y, void* y_shared,
                            void* ws, size_t ws_bytes, moe_stream_t stream);

/* Activation quantisation, step a0 of the FP8 layer (FP8 deployment:
 * mlqm.cn 部署实战; the recipe is this library's, see moe_dtype_t): per row
 * and 128 columns, scale = amax / 448 (1 for an all-zero block) and
 * code = e4m3(x / scale), round to nearest even, saturating to +-448; both
 * in correctly rounded binary32.
 *   x bf16 [rows, cols] (cols a multiple of 128), q e4m3 codes [rows, cols]
 *   out, scale fp32 [rows, cols/128] out.  No workspace.                    */
moe_status_t moe_quantize_act(const void* x, int32_t rows, int32_t cols, uint8_t* q, float* scale,
                              moe_stream_t stream);

/* Combine: step a9 (Deep Dive §3.3 "Weighted sum" then shared "add").
 * out_t = sum_{j=0..k-1} y[pos[t*k + j]] + y_shared_t, summed in fp32 in
 * that fixed order (no atomics: bitwise reproducible), rounded once to bf16.
 *   y bf16 [T*k, H] (fp32 when k == 1), pos int32 [T*k], y_shared fp32 [T, H] or NULL,
 *   out bf16 [T, H]                                                        */
moe_status_t moe_combine(const moe_config_t* cfg, const void* y, const int32_t* pos,
                         const void* y_shared, void* out, moe_stream_t stream);

/* The whole layer (steps a1-a9) on one stream, intermediates in `ws`.
 * Arguments as above; out bf16 [T, H].  stage_events: NULL, or
 * MOE_NUM_STAGES + 1 cudaEvent_t handles recorded at the stage boundaries
 * (for timing; the library only records them). */
moe_status_t moe_forward(const moe_config_t* cfg, const void* x, const void* w_router,
                         const float* bias, const void* w13, const float* w13_scale,
                         const void* w2, const float* w2_scale, const void* w13s,
                         const float* w13s_scale, const void* w2s, const float* w2s_scale,
                         void* out, void* ws, size_t ws_bytes, void* const* stage_events,
                         moe_stream_t stream);

/* Pre-norm of the block input.  Pages: Deep Dive §3.3 layer diagram (the
 * "Residual + RMSNorm" box ahead of the MoE FFN); Dots1 config table
 * (rms_norm_eps = 1e-6) and its source notes (variance in fp32, scaling by
 * the reciprocal square root, then the weight).  Per row t, in fp32 with
 * correctly rounded divide and square root:
 *   u[t, :] = bf16( gamma * (h[t, :] * r_t) ),
 *   r_t = 1 / sqrt(sum_i h[t, i]^2 / H + eps)
 *   h     bf16 [T, H]  (16-byte aligned)
 *   gamma bf16 [H]     norm weight
 *   u     bf16 [T, H]  output; must not overlap h
 *   eps   finite, >= 0 (the pages' value is 1e-6)
 * Only cfg->T and cfg->H are read; H must be a multiple of 8. */
moe_status_t moe_rmsnorm(const moe_config_t* cfg, const void* h, const void* gamma, float eps,
                         void* u, moe_stream_t stream);

/* One pre-norm MoE block, out = h + MoE(RMSNorm(h)): the same diagram's
 * "Residual + RMSNorm" -> MoE FFN -> "Residual + Output".  h is the residual
 * stream (bf16 [T, H]); the layer runs on u = RMSNorm(h) (as moe_rmsnorm,
 * kept in the workspace, see moe_workspace_offset item 8), and the combine
 * adds h in the same fp32 sum as the expert outputs, before the single bf16
 * rounding:  out[t] = bf16( sum_j y[pos[t*k+j]] + y_shared[t] + h[t] ).
 * out may be h itself (in-place residual update); otherwise it must not
 * overlap h.  Other arguments as moe_forward; stage 0 of stage_events also
 * covers the norm. */
moe_status_t moe_forward_block(const moe_config_t* cfg, const void* h, const void* gamma,
                               float eps, const void* w_router, const float* bias,
                               const void* w13, const float* w13_scale, const void* w2,
                               const float* w2_scale, const void* w13s, const float* w13s_scale,
                               const void* w2s, const float* w2s_scale, void* out, void* ws,
                               size_t ws_bytes, void* const* stage_events, moe_stream_t stream);

/* Device byte offsets, inside the workspace, of the intermediates that
 * moe_forward leaves there (for inspection and tests):
 * which = 0 logits fp32 [T,E], 1 topk_idx int32 [T,k], 2 topk_w fp32 [T,k],
 * 3 offsets int32 [E+1], 4 rows int32 [T*k], 5 pos int32 [T*k],
 * 6 y bf16 [T*k,H] (fp32 when k == 1), 7 y_shared fp32 [T,H], 8 u bf16 [T,H] (the normalised
 * input of moe_forward_block).  Returns (size_t)-1 if invalid. */
size_t moe_workspace_offset(const moe_config_t* cfg, int32_t which);

/* ------------------------------------------------------------------------
 * Expert parallelism (experts split over ep_size ranks; Deep Dive §8.2
 * FUSED_MC2 "dispatch -> gmm1 -> swiglu -> gmm2 -> combine" across devices,
 * §10.2 expert parallelism with an all-to-all backend).  Rank d owns experts
 * [d E/ep_size, (d+1) E/ep_size).  One rank's step:
 *   1. moe_route, moe_permute on its own tokens (global expert ids);
 *   2. moe_ep_pack: its routed rows in expert order, which is destination
 *      order, with per-destination counts;
 *   3. all-to-all of counts, then of rows, weights and local expert ids (the
 *      caller's collective: NCCL over NVLink, or any other);
 *   4. the received rows are a k = 1 layer over the rank's E/ep_size experts:
 *      moe_permute, moe_expert_ffn (no shared expert; routed outputs fp32),
 *      moe_combine back to the receive order;
 *   5. the reverse all-to-all returns each row to its sender, in its send
 *      order;
 *   6. moe_shared_expert and moe_combine on the sender give out.
 *
 * moe_ep_pack: for each slot s = t*k + j with sorted row r = pos[s],
 *   x_send[r] = x[t] (bf16 [T*k, H]), w_send[r] = topk_w[s] (fp32 [T*k]),
 *   e_send[r] = expert - owner * E/ep_size (int32 [T*k]);
 *   send_counts[d] = rows for rank d (int32 [ep_size]): the chunk for rank d
 *   is rows offsets[d E/ep_size] .. offsets[(d+1) E/ep_size] - 1.
 * ep_size must divide E.  x and x_send 16-byte aligned.                     */
moe_status_t moe_ep_pack(const moe_config_t* cfg, int32_t ep_size, const void* x,
                         const int32_t* topk_idx, const float* topk_w, const int32_t* offsets,
                         const int32_t* pos, void* x_send, float* w_send, int32_t* e_send,
                         int32_t* send_counts, moe_stream_t stream);

/* The same exchange over peer memory: the rows move by the library's own
 * stores and loads instead of all-to-alls.  Each rank owns three receive
 * buffers that every rank can address (peer-mapped device memory over NVLink,
 * e.g. CUDA IPC or symmetric memory; on one device, plain pointers):
 * x_recv bf16 [recv_cap, H], w_recv fp32 [recv_cap], y_recv fp32 [recv_cap, H].
 * A step of rank r:
 *   1. moe_route and moe_permute on its tokens; moe_ep_expert_counts writes
 *      counts[e] = rows of its tokens for expert e (int32 [E]);
 *   2. the caller all-gathers the counts: counts_all int32 [ep_size][E];
 *   3. moe_ep_plan: the owner's receive buffer is expert-major (its experts in
 *      order, each expert's rows by source rank, each source's rows in its
 *      sorted order), so the q-th row of rank r's segment of expert e lands at
 *      row exp_base[e] + src_base[e] + q of its owner's buffer (int32 [E]
 *      each); recv_offsets int32 [E/ep_size + 1] are rank r's own segments and
 *      recv_ident int32 [recv_cap] gets 0, 1, ... for its received rows.  A
 *      total beyond recv_cap sets a flag in the status word of `ws` (a layer
 *      workspace; moe_check_device_status reports MOE_ERR_WORKSPACE) and the
 *      rows beyond it are dropped;
 *   4. moe_ep_dispatch_peer stores each routed row (H bf16) and its weight into
 *      the owner's x_recv / w_recv (x_recv, w_recv: device arrays of ep_size
 *      pointers, index = owner rank);
 *   5. the caller orders every rank's dispatch before any rank's expert GEMMs
 *      (a cross-device barrier);
 *   6. each rank runs its experts as a k = 1 layer over its R received rows
 *      (R = recv_offsets[E/ep_size]): moe_expert_ffn with T = R, E/ep_size
 *      experts, offsets = recv_offsets, rows = pos = recv_ident, topk_w =
 *      w_recv, no shared expert, y = its y_recv (fp32 rows);
 *   7. a barrier, then moe_shared_expert and moe_ep_combine_peer: out_t = the
 *      sum over slots j (in order) of the row's output loaded from its owner's
 *      y_recv (y_recv: a device array of ep_size pointers), rounded to bf16
 *      first when k > 1, plus the shared expert's row; one bf16 rounding.
 * The output equals moe_forward's bit for bit.  ep_rank in [0, ep_size).     */
moe_status_t moe_ep_expert_counts(const moe_config_t* cfg, const int32_t* offsets, int32_t* counts,
                                  moe_stream_t stream);
moe_status_t moe_ep_plan(const moe_config_t* cfg, int32_t ep_size, int32_t ep_rank,
                         const int32_t* counts_all, int32_t* exp_base, int32_t* src_base,
                         int32_t* recv_offsets, int32_t* recv_ident, int32_t recv_cap, void* ws,
                         moe_stream_t stream);
moe_status_t moe_ep_dispatch_peer(const moe_config_t* cfg, int32_t ep_size, int32_t ep_rank,
                                  const void* x, const int32_t* topk_idx, const float* topk_w,
                                  const int32_t* offsets, const int32_t* pos,
                                  const int32_t* exp_base, const int32_t* src_base,
                                  void* const* x_recv, float* const* w_recv, int32_t recv_cap,
                                  moe_stream_t stream);
moe_status_t moe_ep_combine_peer(const moe_config_t* cfg, int32_t ep_size, int32_t ep_rank,
                                 const int32_t* topk_idx, const int32_t* offsets,
                                 const int32_t* pos, const int32_t* exp_base,
                                 const int32_t* src_base, const float* const* y_recv,
                                 const float* y_shared, void* out, int32_t recv_cap,
                                 moe_stream_t stream);

/* The shared expert alone (bf16 layers): y_shared fp32 [T, H] =
 * SwiGLU_shared(x) with w13s bf16 [2 Is, H], w2s bf16 [H, Is] (Is =
 * n_shared * I > 0).  ws: moe_workspace_size(cfg) bytes.  Step 6 above; the
 * pages' "always-on" shared expert (Deep Dive §3.1/§3.3).                    */
moe_status_t moe_shared_expert(const moe_config_t* cfg, const void* x, const void* w13s,
                               const void* w2s, float* y_shared, void* ws, size_t ws_bytes,
                               moe_stream_t stream);

/* ------------------------------------------------------------------------
 * Backward pass (training side of the layer), bf16 layers.  The pages give
 * the forward pass only (Deep Dive §3.1 gate -> scores -> top-k ->
 * renormalise -> shared + weighted routed sum, §8.2 gmm1 -> swiglu -> gmm2;
 * mlqm.cn 稀疏激活: sigmoid scores, noaux_tc, norm_topk_prob); this is the
 * chain rule through it with the expert choice held fixed, for the loss
 * sum(out * dout).  The choice (top-k of score + bias) is piecewise constant:
 * no gradient flows through it and the expert bias gets none.
 *
 * Bytes of workspace moe_backward needs (256-byte aligned; no zero-fill
 * needed): the dispatch plan, rows padded per expert to multiples of 16, the
 * recomputed gate/up pre-activations and the intermediate gradients.  0 if
 * the configuration is invalid.                                             */
size_t moe_backward_workspace_size(const moe_config_t* cfg);

/* Stages of moe_backward: 0 dispatch (permute, padded plan, gather), 1 gate/up
 * recompute GEMM, 2 down backward GEMM (SwiGLU backward epilogue), 3 router
 * gradient, 4 input-gradient GEMMs, 5 weight-gradient GEMMs, 6 dx combine. */
#define MOE_NUM_BWD_STAGES 7

/*   x         bf16 [T, H]        the forward's input
 *   w_router  bf16 [E, H]
 *   logits    fp32 [T, E]        the forward's router logits (moe_route)
 *   topk_idx  int32 [T, k]       the forward's choice
 *   topk_w    fp32 [T, k]        the forward's routing weights
 *   w13, w2, w13s, w2s           the weights, as for moe_forward
 *   dout      bf16 [T, H]        gradient of the loss at the layer output
 *   dx        bf16 [T, H]  out   gradient at x (routed + shared + router),
 *                                an fp32 sum rounded once
 *   dw_router fp32 [E, H]  out
 *   dw13      fp32 [E, 2I, H] out, dw2 fp32 [E, H, I] out (zero for an
 *                                expert no token chose)
 *   dw13s     fp32 [2 Is, H] out, dw2s fp32 [H, Is] out (n_shared > 0)
 *   dlogits   fp32 [T, E]  out   gradient at the router logits, zero off the
 *                                chosen experts; may be NULL
 *   ws        moe_backward_workspace_size bytes
 *   stage_events  NULL, or MOE_NUM_BWD_STAGES + 1 cudaEvent_t recorded on
 *             `stream` as the stages start (the last after the last stage)
 * All outputs are overwritten.  Pointers to bf16 data and every output
 * except dlogits must be 16-byte aligned.  fp8 layers return
 * MOE_ERR_UNSUPPORTED.                                                      */
moe_status_t moe_backward(const moe_config_t* cfg, const void* x, const void* w_router,
                          const float* logits, const int32_t* topk_idx, const float* topk_w,
                          const void* w13, const void* w2, const void* w13s, const void* w2s,
                          const void* dout, void* dx, float* dw_router, float* dw13, float* dw2,
                          float* dw13s, float* dw2s, float* dlogits, void* ws, size_t ws_bytes,
                          void* const* stage_events, moe_stream_t stream);

/* Expert-bias update of noaux_tc routing (the training side of the selection
 * bias).  mlqm.cn 稀疏激活 names noaux_tc (a per-expert bias steers the
 * top-k choice and stays out of the routing weights; no auxiliary loss) but
 * prints no update rule; the rule here is the plainest reading of it: after
 * a routed batch, each expert whose load is above the batch mean loses gamma
 * from its bias, each one below gains gamma, one exactly at the mean keeps it:
 *   load_e = #{(t, j) : topk_idx[t, j] = e},   b_e += gamma * sign(T*k/E - load_e)
 * The comparison is exact (integers); the update is one fp32 addition.
 *   topk_idx int32 [T, k]   the batch's choice (moe_route); entries outside
 *                           [0, E) count for no expert
 *   bias     fp32 [E]       in/out, updated in place
 *   gamma    >= 0, finite   the step
 * One launch (one block; its histogram is integer, so the result does not
 * depend on scheduling).  T = 0 leaves the bias unchanged and launches
 * nothing.  Returns MOE_ERR_INVALID_ARG for NULL pointers or a bad gamma.   */
moe_status_t moe_bias_update(const moe_config_t* cfg, const int32_t* topk_idx, float* bias,
                             float gamma, moe_stream_t stream);

/* Synchronise `stream`, read the workspace status block of `ws` (the layer's
 * or the DSA indexer's) and clear it.  Returns MOE_OK; MOE_ERR_TIMEOUT if a
 * kernel gave up a bounded wait; or MOE_ERR_WORKSPACE if a tile-claim counter
 * was non-zero after the stream drained, i.e. a claiming launch stopped
 * part-way (its output is incomplete).  Either way the block is zero after
 * the call, so the next call on the workspace starts clean.               */
moe_status_t moe_check_device_status(void* ws, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
