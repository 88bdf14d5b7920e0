/*
 * moe.h -- C ABI of the B200 (sm_100a) routed mixture-of-experts layer forward.
 *
 * The layer, as the source pages state it:
 *   [V3] "DeepSeek V3架构拆解：Kimi-K2-Thinking-NVFP4的MLA注意力与MoE路由实现原理",
 *        section 三 "MoE 路由": 1 打分 (fp32 router linear, sigmoid scores),
 *        2 选专家 (e_score_correction_bias, noaux_tc group-limited top-k),
 *        3 权重归一化 + 路由缩放 (norm_topk_prob, routed_scaling_factor),
 *        4 推理执行 (moe_infer: per-expert counts, argsort by expert id, per-expert
 *        gate/up/down SwiGLU, scatter back with top-k weights, plus shared experts).
 *   [V4] "DeepSeek-V4-Pro 架构与代码概述", 架构 (sqrtsoftplus scoring, route_scale,
 *        FP4 experts with UE8M0 scales) and 文件说明 (kernel.py act_quant_kernel,
 *        fp4_gemm_kernel; model.py MOE, FFNSwiGLU).
 *   [MX] "开源巨头开放2.8T MoE权重:架构创新与本地部署实践指南", 存储与量化策略
 *        (MXFP4 weights, MXFP8 activations).
 *
 * Conventions shared by every entry point:
 *  - Pointers named x, gate_w, topk_idx, ... and every buffer inside moe_weights
 *    and the workspace are DEVICE pointers, allocated and freed by the caller.
 *    moe_config and moe_weights structs themselves live in host memory and are
 *    read during the call only. The library never allocates, frees or
 *    synchronises; it keeps no state across calls except a per-device cache of
 *    the SM count and the set of (kernel, device) pairs whose shared-memory limit
 *    was raised.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream). All work is
 *    enqueued on it in order; outputs are valid once the stream reaches them.
 *    Kernels are launched with programmatic stream serialization: one may be
 *    scheduled while the kernel before it on the stream is finishing, but it
 *    waits on the device for that kernel to complete (and its writes to become
 *    visible) before touching memory, so the ordering is that of the stream.
 *    Each kernel signals its dependents as it starts: a caller's kernel launched
 *    next on the same stream WITH programmatic serialization must itself wait
 *    (griddepcontrol.wait) before reading outputs; one launched without it, any
 *    copy, and any event or host synchronisation see finished results.
 *  - A kernel's shared-memory limit is raised on each device the first time
 *    the kernel is launched there (the device current at the call), so one
 *    process may drive several GPUs, switching with cudaSetDevice.
 *  - Arguments are checked on the host before anything is launched; a bad
 *    argument returns MOE_ERR_INVALID_ARG (or MOE_ERR_UNSUPPORTED for a valid
 *    but unimplemented combination, MOE_ERR_WORKSPACE for a short workspace)
 *    and launches nothing. A failed launch returns MOE_ERR_CUDA.
 *  - Errors found on the device (an expert id out of range, a pipeline wait
 *    that exceeded its time limit) are OR-ed into *dev_status (a caller-owned
 *    device int32 the caller zeroes) as MOE_DEV_* bits; kernels never trap.
 *  - Row-major layouts, leading index first. T = tokens, H = hidden,
 *    E = n_routed_experts, k = num_experts_per_tok, I = moe_intermediate_size,
 *    N = T*k (token, slot) pairs, S = n_shared_experts.
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
    MOE_ERR_INVALID_ARG = 1,
    MOE_ERR_UNSUPPORTED = 2,
    MOE_ERR_WORKSPACE = 3,
    MOE_ERR_CUDA = 4
} moe_status;

/* bits OR-ed into *dev_status by kernels */
#define MOE_DEV_BAD_EXPERT 1 /* a topk_idx entry outside [0, E): pair skipped    */
#define MOE_DEV_TIMEOUT 2    /* a pipeline wait exceeded its limit: work dropped */

/* scoring function ([V3] 三.1 sigmoid; [V4] 架构 sqrtsoftplus = sqrt(softplus)) */
#define MOE_SCORE_SIGMOID 0
#define MOE_SCORE_SQRTSOFTPLUS 1
/* softmax over a token's E logits (the alternative [V3] 三.1 contrasts with
 * sigmoid): s_e = exp(l_e - m) / sum_e' exp(l_e' - m), m = max_e l_e */
#define MOE_SCORE_SOFTMAX 2

/* expert weight formats (routed and shared experts use the same one)
 *  BF16:              bf16 codes.
 *  FP8_E4M3_B128x128: uint8 E4M3 codes + fp32 scale per 128x128 block,
 *                     w13_scale [E][2I/128][H/128], w2_scale [E][H/128][I/128].
 *  FP4_E2M1_UE8M0_B32 and MXFP4: uint8, two E2M1 codes per byte (even column in
 *                     the low nibble) + uint8 E8M0 scale code per 32 columns,
 *                     w13_scale [E][2I][H/32], w2_scale [E][H][I/32]. The two
 *                     differ only in how the producer chose the scales. */
#define MOE_W_BF16 0
#define MOE_W_FP8_E4M3_B128x128 1
#define MOE_W_FP4_E2M1_UE8M0_B32 2
#define MOE_W_MXFP4 3
/* NVFP4 ([V3] 四 NVFP4 量化): routed experts only, with MOE_A_NVFP4. uint8, two
 * E2M1 codes per byte (even column in the low nibble) + uint8 E4M3 scale code
 * per 16 columns (w13_scale [E][2I][H/16], w2_scale [E][H][I/16]) + one fp32
 * tensor scale per expert matrix (moe_weights.w13_gscale / w2_gscale [E]):
 * value = e2m1 * e4m3(scale) * tensor scale. The shared experts stay bf16
 * (the recipe's exclusion list): sh_w13 / sh_w2 hold bf16 values. */
#define MOE_W_NVFP4 4

/* activation formats the experts consume (the router always reads bf16 x)
 *  BF16:               no quantisation.
 *  FP8_E4M3_POW2_B128: E4M3 codes + power-of-two scale per 128 elements, scale
 *                      = smallest 2^e with amax <= 448*2^e, stored as E8M0 code
 *                      e+127 (code 127 for an all-zero block) ([V4] act_quant).
 *  MXFP8:              E4M3 codes + E8M0 scale per 32 elements, scale
 *                      2^(floor(log2 amax) - 8) clamped to [2^-127, 2^127],
 *                      2^-127 for an all-zero block (OCP MX; [MX]).
 *  Elements are round-to-nearest-even, saturating at +-448. */
#define MOE_A_BF16 0
#define MOE_A_FP8_E4M3_POW2_B128 1
#define MOE_A_MXFP8 2
/* NVFP4 activations of the routed experts (with MOE_W_NVFP4 only): E2M1 codes
 * (two per byte) + E4M3 scale code per 16 elements + a per-tensor fp32 scale g
 * (moe_config.nvfp4_x_scale for the experts' input, nvfp4_h_scale for their
 * intermediate): per 16-group s = E4M3_RNE(amax / (6 g)) and
 * q = E2M1_RNE(v / (e4m3(s) g)) (saturating at +-6; zero codes where s is 0),
 * decided in double precision for the bf16 input rows. The shared experts read
 * the bf16 input. */
#define MOE_A_NVFP4 3

/* Layer configuration; field names follow the configuration the pages quote. */
typedef struct {
    int32_t hidden;                   /* H, multiple of 128                     */
    int32_t n_routed_experts;         /* E, 1..1024                             */
    int32_t num_experts_per_tok;      /* k, 1..32, k <= E                       */
    int32_t n_group;                  /* 1..32, divides E                       */
    int32_t topk_group;               /* 1..n_group, k <= topk_group*E/n_group  */
    int32_t moe_intermediate_size;    /* I, multiple of 128                     */
    int32_t n_shared_experts;         /* S, 0..4                                */
    int32_t shared_intermediate_size; /* must equal I when S > 0                */
    int32_t norm_topk_prob;           /* 0 or 1                                 */
    float routed_scaling_factor;      /* > 0                                    */
    int32_t score_fn;                 /* MOE_SCORE_*                            */
    int32_t wfmt;                     /* MOE_W_*                                */
    int32_t afmt;                     /* MOE_A_*                                */
    /* [V4] 架构 FFNSwiGLU's optional swiglu_limit: 0 = off; L > 0 computes
     * SiLU(min(g, L)) * clamp(u, -L, L) in every expert (finite, >= 0) */
    float swiglu_limit;
    /* NVFP4 tensor scales of the routed experts' activations (used only with
     * MOE_A_NVFP4; calibrated constants, > 0): the input x, the intermediate h */
    float nvfp4_x_scale;
    float nvfp4_h_scale;
} moe_config;

/* Device pointers to the layer's parameters.
 *  w13 [E][2I][H]: rows 0..I-1 are the gate projection W1, rows I..2I-1 the
 *      up projection W3 of each expert; w2 [E][H][I] the down projection.
 *  sh_w13 / sh_w2: the same for the S shared experts ([S][2I][H], [S][H][I]).
 *  *_scale: per wfmt above (NULL for BF16).
 *  gate_w fp32 [E][H]: router weight; gate_bias fp32 [E]: e_score_correction_bias. */
typedef struct {
    const void *w13, *w13_scale, *w2, *w2_scale;
    const void *sh_w13, *sh_w13_scale, *sh_w2, *sh_w2_scale;
    const float *gate_w, *gate_bias;
    /* NVFP4 only: fp32 tensor scale of each routed expert's w13 and w2 [E] */
    const float *w13_gscale, *w2_gscale;
} moe_weights;

/* Bytes of device workspace that moe_layer_forward needs for T tokens; every
 * other entry point needs at most this much. 0 for an invalid config. */
size_t moe_workspace_bytes(const moe_config *cfg, int32_t T);

/* Router and selection ([V3] 三.1-三.3; [V4] 架构 for sqrtsoftplus / route_scale).
 *  x bf16 [T][H]; gate_w fp32 [E][H]; gate_bias fp32 [E].
 *  logits = x . gate_w^T with fp32-class accuracy (on the tensor cores, with
 *  gate_w split exactly into three bf16 planes and fp32 accumulation);
 *  s = score(logits) (sigmoid / sqrtsoftplus per logit, or softmax over the
 *  token's logits); s' = s + bias; with n_group > 1 the E experts form
 *  n_group contiguous groups scored by the sum of their two largest s' (a
 *  one-expert group by its s'), the topk_group best groups are kept, then the
 *  k largest s' among kept experts are chosen (ties to the lower index).
 *  topk_idx int32 [T][k] in s'-descending slot order; topk_w fp32 [T][k] = s
 *  (unbiased) of the chosen experts, divided by their sum when norm_topk_prob,
 *  times routed_scaling_factor. dev_status: MOE_DEV_TIMEOUT if a pipeline wait
 *  ran out (may be NULL). ws: workspace (>= moe_workspace_bytes). */
moe_status moe_gate_topk(const moe_config *cfg, const void *x, int32_t T, const float *gate_w,
                         const float *gate_bias, int32_t *topk_idx, float *topk_w,
                         int32_t *dev_status, void *ws, size_t ws_bytes, void *stream);

/* Dispatch permutation ([V3] 三.4: count tokens per expert, argsort by expert id).
 *  topk_idx int32 [T][k]. Pairs p = t*k + j are ordered by (expert, p)
 *  ascending, a stable sort that is deterministic run to run.
 *  expert_offsets int32 [E+1]: start row of each expert's block, [E] = N;
 *  sorted_pair int32 [N]: the pair index at each row; row_of int32 [N]: the
 *  row of each pair (the inverse). Pairs with an expert id outside [0, E) are
 *  left out (row_of = -1) and MOE_DEV_BAD_EXPERT is set in *dev_status. */
moe_status moe_permute(const moe_config *cfg, const int32_t *topk_idx, int32_t T,
                       int32_t *expert_offsets, int32_t *sorted_pair, int32_t *row_of,
                       int32_t *dev_status, void *ws, size_t ws_bytes, void *stream);

/* Permutation for callers that cannot allocate device memory.
 * No counterpart on the source pages: this is a packaging variant of
 * moe_permute for callers that are not allowed to allocate -- for example a
 * plugin running inside a host runtime that owns every device allocation, or a
 * latency-critical serving loop that may not enter the allocator (cudaMalloc
 * can synchronise the device). Such callers have no workspace to pass.
 *
 * Same arguments, results and device-status behaviour as moe_permute, minus
 * the workspace: its per-chunk expert counts live in one file-scope device
 * array of MOE_PERMUTE_NOALLOC_MAX_COUNTS int32 (1 MiB), which every GPU that
 * loads the library holds until the process exits. Limit: ceil(T*k / 4096) *
 * n_routed_experts <= MOE_PERMUTE_NOALLOC_MAX_COUNTS, else MOE_ERR_WORKSPACE
 * and nothing is launched. The call allocates and frees nothing.
 * The first call on each device looks up the array's device address (with that
 * device current); make that first call before any stream capture. All calls
 * share the one array, so calls that overlap on the GPU (other streams, other
 * threads) race and must be serialised by the caller. Each call writes every
 * count it later reads, so nothing left from an earlier call is used. */
#define MOE_PERMUTE_NOALLOC_MAX_COUNTS 262144
moe_status moe_permute_noalloc(const moe_config *cfg, const int32_t *topk_idx, int32_t T,
                               int32_t *expert_offsets, int32_t *sorted_pair, int32_t *row_of,
                               int32_t *dev_status, void *stream);

/* Activation quantisation of the layer input in the config's afmt ([V4]
 * act_quant_kernel; [MX] MXFP8), rows in token order. x bf16 [T][H] -> xq
 * uint8 E4M3 [T][H] and xq_scale uint8 E8M0 codes [T][H/block] (block 128 for
 * FP8_E4M3_POW2_B128, 32 for MXFP8). MOE_ERR_INVALID_ARG for afmt BF16. */
moe_status moe_quantize_activations(const moe_config *cfg, const void *x, int32_t T, void *xq,
                                    void *xq_scale, void *stream);

/* Expert input rows (step in front of the expert GEMMs; activation quantisation
 * per [V4] act_quant_kernel / [MX] MXFP8). x bf16 [T][H]; sorted_pair from
 * moe_permute. Row r < N of xa holds token sorted_pair[r] / k of x, rows N..N+T-1
 * hold the tokens in order (the shared experts' input). xa is bf16 [N+T][H]
 * for BF16 activations with BF16 weights; with FP8 weights (BF16 activations) xa
 * is f16 [N+T][H] holding the row times 2^-e and xa_scale int8 [N+T] holds e
 * (the row's largest magnitude scaled into [2^13, 2^14); exact for every
 * element within 2^-30 of it), the input of the f16 tensor-core gate/up GEMM;
 * for quantised activations xa is uint8 E4M3 [N+T][H] with xa_scale uint8 E8M0
 * [N+T][H/32]: one code per 32 elements, the power-of-two format's per-128 code
 * repeated over its four 32-element sub-blocks (xa_scale unused for BF16
 * activations with BF16 weights). */
moe_status moe_pack_expert_inputs(const moe_config *cfg, const void *x, int32_t T,
                                  const int32_t *sorted_pair, void *xa, void *xa_scale,
                                  void *stream);

/* Gate and up projections with SwiGLU ([V3] 三.4; [V4] FFNSwiGLU), routed and
 * shared experts in one launch: for every row r of expert e's block
 * [expert_offsets[e], expert_offsets[e+1]) and for the shared rows,
 *   a = SiLU(W1 xa[r]) * (W3 xa[r])   (fp32 accumulation on the tensor cores)
 * written to h as bf16 (BF16 activations with BF16 weights), as f16 rows holding
 * the bf16-rounded row times 2^-e with e in h_scale int8 [N + S*T] (FP8 weights:
 * the same rule as for xa, the input of the f16 down GEMM), or as E4M3 + E8M0
 * block scales along I (quantised activations). h is [N + S*T][I]: rows 0..N-1
 * follow xa, rows N + s*T + t belong to shared expert s and token t; for
 * quantised activations h_scale is [N + S*T][I/32] (one E8M0 code per 32
 * features, per-128 codes repeated as for xa_scale).
 * xa / xa_scale as written by moe_pack_expert_inputs for the same config.
 * E2M1 / MXFP4 weights need E4M3 activations and H, I multiples of 512.
 * A pipeline wait past its time limit sets MOE_DEV_TIMEOUT. */
moe_status moe_expert_gate_up(const moe_config *cfg, const void *xa, const void *xa_scale,
                              int32_t T, const int32_t *expert_offsets, const moe_weights *w,
                              void *h, void *h_scale, int32_t *dev_status, void *stream);

/* Down projection ([V3] 三.4): y[r] = W2_e h[r] for the routed rows (bf16 [N][H],
 * sorted row order) and shared_y[s][t] = W2_s h[N + s*T + t] (bf16 [S][T][H]). */
moe_status moe_expert_down(const moe_config *cfg, const void *h, const void *h_scale, int32_t T,
                           const int32_t *expert_offsets, const moe_weights *w, void *y,
                           void *shared_y, int32_t *dev_status, void *stream);

/* Expert computation in one call: moe_pack_expert_inputs, moe_expert_gate_up and
 * moe_expert_down with their intermediates (xa, h) in the workspace.
 *  x bf16 [T][H]; sorted_pair / expert_offsets from moe_permute.
 *  For each row r of expert e (pair p = sorted_pair[r], token t = p / k):
 *    a = SiLU(W1_e xin_t) * (W3_e xin_t),  y[r] = W2_e a,
 *  where xin_t is x[t] quantised in afmt (bf16 when afmt is BF16) and a is
 *  rounded to bf16 (BF16 activations) or block-quantised along I in afmt.
 *  y bf16 [N][H] (row order of sorted_pair); shared_y bf16 [S][T][H] holds
 *  each shared expert's output for every token. ws >= moe_workspace_bytes. */
moe_status moe_grouped_swiglu(const moe_config *cfg, const void *x, int32_t T,
                              const int32_t *sorted_pair, const int32_t *expert_offsets,
                              const moe_weights *w, void *y, void *shared_y, void *ws,
                              size_t ws_bytes, int32_t *dev_status, void *stream);

/* Weighted scatter-back combine ([V3] 三.4 "按原顺序放回，乘上 top-k 权重求和" and
 * the shared-expert addition in DeepseekV3MoE.forward):
 *   out[t] = bf16( sum_j topk_w[t][j] * y[row_of[t*k+j]] + sum_s shared_y[s][t] ),
 * summed in fp32 in slot order then shared order, rounded once.
 *  y bf16 [N][H]; shared_y bf16 [S][T][H] (may be NULL when S = 0);
 *  row_of int32 [N]; topk_w fp32 [T][k]; out bf16 [T][H]. */
moe_status moe_combine(const moe_config *cfg, const void *y, const void *shared_y,
                       const int32_t *row_of, const float *topk_w, int32_t T, void *out,
                       void *stream);

/* The whole layer: moe_gate_topk, moe_permute, moe_grouped_swiglu and
 * moe_combine in order on one stream, no host synchronisation.
 *  x bf16 [T][H] -> out bf16 [T][H]. ws >= moe_workspace_bytes(cfg, T). */
moe_status moe_layer_forward(const moe_config *cfg, const void *x, int32_t T,
                             const moe_weights *w, void *out, void *ws, size_t ws_bytes,
                             int32_t *dev_status, void *stream);

/* Post-attention RMSNorm fused with the expert-input quantisation: the
 * prologue in front of the router ([V3] 三, the decoder layer: input_layernorm
 * -> attention -> residual -> post_attention_layernorm -> MoE; [V4] 文件说明,
 * model.py RMSNorm, its weight kept in fp32, and kernel.py act_quant_kernel).
 *  x bf16 [T][H]: the hidden state after the attention residual (the norm's
 *  input); norm_w fp32 [H]; eps >= 0 (finite).
 *  x_norm bf16 [T][H]: per token r = 1 / sqrt(sum_h x_h^2 / H + eps) and
 *  x_norm_h = (x_h * r) * norm_w_h, evaluated in double precision and rounded
 *  once to bf16 (round to nearest even). The sum's order is the kernel's own,
 *  so a value within ~2^-40 (relative) of a bf16 rounding midpoint may round
 *  either way; every other value is fixed by the formula.
 *  For afmt FP8_E4M3_POW2_B128 / MXFP8 the same pass writes the quantised rows
 *  of x_norm: xq uint8 E4M3 [T][H] and xq_scale uint8 E8M0 [T][H/32] (one code
 *  per 32 elements, the power-of-two format's per-128 code repeated over its
 *  four sub-blocks -- the row layout moe_pack_expert_inputs writes), by the
 *  rule of moe_quantize_activations; H must then be a multiple of 512. For
 *  afmt BF16, xq and xq_scale are ignored (may be NULL).
 *  All pointers 16-byte aligned. One read of x, writes of x_norm (and xq). */
moe_status moe_rmsnorm_prologue(const moe_config *cfg, const void *x, int32_t T,
                                const float *norm_w, float eps, void *x_norm, void *xq,
                                void *xq_scale, void *stream);

/* The whole layer from the un-normalised hidden state: moe_rmsnorm_prologue,
 * then the router and top-k on x_norm, the permutation, the expert-input
 * gather (quantised activations: a byte gather of the rows the prologue
 * quantised; bf16 activations: the inputs built from x_norm as in
 * moe_pack_expert_inputs), the expert GEMMs and the combine. Equal to
 * moe_layer_forward applied to the prologue's x_norm.
 *  x bf16 [T][H] -> out bf16 [T][H]; norm_w fp32 [H]; ws >= moe_workspace_bytes
 *  (which includes the x_norm buffer, offset selector 11). */
moe_status moe_layer_forward_prenorm(const moe_config *cfg, const void *x, int32_t T,
                                     const float *norm_w, float eps, const moe_weights *w,
                                     void *out, void *ws, size_t ws_bytes, int32_t *dev_status,
                                     void *stream);

/* Byte offsets inside the workspace of the intermediate results that
 * moe_layer_forward leaves there (for inspection, tests and step-by-step use):
 *  which = 0 topk_idx, 1 topk_w, 2 expert_offsets, 3 sorted_pair, 4 row_of,
 *          5 y, 6 shared_y, 7 xa, 8 xa_scale, 9 h, 10 h_scale,
 *          11 x_norm (moe_layer_forward_prenorm's RMSNorm output).
 *  Returns (size_t)-1 for an invalid config or which. */
size_t moe_workspace_offset(const moe_config *cfg, int32_t T, int32_t which);

/* Self-test of the pipeline waits' time limit: one warp waits, with the same
 * bounded mbarrier wait every GEMM pipeline uses, on a barrier that nothing
 * arrives on; once the limit (2 s) has passed it sets MOE_DEV_TIMEOUT in
 * *dev_status (device int32, OR-ed into) and returns normally, so the context
 * stays usable. Asynchronous on `stream`. MOE_ERR_INVALID_ARG for a null
 * dev_status, MOE_ERR_CUDA if the launch fails. */
moe_status moe_selftest_wait_limit(int32_t *dev_status, void *stream);

/* Human-readable name of a status code (static string). */
const char *moe_status_string(moe_status s);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
