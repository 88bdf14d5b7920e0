/*
 * moe_oracle.c -- float64 CPU oracle of the routed mixture-of-experts layer
 * forward pass (router, group-limited top-k, dispatch permutation, per-expert
 * SwiGLU on dequantised weights, weighted combine plus shared experts).
 *
 * TEST INFRASTRUCTURE. Only the test-suite, the package smoke check and the
 * benchmark's CPU-baseline leg load this library. It shares no code, header,
 * table or constant with the CUDA library and includes nothing from it.
 *
 * Plain loops in double precision, one token (or one output element) at a
 * time; OpenMP only splits independent outputs across threads and never
 * changes the arithmetic of any single output. Every function names the
 * passage it restates. Sources (page title, section):
 *
 *   [V3]  "DeepSeek V3架构拆解：Kimi-K2-Thinking-NVFP4的MLA注意力与MoE路由实现原理",
 *         section 三 "MoE 路由", items 1 (打分), 2 (选专家), 3 (权重归一化 + 路由缩放),
 *         4 (推理执行).
 *   [V4]  "DeepSeek-V4-Pro 架构与代码概述", the 架构 list (sqrtsoftplus, route_scale,
 *         FP4 experts with UE8M0 scales) and 文件说明 (model.py: FFNSwiGLU, MOE;
 *         kernel.py: act_quant_kernel, fp4_quant_kernel, fp4_gemm_kernel; convert.py:
 *         e2m1 -> e4m3 lossless conversion).
 *   [MX]  "开源巨头开放2.8T MoE权重:架构创新与本地部署实践指南", section
 *         "存储与量化策略：MXFP格式下的1.56TB精粹" (MXFP4 weights, MXFP8 activations).
 *   The post-attention RMSNorm in front of the layer follows [V3] 三 (the
 *   decoder layer: post_attention_layernorm -> MoE) and [V4] 文件说明
 *   (model.py RMSNorm, weight kept in fp32).
 *
 * Where the pages are silent the oracle takes one stated reading; each such
 * place is marked READING below.
 *
 * Formats decoded here are restated from their public definitions: bfloat16
 * (top half of an IEEE binary32), OCP FP8 E4M3 ("e4m3fn": bias 7, no
 * infinities, S.1111.111 is NaN), OCP FP4 E2M1 (bias 1), and the OCP
 * microscaling E8M0 scale (2^(code-127), code 255 is NaN).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ enums */
/* weight formats */
#define OR_W_BF16 0 /* bf16 [rows][cols]                                      */
#define OR_W_FP8 1  /* e4m3 [rows][cols] + fp32 scale [rows/128][cols/128]     */
#define OR_W_FP4 2  /* e2m1 packed 2/byte (even col in low nibble) + E8M0 [rows][cols/32] */
#define OR_W_MXFP4 3 /* same bytes as OR_W_FP4 (OCP MX scale rule on the host)  */
/* activation formats */
#define OR_A_BF16 0 /* no quantisation                                        */
#define OR_A_FP8_POW2_128 1 /* e4m3 + power-of-two scale per 128 elements        */
#define OR_A_MXFP8 2 /* e4m3 + E8M0 scale per 32 elements (OCP MX)               */
/* scoring */
#define OR_SCORE_SIGMOID 0
#define OR_SCORE_SQRTSOFTPLUS 1
#define OR_SCORE_SOFTMAX 2

#define OR_OK 0
#define OR_ERR_ARG 1
#define OR_ERR_ZERO_SUM 2

/* ---------------------------------------------------------- format decode */
double or_bf16_value(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* OCP E4M3: value = (1 + m/8) * 2^(e-7) for e >= 1, (m/8) * 2^-6 for e == 0. */
double or_e4m3_value(uint8_t c) {
    int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    double v = (e == 0) ? ldexp((double)m, -9) : ldexp((double)(8 + m), e - 10);
    return s ? -v : v;
}

/* OCP E2M1: value = (1 + m/2) * 2^(e-1) for e >= 1, m/2 for e == 0. */
double or_e2m1_value(uint8_t c) {
    int s = (c >> 3) & 1, e = (c >> 1) & 3, m = c & 1;
    double v = (e == 0) ? 0.5 * m : ldexp((double)(2 + m), e - 2);
    return s ? -v : v;
}

/* OCP E8M0 / UE8M0 scale: 2^(code - 127); code 255 encodes NaN. */
double or_e8m0_value(uint8_t c) { return c == 255 ? NAN : ldexp(1.0, (int)c - 127); }

/* ---------------------------------------------------------- format encode */
/* Round-to-nearest-even onto the E4M3 grid, saturating to +-448 (the largest
 * finite E4M3 value). Plain search: codes 0x00..0x7E are the non-negative
 * finite values in increasing order, so find the largest code not above |v|
 * and pick between it and the next one; an exact midpoint goes to the code
 * whose mantissa LSB is 0. The sign bit is copied from v (so -0.0 -> 0x80). */
uint8_t or_e4m3_encode(double v) {
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs(v);
    if (isnan(v)) return 0x7F;
    if (a >= 448.0) return sign | 0x7E;
    int lo = 0, hi = 0x7E;
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (or_e4m3_value((uint8_t)mid) <= a) lo = mid; else hi = mid - 1;
    }
    double below = or_e4m3_value((uint8_t)lo), above = or_e4m3_value((uint8_t)(lo + 1));
    double midpoint = 0.5 * (below + above); /* exact: both are short binary fractions */
    int c;
    if (a < midpoint) c = lo;
    else if (a > midpoint) c = lo + 1;
    else c = (lo & 1) ? lo + 1 : lo;
    return sign | (uint8_t)c;
}

/* Smallest integer e with amax <= qmax * 2^e (amax > 0): the exponent of the
 * power-of-two scale 2^ceil(log2(amax/qmax)), found with exact comparisons. */
int or_pow2_ceil_exp(double amax, double qmax) {
    int e;
    frexp(amax / qmax, &e);
    while (ldexp(qmax, e - 1) >= amax) e--;
    while (ldexp(qmax, e) < amax) e++;
    return e;
}

/* floor(log2(amax)) for amax > 0, exact (frexp gives amax = f*2^e, f in [0.5,1)). */
int or_floor_log2(double amax) {
    int e;
    frexp(amax, &e);
    return e - 1;
}

/* Activation block quantiser, one vector v[n] split into consecutive blocks.
 *  OR_A_FP8_POW2_128  [V4] 文件说明, kernel.py act_quant_kernel: FP8 per block of
 *      128 with a power-of-two scale. READING: scale = 2^ceil(log2(amax/448)),
 *      i.e. the smallest power of two that brings the block into E4M3 range;
 *      scale 1 (code 127) for an all-zero block.
 *  OR_A_MXFP8  [MX] 存储与量化策略 (activations in MXFP8) and the OCP MX rule:
 *      X = 2^(floor(log2(amax)) - 8) per 32 elements (8 = exponent of E4M3's
 *      largest power of two), X = 2^-127 and all-zero codes for a zero block;
 *      the exponent is clamped to the E8M0 range [-127, 127].
 * Elements: q = RNE-saturating E4M3 of v / scale. Scales are written as E8M0
 * codes (exponent + 127). q[n] codes, sc[n / block] codes. Returns the block
 * size, or -1 for a bad format or n not a multiple of it. */
int or_quant_act(int afmt, const double *v, int n, uint8_t *q, uint8_t *sc) {
    int blk = (afmt == OR_A_FP8_POW2_128) ? 128 : (afmt == OR_A_MXFP8) ? 32 : -1;
    if (blk < 0 || n % blk) return -1;
    for (int b = 0; b < n / blk; b++) {
        double amax = 0.0;
        for (int i = 0; i < blk; i++) {
            double a = fabs(v[b * blk + i]);
            if (a > amax) amax = a;
        }
        int e;
        if (amax == 0.0) e = (afmt == OR_A_FP8_POW2_128) ? 0 : -127;
        else if (afmt == OR_A_FP8_POW2_128) e = or_pow2_ceil_exp(amax, 448.0);
        else e = or_floor_log2(amax) - 8;
        if (e < -127) e = -127;
        if (e > 127) e = 127;
        sc[b] = (uint8_t)(e + 127);
        for (int i = 0; i < blk; i++) q[b * blk + i] = or_e4m3_encode(ldexp(v[b * blk + i], -e));
    }
    return blk;
}

/* Dequantised value of a quantised activation vector (inverse of the above). */
int or_dequant_act(int afmt, const uint8_t *q, const uint8_t *sc, int n, double *out) {
    int blk = (afmt == OR_A_FP8_POW2_128) ? 128 : (afmt == OR_A_MXFP8) ? 32 : -1;
    if (blk < 0 || n % blk) return -1;
    for (int i = 0; i < n; i++) out[i] = or_e4m3_value(q[i]) * or_e8m0_value(sc[i / blk]);
    return blk;
}

/* One weight element W[e][r][c] of a [n_mat][rows][cols] weight tensor, decoded
 * from the bytes the caller stores.
 *  OR_W_BF16   plain bf16.
 *  OR_W_FP8    e4m3 code times the fp32 scale of its 128x128 block
 *              ([V4] 文件说明: Linear with per-block scales; block size 128x128).
 *  OR_W_FP4 / OR_W_MXFP4  e2m1 code (two per byte, even column in the low
 *              nibble) times the E8M0 scale of its 32-element block along cols
 *              ([V4] 架构: FP4 experts with UE8M0 scales; kernel.py fp4_quant_kernel
 *              block 32; [MX] MXFP4). */
static inline double w_at(int fmt, const void *w, const void *s, int rows, int cols, int e, int r,
                          int c) {
    size_t idx = ((size_t)e * rows + r) * cols + c;
    switch (fmt) {
    case OR_W_BF16:
        return or_bf16_value(((const uint16_t *)w)[idx]);
    case OR_W_FP8: {
        size_t sidx = ((size_t)e * (rows / 128) + r / 128) * (cols / 128) + c / 128;
        return or_e4m3_value(((const uint8_t *)w)[idx]) * (double)((const float *)s)[sidx];
    }
    case OR_W_FP4:
    case OR_W_MXFP4: {
        uint8_t byte = ((const uint8_t *)w)[idx / 2];
        uint8_t nib = (c & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15);
        size_t sidx = ((size_t)e * rows + r) * (cols / 32) + c / 32;
        return or_e2m1_value(nib) * or_e8m0_value(((const uint8_t *)s)[sidx]);
    }
    }
    return NAN;
}

double or_weight_value(int fmt, const void *w, const void *s, int rows, int cols, int e, int r,
                       int c) {
    return w_at(fmt, w, s, rows, cols, e, r, c);
}

/* ------------------------------------------------------------------ router */
/* icfg layout (ints): 0 hidden, 1 n_routed_experts, 2 num_experts_per_tok,
 * 3 n_group, 4 topk_group, 5 moe_intermediate_size, 6 n_shared_experts,
 * 7 shared_intermediate_size, 8 norm_topk_prob, 9 score_fn, 10 wfmt, 11 afmt. */
enum { C_H, C_E, C_K, C_NG, C_TG, C_I, C_NS, C_ISH, C_NORM, C_SCORE, C_WFMT, C_AFMT, C_N };

/* [V3] 三.1: each expert scored independently from the fp32 router product.
 * sigmoid(l) = 1/(1+exp(-l)). [V4] 架构: sqrtsoftplus scoring. READING:
 * sqrt(softplus(l)) with softplus(l) = log(1+exp(l)) written in the overflow-free
 * form max(l,0) + log1p(exp(-|l|)). */
double or_score(double l, int score_fn) {
    if (score_fn == OR_SCORE_SIGMOID) return 1.0 / (1.0 + exp(-l));
    if (score_fn == OR_SCORE_SOFTMAX) return NAN; /* depends on all of a token's logits */
    double sp = (l > 0 ? l : 0.0) + log1p(exp(-fabs(l)));
    return sqrt(sp);
}

/* [V3] 三.1 contrasts the independent sigmoid scores with softmax ("此消彼长":
 * one expert's gain is the others' loss). READING: softmax scoring is the usual
 * softmax over the token's E router logits, s_e = exp(l_e - m) / sum_e' exp(l_e' - m)
 * with m = max_e l_e (the shift changes nothing mathematically and keeps exp
 * finite); bias, group selection, top-k and weights then proceed as for the
 * other scores. */
static void softmax_scores(const double *l, int E, double *s) {
    double m = -INFINITY, z = 0.0;
    for (int e = 0; e < E; e++) m = fmax(m, l[e]);
    for (int e = 0; e < E; e++) {
        s[e] = exp(l[e] - m);
        z += s[e];
    }
    for (int e = 0; e < E; e++) s[e] /= z;
}

/* "a comes before b": larger value first, equal values by lower index
 * (READING: the pages fix no tie-break). */
static inline int before(double va, int ia, double vb, int ib) {
    return va > vb || (va == vb && ia < ib);
}

static double rel_gap(double a, double b) {
    double m = fmax(fabs(a), fabs(b));
    return m > 0 ? fabs(a - b) / m : 0.0;
}

/* Routing of one token.
 *  [V3] 三.1  logits l_e = sum_h x_h * Wg[e][h] (fp32 inputs, exact double sum here),
 *             score s_e = score(l_e).
 *  [V3] 三.2  biased score s'_e = s_e + b_e. With n_group > 1 the experts form
 *             n_group groups (READING: contiguous ranges of E/n_group experts);
 *             a group's score is the sum of its two largest s' (READING: a group
 *             of one expert scores that one value); the topk_group best groups are
 *             kept (READING of the garbled sentence: keep the highest-scoring
 *             groups); then the k largest s' among experts of kept groups are
 *             chosen. n_group == 1 keeps everything (the page's own special case).
 *  [V3] 三.3  w_j = s_{idx_j} (READING: the unbiased score; the bias only steers
 *             selection), normalised to sum 1 when norm_topk_prob, then times
 *             routed_scaling_factor.
 * Slot order: s' descending, ties to the lower expert index.
 * near_tie is set when the k-th and (k+1)-th candidate s' (or the topk_group-th
 * and next group score) differ by less than tie_rel relatively; gap_out gets the
 * smallest such relative gap (or +inf when no competitor exists).
 * order_gap_out (if given) gets the smallest relative gap between the s' of two
 * consecutive slots (+inf for k = 1): below tie_rel the slot order of the
 * chosen experts is a near-tie, though their set is not. */
int or_route_token(const int *icfg, double rsf, const uint16_t *xrow, const float *wg,
                   const float *bias, double tie_rel, int32_t *idx, double *w, uint8_t *near_tie,
                   double *gap_out, double *logits_out, double *order_gap_out) {
    const int H = icfg[C_H], E = icfg[C_E], K = icfg[C_K], NG = icfg[C_NG], TG = icfg[C_TG];
    double *s = (double *)malloc(sizeof(double) * E);
    double *sp = (double *)malloc(sizeof(double) * E);
    uint8_t *cand = (uint8_t *)malloc(E);
    double *gscore = (double *)malloc(sizeof(double) * NG);
    uint8_t *gkept = (uint8_t *)malloc(NG);
    int rc = OR_OK;
    double gap = INFINITY;

    for (int e = 0; e < E; e++) {
        double l = 0.0;
        for (int h = 0; h < H; h++) l += or_bf16_value(xrow[h]) * (double)wg[(size_t)e * H + h];
        if (logits_out) logits_out[e] = l;
        s[e] = (icfg[C_SCORE] == OR_SCORE_SOFTMAX) ? l : or_score(l, icfg[C_SCORE]);
    }
    if (icfg[C_SCORE] == OR_SCORE_SOFTMAX) softmax_scores(s, E, s);
    for (int e = 0; e < E; e++) sp[e] = s[e] + (double)bias[e];

    /* group selection */
    int gsz = E / NG;
    for (int g = 0; g < NG; g++) {
        double b1 = -INFINITY, b2 = -INFINITY;
        for (int e = g * gsz; e < (g + 1) * gsz; e++) {
            if (sp[e] > b1) { b2 = b1; b1 = sp[e]; }
            else if (sp[e] > b2) b2 = sp[e];
        }
        gscore[g] = (gsz == 1) ? b1 : b1 + b2;
        gkept[g] = 0;
    }
    if (NG > 1) {
        for (int r = 0; r < TG; r++) {
            int best = -1;
            for (int g = 0; g < NG; g++)
                if (!gkept[g] && (best < 0 || before(gscore[g], g, gscore[best], best))) best = g;
            gkept[best] = 1;
        }
        if (TG < NG) {
            /* weakest kept group against strongest dropped group */
            int wk = -1, sd = -1;
            for (int g = 0; g < NG; g++) {
                if (gkept[g] && (wk < 0 || before(gscore[wk], wk, gscore[g], g))) wk = g;
                if (!gkept[g] && (sd < 0 || before(gscore[g], g, gscore[sd], sd))) sd = g;
            }
            gap = fmin(gap, rel_gap(gscore[wk], gscore[sd]));
        }
    } else {
        gkept[0] = 1;
    }
    int ncand = 0;
    for (int e = 0; e < E; e++) {
        cand[e] = gkept[e / gsz];
        ncand += cand[e];
    }
    if (ncand < K) { rc = OR_ERR_ARG; goto done; }

    /* top-k among candidates by repeated selection of the best remaining */
    for (int j = 0; j < K; j++) {
        int best = -1;
        for (int e = 0; e < E; e++)
            if (cand[e] && (best < 0 || before(sp[e], e, sp[best], best))) best = e;
        idx[j] = best;
        cand[best] = 0;
    }
    if (ncand > K) {
        int nxt = -1;
        for (int e = 0; e < E; e++)
            if (cand[e] && (nxt < 0 || before(sp[e], e, sp[nxt], nxt))) nxt = e;
        gap = fmin(gap, rel_gap(sp[idx[K - 1]], sp[nxt]));
    }

    if (order_gap_out) {
        double og = INFINITY;
        for (int j = 0; j + 1 < K; j++) og = fmin(og, rel_gap(sp[idx[j]], sp[idx[j + 1]]));
        *order_gap_out = og;
    }

    /* weights */
    double sum = 0.0;
    for (int j = 0; j < K; j++) {
        w[j] = s[idx[j]];
        sum += w[j];
    }
    if (icfg[C_NORM]) {
        if (sum == 0.0) { rc = OR_ERR_ZERO_SUM; goto done; }
        for (int j = 0; j < K; j++) w[j] /= sum;
    }
    for (int j = 0; j < K; j++) w[j] *= rsf;

done:
    *near_tie = (uint8_t)(gap < tie_rel);
    *gap_out = gap;
    free(s); free(sp); free(cand); free(gscore); free(gkept);
    return rc;
}

/* Routing of a list of tokens (independent per token). */
int or_route(const int *icfg, double rsf, const uint16_t *x, int T, const int32_t *tokens,
             int ntok, const float *wg, const float *bias, double tie_rel, int32_t *idx, double *w,
             uint8_t *near_tie, double *gap, double *order_gap) {
    const int H = icfg[C_H], K = icfg[C_K];
    if (icfg[C_NG] < 1 || icfg[C_E] % icfg[C_NG] || icfg[C_TG] < 1 || icfg[C_TG] > icfg[C_NG] ||
        K < 1)
        return OR_ERR_ARG;
    int rc = OR_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < ntok; i++) {
        int t = tokens ? tokens[i] : i;
        if (t < 0 || t >= T) { rc = OR_ERR_ARG; continue; }
        int r = or_route_token(icfg, rsf, x + (size_t)t * H, wg, bias, tie_rel, idx + (size_t)i * K,
                               w + (size_t)i * K, near_tie + i, gap + i, NULL,
                               order_gap ? order_gap + i : NULL);
        if (r != OR_OK) rc = r;
    }
    return rc;
}

/* ------------------------------------------------------------- dispatch */
/* [V3] 三.4: count the tokens of each expert, then argsort the (token, slot)
 * pairs by expert id so each expert's tokens form one contiguous block.
 * READING: the sort is stable, i.e. within an expert pairs keep ascending
 * p = t*k + j order (equivalently ascending token, since a token picks an
 * expert at most once). Written as a counting sort:
 *   offsets[e] = number of pairs with expert < e (offsets[E] = T*k),
 *   sorted_pair[r] = p for the r-th pair in (expert, p) order,
 *   row_of[p] = r (the inverse, used to "put results back in original order"). */
int or_permute(const int32_t *idx, int T, int K, int E, int32_t *offsets, int32_t *sorted_pair,
               int32_t *row_of) {
    long N = (long)T * K;
    for (long p = 0; p < N; p++)
        if (idx[p] < 0 || idx[p] >= E) return OR_ERR_ARG;
    for (int e = 0; e <= E; e++) offsets[e] = 0;
    for (long p = 0; p < N; p++) offsets[idx[p] + 1]++;
    for (int e = 0; e < E; e++) offsets[e + 1] += offsets[e];
    int32_t *fill = (int32_t *)malloc(sizeof(int32_t) * (E > 0 ? E : 1));
    for (int e = 0; e < E; e++) fill[e] = offsets[e];
    for (long p = 0; p < N; p++) {
        int e = idx[p];
        sorted_pair[fill[e]] = (int32_t)p;
        row_of[p] = fill[e];
        fill[e]++;
    }
    free(fill);
    return OR_OK;
}

/* ------------------------------------------------------------- experts */
/* Layer input as the experts see it: the bf16 value for bf16 activations,
 * otherwise the dequantised block quantisation of it (act_quant, [V4] 文件说明
 * kernel.py; [MX] MXFP8 activations). x: n rows of H bf16 codes. */
int or_expert_input(int afmt, const uint16_t *x, int n, int H, double *xin, uint8_t *q_out,
                    uint8_t *sc_out) {
    int rc = OR_OK;
#pragma omp parallel for schedule(static)
    for (int i = 0; i < n; i++) {
        double *row = xin + (size_t)i * H;
        for (int h = 0; h < H; h++) row[h] = or_bf16_value(x[(size_t)i * H + h]);
        if (afmt == OR_A_BF16) continue;
        uint8_t *q = (uint8_t *)malloc(H);
        uint8_t *sc = (uint8_t *)malloc(H / 32 + 1);
        int blk = or_quant_act(afmt, row, H, q, sc);
        if (blk < 0) { rc = OR_ERR_ARG; free(q); free(sc); continue; }
        or_dequant_act(afmt, q, sc, H, row);
        if (q_out) memcpy(q_out + (size_t)i * H, q, H);
        if (sc_out) memcpy(sc_out + (size_t)i * (H / blk), sc, H / blk);
        free(q);
        free(sc);
    }
    return rc;
}

/* One expert's SwiGLU MLP on n input rows ([V3] 三.4: each expert is the
 * gate/up/down MLP with SiLU; [V4] 文件说明 model.py FFNSwiGLU):
 *   g_i = sum_h W13[e][i][h] * xin_h,   u_i = sum_h W13[e][I+i][h] * xin_h,
 *   with limit > 0 ([V4] 架构: FFNSwiGLU with an optional swiglu_limit cut-off;
 *   READING: g_i = min(g_i, limit), u_i = clamp(u_i, -limit, limit)),
 *   a_i = SiLU(g_i) * u_i = g_i / (1 + exp(-g_i)) * u_i,
 *   a   -> block quantised along I when activations are quantised (READING:
 *          the second GEMM consumes the intermediate in the layer's activation
 *          format; bf16 layers keep it exact here),
 *   y_n = sum_i W2[e][n][i] * a_i.
 * w13 / w2 point at the whole [n_mat][..] tensors; e selects the matrix. */
int or_expert_rows(int wfmt, int afmt, const void *w13, const void *w13s, const void *w2,
                   const void *w2s, int e, int I, int H, const double *xin, int n, double limit,
                   double *y) {
    int blk = (afmt == OR_A_FP8_POW2_128) ? 128 : (afmt == OR_A_MXFP8) ? 32 : 0;
    if (blk && I % blk) return OR_ERR_ARG;
    double *a = (double *)malloc(sizeof(double) * (size_t)I * (n > 0 ? n : 1));
    for (int r = 0; r < n; r++) {
        const double *xr = xin + (size_t)r * H;
        double *ar = a + (size_t)r * I;
#pragma omp parallel for schedule(static)
        for (int i = 0; i < I; i++) {
            double g = 0.0, u = 0.0;
            for (int h = 0; h < H; h++) {
                g += w_at(wfmt, w13, w13s, 2 * I, H, e, i, h) * xr[h];
                u += w_at(wfmt, w13, w13s, 2 * I, H, e, I + i, h) * xr[h];
            }
            if (limit > 0.0) {
                g = fmin(g, limit);
                u = fmax(fmin(u, limit), -limit);
            }
            ar[i] = g / (1.0 + exp(-g)) * u;
        }
        if (blk) {
            uint8_t *q = (uint8_t *)malloc(I);
            uint8_t *sc = (uint8_t *)malloc(I / blk);
            or_quant_act(afmt, ar, I, q, sc);
            or_dequant_act(afmt, q, sc, I, ar);
            free(q);
            free(sc);
        }
        double *yr = y + (size_t)r * H;
#pragma omp parallel for schedule(static)
        for (int o = 0; o < H; o++) {
            double acc = 0.0;
            for (int i = 0; i < I; i++) acc += w_at(wfmt, w2, w2s, H, I, e, o, i) * ar[i];
            yr[o] = acc;
        }
    }
    free(a);
    return OR_OK;
}

/* [V3] 三.4 + the DeepseekV3MoE.forward remark: each token's output is the sum
 * over its k slots of w_j * y_j (results put back in original order), plus the
 * shared experts' outputs on the same input with weight 1 (READING: "added",
 * no factor). y: [n][K][H], ys: [n_shared][n][H]. */
void or_combine(int n, int K, int n_shared, int H, const double *w, const double *y,
                const double *ys, double *out) {
    for (int t = 0; t < n; t++)
        for (int h = 0; h < H; h++) {
            double acc = 0.0;
            for (int j = 0; j < K; j++) acc += w[(size_t)t * K + j] * y[((size_t)t * K + j) * H + h];
            for (int s = 0; s < n_shared; s++) acc += ys[((size_t)s * n + t) * H + h];
            out[(size_t)t * H + h] = acc;
        }
}

/* ------------------------------------------------- post-attention RMSNorm */
/* Round-to-nearest-even of a double onto the bfloat16 grid in one step (no
 * intermediate binary32 rounding). bfloat16 keeps 8 significant bits with the
 * binary32 exponent range: in [2^(E), 2^(E+1)) with E >= -126 its spacing is
 * 2^(E-7); below 2^-126 (subnormal) it is 2^-133. q = |v| / spacing is exact
 * (a power-of-two division), so the two neighbours are floor(q) and
 * floor(q) + 1 spacings; an exact midpoint goes to the even multiple (the code
 * whose last bit is 0). Magnitudes that round past the largest finite value
 * (2 - 2^-7) * 2^127 become infinity. *near (if given) is set to 1 when |v|
 * lies within tie_rel * |v| of a midpoint between two neighbours. */
uint16_t or_bf16_encode(double v, double tie_rel, uint8_t *near) {
    if (near) *near = 0;
    if (isnan(v)) return 0x7FC0;
    uint16_t sign = signbit(v) ? 0x8000 : 0x0000;
    double a = fabs(v);
    if (a == 0.0) return sign;
    if (isinf(v)) return sign | 0x7F80;
    int e;
    frexp(a, &e); /* a = f * 2^e, f in [0.5, 1): leading bit 2^(e-1) */
    int lead = e - 1;
    if (lead < -126) lead = -126; /* subnormal spacing */
    double spacing = ldexp(1.0, lead - 7);
    double q = a / spacing; /* exact */
    double lo = floor(q);
    double frac = q - lo; /* exact */
    if (near && fabs(a - (lo + 0.5) * spacing) <= tie_rel * a) *near = 1;
    double n;
    if (frac > 0.5) n = lo + 1.0;
    else if (frac < 0.5) n = lo;
    else n = (fmod(lo, 2.0) == 0.0) ? lo : lo + 1.0;
    double r = n * spacing; /* a bfloat16 value (or 2^128) */
    if (r >= ldexp(1.0, 128)) return sign | 0x7F80;
    float f = (float)r; /* exact: r has at most 8 significant bits in range */
    uint32_t u;
    memcpy(&u, &f, 4);
    return sign | (uint16_t)(u >> 16);
}

/* The post-attention RMSNorm in front of the MoE block ([V3] 三, the decoder
 * layer: post_attention_layernorm -> MoE/MLP; [V4] 文件说明, model.py RMSNorm:
 * the standard form with its weight kept in fp32):
 *   r = 1 / sqrt( (sum_h x_h^2) / H + eps ),   y_h = (x_h * r) * w_h,
 * READING: the pages fix neither the working precision nor eps. Here every
 * step is evaluated in double in the order written (the sum sequentially over
 * h, then the mean, eps, sqrt and reciprocal, then the two products), and y_h
 * is rounded once to bf16 (RNE) -- the output the router and the expert
 * inputs read. x [n][H] bf16 codes, w [H] fp32, out [n][H] bf16 codes;
 * near[n][H] (if given) flags outputs within tie_rel * |y| of a bf16 rounding
 * midpoint, where an implementation summing the squares in another order may
 * round the other way. Returns OR_ERR_ARG for n < 0, H < 1 or eps < 0. */
int or_rmsnorm(const uint16_t *x, int n, int H, const float *w, double eps, double tie_rel,
               uint16_t *out, uint8_t *near) {
    if (n < 0 || H < 1 || !(eps >= 0.0)) return OR_ERR_ARG;
#pragma omp parallel for schedule(static)
    for (int t = 0; t < n; t++) {
        const uint16_t *xr = x + (size_t)t * H;
        double ss = 0.0;
        for (int h = 0; h < H; h++) {
            double v = or_bf16_value(xr[h]);
            ss += v * v;
        }
        double r = 1.0 / sqrt(ss / (double)H + eps);
        for (int h = 0; h < H; h++) {
            double y = (or_bf16_value(xr[h]) * r) * (double)w[h];
            uint8_t nt = 0;
            out[(size_t)t * H + h] = or_bf16_encode(y, tie_rel, &nt);
            if (near) near[(size_t)t * H + h] = nt;
        }
    }
    return OR_OK;
}

/* ------------------------------------------------------------------ NVFP4 */
/* [V3] 四 NVFP4 量化: the routed experts' weights and their input activations
 * are 4-bit floats (E2M1) in groups of 16 sharing one FP8 (E4M3) scale; the
 * shared experts, like attention and lm_head, stay in high precision.
 * READING (the page gives the group size and the scale type only): NVIDIA's
 * NVFP4 as it is usually stored -- value = e2m1(q) * e4m3(s) * g, with s the
 * group's scale code (non-negative E4M3) and g one fp32 scale per tensor (per
 * expert matrix for weights; one per layer input for activations, a calibrated
 * constant).
 * Round-to-nearest-even onto the E2M1 grid {0, 0.5, 1, 1.5, 2, 3, 4, 6},
 * saturating to +-6; an exact midpoint goes to the code whose last bit is 0;
 * the sign is copied from v. Plain search over the eight magnitudes. */
uint8_t or_e2m1_encode(double v) {
    uint8_t sign = signbit(v) ? 8 : 0;
    double a = fabs(v);
    if (isnan(v)) return 7; /* no NaN in E2M1: saturate */
    if (a >= 6.0) return sign | 7;
    int lo = 0;
    while (lo < 7 && or_e2m1_value((uint8_t)(lo + 1)) <= a) lo++;
    double below = or_e2m1_value((uint8_t)lo), above = or_e2m1_value((uint8_t)(lo + 1));
    double mid = 0.5 * (below + above); /* exact */
    int c;
    if (a < mid) c = lo;
    else if (a > mid) c = lo + 1;
    else c = (lo & 1) ? lo + 1 : lo;
    return sign | (uint8_t)c;
}

/* NVFP4 quantiser of one vector v[n] (n a multiple of 16) with tensor scale g:
 * per group of 16, s = E4M3_RNE(amax / (6 g)) (the scale that maps the group's
 * largest magnitude onto E2M1's largest value 6, rounded to its FP8 code,
 * saturating at 448), then q_i = E2M1_RNE(v_i / (e4m3(s) g)); a group whose
 * scale code decodes to 0 stores zero codes. READING: the quotients are formed
 * in double (for bf16 inputs and fp32 g they decide each code exactly). q[n]
 * codes (one per byte here), sc[n/16] codes. Returns 16, or -1 for bad n or
 * g <= 0. */
int or_quant_nvfp4(const double *v, int n, double g, uint8_t *q, uint8_t *sc) {
    if (n % 16 || !(g > 0.0)) return -1;
    for (int b = 0; b < n / 16; b++) {
        double amax = 0.0;
        for (int i = 0; i < 16; i++) {
            double a = fabs(v[b * 16 + i]);
            if (a > amax) amax = a;
        }
        uint8_t s = or_e4m3_encode(amax / (6.0 * g));
        sc[b] = s;
        double sv = or_e4m3_value(s);
        for (int i = 0; i < 16; i++)
            q[b * 16 + i] = (sv == 0.0) ? 0 : or_e2m1_encode(v[b * 16 + i] / (sv * g));
    }
    return 16;
}

/* Dequantised NVFP4 vector: e2m1(q_i) * e4m3(sc[i/16]) * g. */
int or_dequant_nvfp4(const uint8_t *q, const uint8_t *sc, int n, double g, double *out) {
    if (n % 16) return -1;
    for (int i = 0; i < n; i++) out[i] = or_e2m1_value(q[i]) * or_e4m3_value(sc[i / 16]) * g;
    return 16;
}

/* One NVFP4 weight element W[e][r][c]: E2M1 codes two per byte (even column in
 * the low nibble), E4M3 scale codes [n_mat][rows][cols/16], tensor scale g[e]. */
static inline double w_nvfp4(const uint8_t *w, const uint8_t *s, const float *g, int rows, int cols,
                             int e, int r, int c) {
    size_t idx = ((size_t)e * rows + r) * cols + c;
    uint8_t byte = w[idx / 2];
    uint8_t nib = (c & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15);
    size_t sidx = ((size_t)e * rows + r) * (cols / 16) + c / 16;
    return or_e2m1_value(nib) * or_e4m3_value(s[sidx]) * (double)g[e];
}

double or_weight_value_nvfp4(const uint8_t *w, const uint8_t *s, const float *g, int rows, int cols,
                             int e, int r, int c) {
    return w_nvfp4(w, s, g, rows, cols, e, r, c);
}

/* One routed expert e on n input rows xin[n][H] (already the dequantised NVFP4
 * activations, tensor scale ga13), [V3] 三.4 with the NVFP4 recipe of [V3] 四:
 *   g = W1 x, u = W3 x  (dequantised NVFP4 weights, tensor scale g13[e]),
 *   a = SiLU(g) * u  (limit > 0: SiLU(min(g, limit)) * clamp(u, -limit, limit)),
 *   a quantised to NVFP4 with tensor scale ga2 and dequantised,
 *   y = W2 a  (NVFP4 weights, tensor scale g2[e]).
 * All in double. y [n][H]. */
int or_expert_rows_nvfp4(const uint8_t *w13, const uint8_t *w13s, const float *g13,
                         const uint8_t *w2, const uint8_t *w2s, const float *g2, int e, int I,
                         int H, const double *xin, int n, double ga2, double limit, double *y) {
    if (I % 16 || H % 16 || !(ga2 > 0.0)) return OR_ERR_ARG;
    double *a = (double *)malloc(sizeof(double) * (size_t)n * I);
    for (int r = 0; r < n; r++) {
        const double *xr = xin + (size_t)r * H;
        double *ar = a + (size_t)r * I;
#pragma omp parallel for schedule(static)
        for (int i = 0; i < I; i++) {
            double gsum = 0.0, usum = 0.0;
            for (int h = 0; h < H; h++) {
                gsum += w_nvfp4(w13, w13s, g13, 2 * I, H, e, i, h) * xr[h];
                usum += w_nvfp4(w13, w13s, g13, 2 * I, H, e, I + i, h) * xr[h];
            }
            if (limit > 0.0) {
                gsum = fmin(gsum, limit);
                usum = fmax(fmin(usum, limit), -limit);
            }
            ar[i] = gsum / (1.0 + exp(-gsum)) * usum;
        }
        uint8_t *q = (uint8_t *)malloc(I);
        uint8_t *sc = (uint8_t *)malloc(I / 16);
        or_quant_nvfp4(ar, I, ga2, q, sc);
        or_dequant_nvfp4(q, sc, I, ga2, ar);
        free(q);
        free(sc);
        double *yr = y + (size_t)r * H;
#pragma omp parallel for schedule(static)
        for (int o = 0; o < H; o++) {
            double acc = 0.0;
            for (int i = 0; i < I; i++) acc += w_nvfp4(w2, w2s, g2, H, I, e, o, i) * ar[i];
            yr[o] = acc;
        }
    }
    free(a);
    return OR_OK;
}
