// gate_topk.cu -- warp-per-token expert selection, and the reduction of the
// router's split-K partial sums (the router GEMM itself is router_tc.cu).
//
// Selection ("DeepSeek V3架构拆解：Kimi-K2-Thinking-NVFP4的MLA注意力与MoE路由实现原理",
// 三.2 选专家 and 三.3 权重归一化 + 路由缩放; sqrtsoftplus scoring and route_scale
// from "DeepSeek-V4-Pro 架构与代码概述", 架构; softmax, the alternative 三.1
// contrasts with sigmoid, over a token's logits): score, bias, group-limited top-k,
// normalised and scaled weights. The reduction adds each logit's partials in
// split order (in fp64), so the logits are deterministic.
#include <cuda_bf16.h>

#include <cfloat>
#include <climits>

#include "internal.h"
#include "sm100.cuh"

namespace moe {

namespace {

// logits = sum over splits of the partial sums, added in split order in fp64
// and rounded once to fp32; written over split 0 so the selection kernel reads
// one slab. Eight splits' loads are issued before their adds, which still run
// in split order.
__global__ void __launch_bounds__(256) router_reduce_kernel(float* __restrict__ part, long n,
                                                            int splits) {
    pdl_wait();
    pdl_trigger();
    const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    double l = 0.0;
    int s = 0;
    for (; s + 8 <= splits; s += 8) {
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = part[(size_t)(s + j) * n + i];
#pragma unroll
        for (int j = 0; j < 8; ++j) l += (double)v[j];
    }
    for (; s < splits; ++s) l += (double)part[(size_t)s * n + i];
    part[i] = (float)l;
}

__device__ __forceinline__ float score_of(float l, int score_fn) {
    if (score_fn == MOE_SCORE_SIGMOID) return 1.0f / (1.0f + expf(-l));
    return sqrtf(fmaxf(l, 0.0f) + log1pf(expf(-fabsf(l))));
}

// (value, index) order used everywhere: larger value first, then lower index.
__device__ __forceinline__ bool better(float va, int ia, float vb, int ib) {
    return va > vb || (va == vb && ia < ib);
}

struct TopkParams {
    const float* part;  // summed logits [T][E]
    const float* bias;
    int T, E, k, n_group, topk_group, norm, score_fn;
    float rsf;
    int32_t* idx;
    float* w;
};

// One warp per token. Lane l holds experts e = l + 32*j, j < MAXJ.
template <int MAXJ>
__global__ void __launch_bounds__(256) topk_kernel(TopkParams p) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= p.T) return;
    const int E = p.E;

    // only the biased scores stay in registers; a selected expert's score is
    // recomputed from its logit at the end (same arithmetic, same value)
    const float* logit = p.part + (size_t)t * E;  // the router left the summed logits in split 0
    float spv[MAXJ];
    uint32_t avail = 0;
#pragma unroll
    for (int j = 0; j < MAXJ; ++j) {
        const int e = lane + 32 * j;
        spv[j] = -FLT_MAX;
        if (e < E) {
            spv[j] = logit[e];
            avail |= 1u << j;
        }
    }
    // softmax: s_e = exp(l_e - m) / Z over the token's E logits; m and Z come from
    // xor-butterfly reductions, which leave the same value in every lane
    float m = 0.f, z = 1.f;
    if (p.score_fn == MOE_SCORE_SOFTMAX) {
        float lm = -FLT_MAX;
#pragma unroll
        for (int j = 0; j < MAXJ; ++j) lm = fmaxf(lm, spv[j]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) lm = fmaxf(lm, __shfl_xor_sync(0xffffffffu, lm, off));
        m = lm;
        float zs = 0.f;
#pragma unroll
        for (int j = 0; j < MAXJ; ++j)
            if ((avail >> j) & 1u) zs += expf(spv[j] - m);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) zs += __shfl_xor_sync(0xffffffffu, zs, off);
        z = zs;
    }
    auto score = [&](float l) {
        return p.score_fn == MOE_SCORE_SOFTMAX ? expf(l - m) / z : score_of(l, p.score_fn);
    };
#pragma unroll
    for (int j = 0; j < MAXJ; ++j) {
        const int e = lane + 32 * j;
        if ((avail >> j) & 1u) spv[j] = score(spv[j]) + p.bias[e];
    }

    if (p.n_group > 1) {
        const int gsz = E / p.n_group;
        float gs = -FLT_MAX;  // lane g < n_group holds group g's score
        for (int g = 0; g < p.n_group; ++g) {
            float b1 = -FLT_MAX, b2 = -FLT_MAX;
#pragma unroll
            for (int j = 0; j < MAXJ; ++j) {
                const int e = lane + 32 * j;
                if (((avail >> j) & 1u) && e / gsz == g) {
                    const float v = spv[j];
                    if (v > b1) { b2 = b1; b1 = v; }
                    else if (v > b2) b2 = v;
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const float o1 = __shfl_xor_sync(0xffffffffu, b1, off);
                const float o2 = __shfl_xor_sync(0xffffffffu, b2, off);
                const float hi = fmaxf(b1, o1), lo = fminf(b1, o1);
                b2 = fmaxf(lo, fmaxf(b2, o2));
                b1 = hi;
            }
            const float score = (gsz == 1) ? b1 : b1 + b2;
            if (lane == g) gs = score;
        }
        uint32_t kept = 0;
        for (int r = 0; r < p.topk_group; ++r) {
            float bv = (lane < p.n_group && !((kept >> lane) & 1u)) ? gs : -FLT_MAX;
            int bi = (lane < p.n_group && !((kept >> lane) & 1u)) ? lane : INT_MAX;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
                const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
                if (better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
            }
            kept |= 1u << bi;
        }
#pragma unroll
        for (int j = 0; j < MAXJ; ++j) {
            const int e = lane + 32 * j;
            if (((avail >> j) & 1u) && !((kept >> (e / gsz)) & 1u)) avail &= ~(1u << j);
        }
    }

    // Each lane caches its two best available experts (same order as better());
    // a round is one warp argmax over the lanes' heads, the winning lane pops
    // its head and rescans its experts only when its cache runs empty.
    float v1, v2;
    int i1, i2;
    auto refill = [&]() {
        v1 = v2 = -FLT_MAX;
        i1 = i2 = INT_MAX;
#pragma unroll
        for (int j = 0; j < MAXJ; ++j) {
            const int e = lane + 32 * j;
            if ((avail >> j) & 1u) {
                if (better(spv[j], e, v1, i1)) {
                    v2 = v1; i2 = i1;
                    v1 = spv[j]; i1 = e;
                } else if (better(spv[j], e, v2, i2)) {
                    v2 = spv[j]; i2 = e;
                }
            }
        }
    };
    refill();
    int my_idx = 0;
    for (int r = 0; r < p.k; ++r) {
        float bv = v1;
        int bi = i1;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
            if (better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
        }
        if (lane == r) my_idx = bi;
        if (bi != INT_MAX && (bi & 31) == lane) {
            avail &= ~(1u << (bi >> 5));
            v1 = v2; i1 = i2;
            v2 = -FLT_MAX; i2 = INT_MAX;
            if (i1 == INT_MAX) refill();
        }
    }
    float my_w = (lane < p.k && my_idx >= 0 && my_idx < E) ? score(logit[my_idx]) : 0.f;

    float sum = (lane < p.k) ? my_w : 0.f;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (p.norm) my_w = my_w / sum;
    my_w *= p.rsf;
    if (lane < p.k) {
        p.idx[(size_t)t * p.k + lane] = my_idx;
        p.w[(size_t)t * p.k + lane] = my_w;
    }
}

}  // namespace

cudaError_t launch_router_reduce(float* part, long n, int splits, cudaStream_t st) {
    launch_pdl(router_reduce_kernel, (unsigned)((n + 255) / 256), 256, 0, st, part, n, splits);
    return cudaGetLastError();
}

cudaError_t launch_topk(const moe_config* c, const float* part, const float* bias, int T,
                        int32_t* idx, float* w, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    TopkParams p;
    p.part = part;
    p.bias = bias;
    p.T = T;
    p.E = c->n_routed_experts;
    p.k = c->num_experts_per_tok;
    p.n_group = c->n_group;
    p.topk_group = c->topk_group;
    p.norm = c->norm_topk_prob;
    p.score_fn = c->score_fn;
    p.rsf = c->routed_scaling_factor;
    p.idx = idx;
    p.w = w;
    const int warps = 8;
    dim3 grid((T + warps - 1) / warps);
    if (p.E <= 32) launch_pdl(topk_kernel<1>, grid, warps * 32, 0, st, p);
    else if (p.E <= 128) launch_pdl(topk_kernel<4>, grid, warps * 32, 0, st, p);
    else if (p.E <= 512) launch_pdl(topk_kernel<16>, grid, warps * 32, 0, st, p);
    else launch_pdl(topk_kernel<32>, grid, warps * 32, 0, st, p);
    return cudaGetLastError();
}

}  // namespace moe
