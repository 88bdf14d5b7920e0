// pack_combine.cu -- activation gather/quantisation in front of the expert
// GEMMs, and the weighted combine behind them.
//
// Gather + quantise: each expert row r of the GEMM input is token
// sorted_pair[r] / k of x (rows past N are the tokens in order, for the shared
// experts). When those shared-expert rows exist, they are quantised first and
// the routed rows are byte copies of them, so every token is quantised once.
// Quantisation follows the activation format:
//  * FP8_E4M3_POW2_B128 ("DeepSeek-V4-Pro 架构与代码概述", 文件说明, kernel.py
//    act_quant_kernel: FP8 per 128-element block, power-of-two scale): scale
//    2^e with e the smallest integer such that amax <= 448 * 2^e;
//  * MXFP8 ("开源巨头开放2.8T MoE权重:架构创新与本地部署实践指南", 存储与量化策略,
//    MXFP8 activations; OCP MX rule): 2^(floor(log2 amax) - 8) per 32 elements;
// both clamp the exponent to [-127, 127], write it as an E8M0 code, and round
// the elements x / scale to E4M3 with round-to-nearest-even and saturation.
//
// Combine ("DeepSeek V3架构拆解：Kimi-K2-Thinking-NVFP4的MLA注意力与MoE路由实现原理",
// 三.4: put the rows back in order, multiply by the top-k weights and sum; plus
// the shared experts): one CTA per token, 16-byte vector loads of every row it
// needs, fp32 sums in slot order, one bf16 rounding.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "internal.h"
#include "sm100.cuh"

namespace moe {

namespace {

// Token feeding expert row r; -1 when the row holds no valid pair (a row past
// the valid pairs when some topk_idx entries were out of range).
__device__ __forceinline__ int token_of_row(int r, const int32_t* sorted_pair, int N, int k, int T) {
    const int t = r < N ? sorted_pair[r] / k : r - N;
    return (t >= 0 && t < T) ? t : -1;
}

__device__ __forceinline__ void st_stream16(uint4* p, uint4 v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

// Row gather: expert row r (< n_rows) becomes row src_row0 + token_of_row(r) of
// src, row16 16-byte vectors (and, when ssrc is set, the same for srow16-vector
// scale rows; when esrc is set, one exponent byte per row); a row without a
// valid pair is zero-filled. One warp per row,
// four loads in flight per lane, streaming stores (the rows are read once, by
// the GEMM, after the whole gather).
// src and dst may be one buffer (routed rows gathered from its token rows), so
// they carry no __restrict__: the rows read and the rows written never overlap.
__global__ void __launch_bounds__(256) gather_rows_kernel(
    const uint4* src, int src_row0, int row16, const uint4* ssrc, int srow16,
    const int32_t* __restrict__ sorted_pair, int N, int k, int T, int n_rows, uint4* dst,
    uint4* sdst, const int8_t* esrc, int8_t* edst) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (r >= n_rows) return;
    const int t = token_of_row(r, sorted_pair, N, k, T);
    uint4* d = dst + (size_t)r * row16;
    if (t < 0) {
        for (int v = lane; v < row16; v += 32) d[v] = make_uint4(0, 0, 0, 0);
        if (ssrc)
            for (int v = lane; v < srow16; v += 32) sdst[(size_t)r * srow16 + v] = make_uint4(0, 0, 0, 0);
        if (esrc && lane == 0) edst[r] = 0;
        return;
    }
    if (esrc && lane == 0) edst[r] = esrc[src_row0 + t];
    const uint4* s = src + (size_t)(src_row0 + t) * row16;
    int v = lane;
    for (; v + 96 < row16; v += 128) {
        const uint4 a0 = s[v], a1 = s[v + 32], a2 = s[v + 64], a3 = s[v + 96];
        st_stream16(d + v, a0);
        st_stream16(d + v + 32, a1);
        st_stream16(d + v + 64, a2);
        st_stream16(d + v + 96, a3);
    }
    for (; v < row16; v += 32) st_stream16(d + v, s[v]);
    if (ssrc) {
        const uint4* ss = ssrc + (size_t)(src_row0 + t) * srow16;
        for (int w = lane; w < srow16; w += 32) st_stream16(sdst + (size_t)r * srow16 + w, ss[w]);
    }
}

// exponent of the power-of-two scale: smallest e with a <= 448 * 2^e
__device__ __forceinline__ int pow2_scale_exp(float a) {
    if (a == 0.0f) return 0;
    int adj = 0;
    uint32_t b = __float_as_uint(a);
    if ((b >> 23) == 0) {  // subnormal: scale up exactly first
        b = __float_as_uint(a * 0x1p64f);
        adj = -64;
    }
    const int E = (int)(b >> 23) - 127;
    const uint32_t mant = b & 0x7FFFFFu;
    // a = m * 2^E, m in [1,2); 448 = 1.75 * 2^8: a <= 448 * 2^e  <=>  e >= E - 8 (+1 if m > 1.75)
    return E - 8 + (mant > 0x600000u ? 1 : 0) + adj;
}

// OCP MX shared exponent for E4M3 elements: floor(log2 a) - 8, clamped
__device__ __forceinline__ int mx_scale_exp(float a) {
    const uint32_t b = __float_as_uint(a);
    const int f = (int)(b >> 23);
    if (f == 0) return -127;  // zero or subnormal: floor(log2 a) - 8 < -127
    return max(f - 127 - 8, -127);
}

// One warp per row; 4 elements per lane per step (a 128-element block for the
// power-of-two format, four 32-element blocks for MX).
// per32: write one scale code per 32 elements (a 128-element block's code is
// repeated over its four 32-element sub-blocks), the layout the block-scaled
// tensor-core GEMM reads; otherwise one code per block.
template <int AFMT>
__global__ void __launch_bounds__(256) pack_fp8_kernel(const __nv_bfloat16* __restrict__ x, int H,
                                                       const int32_t* __restrict__ sorted_pair,
                                                       int N, int k, int T, int n_rows,
                                                       uint8_t* __restrict__ out,
                                                       uint8_t* __restrict__ out_scale, int per32,
                                                       int row0) {
    pdl_wait();
    pdl_trigger();
    constexpr int BLK = (AFMT == MOE_A_FP8_E4M3_POW2_B128) ? 128 : 32;
    const int SBLK = per32 ? 32 : BLK;  // elements per stored scale
    const int lane = threadIdx.x & 31;
    const int r = row0 + blockIdx.x * 8 + (threadIdx.x >> 5);
    if (r >= n_rows) return;
    const int t = token_of_row(r, sorted_pair, N, k, T);
    const __nv_bfloat16* src = x + (size_t)(t < 0 ? 0 : t) * H;
    uint8_t* dst = out + (size_t)r * H;
    uint8_t* dsc = out_scale + (size_t)r * (H / SBLK);
    for (int c0 = 0; c0 < H; c0 += 128) {
        uint2 raw = make_uint2(0, 0);
        if (t >= 0) raw = *reinterpret_cast<const uint2*>(src + c0 + lane * 4);
        const __nv_bfloat162* pr = reinterpret_cast<const __nv_bfloat162*>(&raw);
        const float2 f01 = __bfloat1622float2(pr[0]);
        const float2 f23 = __bfloat1622float2(pr[1]);
        float amax = fmaxf(fmaxf(fabsf(f01.x), fabsf(f01.y)), fmaxf(fabsf(f23.x), fabsf(f23.y)));
        constexpr int LANES = BLK / 4;  // lanes sharing one scale
#pragma unroll
        for (int off = LANES / 2; off > 0; off >>= 1)
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        int e = (AFMT == MOE_A_FP8_E4M3_POW2_B128) ? pow2_scale_exp(amax) : mx_scale_exp(amax);
        e = min(max(e, -127), 127);
        const float inv = __uint_as_float((uint32_t)(127 - e) << 23);  // 2^-e, e in [-127, 126]
        const __nv_fp8x2_storage_t q01 =
            __nv_cvt_float2_to_fp8x2(make_float2(f01.x * inv, f01.y * inv), __NV_SATFINITE, __NV_E4M3);
        const __nv_fp8x2_storage_t q23 =
            __nv_cvt_float2_to_fp8x2(make_float2(f23.x * inv, f23.y * inv), __NV_SATFINITE, __NV_E4M3);
        const uint32_t packed = (uint32_t)q01 | ((uint32_t)q23 << 16);
        *reinterpret_cast<uint32_t*>(dst + c0 + lane * 4) = packed;
        if ((lane % (SBLK / 4)) == 0) dsc[(c0 + lane * 4) / SBLK] = (uint8_t)(e + 127);
    }
}

// f16 rows with a power-of-two row scale, the input of the f16 tensor-core path
// of the FP8-weight gate/up GEMM: row r holds x[t] * 2^-e_r and xs[r] = e_r,
// with e_r chosen so the row's largest magnitude lies in [2^13, 2^14). A bf16
// value has an 8-bit significand, so it is exact in f16 wherever the scaled
// value is at least 2^-17 (every element within 2^-30 of the row's largest);
// only smaller ones round, by at most 2^-25 of 2^e_r. One warp per row, rows
// from row0; two passes over the row (amax, then conversion).
__global__ void __launch_bounds__(256) pack_f16_kernel(const uint4* __restrict__ x, int H8,
                                                       const int32_t* __restrict__ sorted_pair,
                                                       int N, int k, int T, int n_rows, int row0,
                                                       uint4* __restrict__ out,
                                                       int8_t* __restrict__ xs) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int r = row0 + blockIdx.x * 8 + (threadIdx.x >> 5);
    if (r >= n_rows) return;
    const int t = token_of_row(r, sorted_pair, N, k, T);
    uint4* dst = out + (size_t)r * H8;
    if (t < 0) {
        for (int v = lane; v < H8; v += 32) dst[v] = make_uint4(0, 0, 0, 0);
        if (lane == 0) xs[r] = 0;
        return;
    }
    const uint4* src = x + (size_t)t * H8;
    // bf16 magnitudes order like their bit patterns (sign bit cleared)
    uint32_t m = 0;
    for (int v = lane; v < H8; v += 32) {
        const uint4 u = src[v];
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) m = max(m, max(w[i] & 0x7FFFu, (w[i] >> 16) & 0x7FFFu));
    }
    m = __reduce_max_sync(0xffffffffu, m);
    int e = 0;
    if (m != 0) {
        const int E = ilogbf(__uint_as_float(m << 16));  // floor(log2(amax)), exact
        e = min(max(E - 13, -127), 114);
    }
    const float sc = __uint_as_float((uint32_t)(127 - e) << 23);  // 2^-e, a normal float
    for (int v = lane; v < H8; v += 32) {
        const uint4 u = src[v];
        const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u);
        uint4 o;
        __half2* h = reinterpret_cast<__half2*>(&o);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(b[i]);
            h[i] = __floats2half2_rn(f.x * sc, f.y * sc);
        }
        st_stream16(dst + v, o);
    }
    if (lane == 0) xs[r] = (int8_t)e;
}

// In place: bf16 rows [n_rows][C] become f16 rows holding the row times 2^-e,
// e per row in xs, by the rule pack_f16_kernel uses (the row's largest
// magnitude scaled into [2^13, 2^14); exact for every element within 2^-30 of
// it). One warp per row; each lane rewrites only the vectors it read.
__global__ void __launch_bounds__(256) rows_to_f16_kernel(uint4* __restrict__ rows, int C8, int n_rows,
                                                          int8_t* __restrict__ xs) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (r >= n_rows) return;
    uint4* row = rows + (size_t)r * C8;
    uint32_t m = 0;
    for (int v = lane; v < C8; v += 32) {
        const uint4 u = row[v];
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) m = max(m, max(w[i] & 0x7FFFu, (w[i] >> 16) & 0x7FFFu));
    }
    m = __reduce_max_sync(0xffffffffu, m);
    int e = 0;
    if (m != 0) {
        const int E = ilogbf(__uint_as_float(m << 16));  // floor(log2(amax)), exact
        e = min(max(E - 13, -127), 114);
    }
    const float sc = __uint_as_float((uint32_t)(127 - e) << 23);  // 2^-e, a normal float
    for (int v = lane; v < C8; v += 32) {
        const uint4 u = row[v];
        const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u);
        uint4 o;
        __half2* h = reinterpret_cast<__half2*>(&o);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(b[i]);
            h[i] = __floats2half2_rn(f.x * sc, f.y * sc);
        }
        row[v] = o;
    }
    if (lane == 0) xs[r] = (int8_t)e;
}

// Large batches: one CTA per token, threads striding over the row's 16-byte
// columns, the k expert rows and S shared rows of a column summed in order.
__global__ void __launch_bounds__(128) combine_token_kernel(const __nv_bfloat16* __restrict__ y,
                                                      const __nv_bfloat16* __restrict__ shared_y,
                                                      int S, const int32_t* __restrict__ row_of,
                                                      const float* __restrict__ w, int T, int k,
                                                      int H, __nv_bfloat16* __restrict__ out) {
    pdl_wait();
    pdl_trigger();
    __shared__ int32_t rows[32];
    __shared__ float wts[32];
    const int t = blockIdx.x;
    if (threadIdx.x < k) {
        rows[threadIdx.x] = row_of[(size_t)t * k + threadIdx.x];
        wts[threadIdx.x] = w[(size_t)t * k + threadIdx.x];
    }
    __syncthreads();
    const int H8 = H / 8;
    for (int v = threadIdx.x; v < H8; v += blockDim.x) {
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.f;
        for (int j = 0; j < k; ++j) {
            const int r = rows[j];
            if (r < 0) continue;
            const float wj = wts[j];
            const uint4 u = *reinterpret_cast<const uint4*>(y + (size_t)r * H + (size_t)v * 8);
            const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(b[i]);
                acc[2 * i] = fmaf(wj, f.x, acc[2 * i]);
                acc[2 * i + 1] = fmaf(wj, f.y, acc[2 * i + 1]);
            }
        }
        for (int s = 0; s < S; ++s) {
            const uint4 u =
                *reinterpret_cast<const uint4*>(shared_y + ((size_t)s * T + t) * H + (size_t)v * 8);
            const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(b[i]);
                acc[2 * i] += f.x;
                acc[2 * i + 1] += f.y;
            }
        }
        uint4 o;
        __nv_bfloat162* ob = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
        for (int i = 0; i < 4; ++i) ob[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
        *reinterpret_cast<uint4*>(out + (size_t)t * H + (size_t)v * 8) = o;
    }
}

// Small batches: one CTA per (token, block of 128 16-byte columns): thread v loads column v of all of
// the token's k expert rows and S shared rows first (up to 32 + 4 loads in
// flight), then sums them in slot order, then shared order, in fp32, and
// rounds once to bf16. MAXR >= k + S rows are held per thread (k <= 32, S <= 4).
template <int MAXR>
__global__ void __launch_bounds__(128) combine_kernel(const __nv_bfloat16* __restrict__ y,
                                                      const __nv_bfloat16* __restrict__ shared_y,
                                                      int S, const int32_t* __restrict__ row_of,
                                                      const float* __restrict__ w, int T, int k,
                                                      int H, __nv_bfloat16* __restrict__ out) {
    pdl_wait();
    pdl_trigger();
    __shared__ int32_t rows[32];
    __shared__ float wts[32];
    // column blocks of one token are consecutive CTAs, so each token's rows are
    // read front to back in time
    const int H8 = H / 8;
    const int nblk = (H8 + 127) / 128;
    const int t = blockIdx.x / nblk;
    if (threadIdx.x < k) {
        rows[threadIdx.x] = row_of[(size_t)t * k + threadIdx.x];
        wts[threadIdx.x] = w[(size_t)t * k + threadIdx.x];
    }
    __syncthreads();
    const int v = (blockIdx.x % nblk) * blockDim.x + threadIdx.x;
    if (v >= H8) return;
    const int nr = k + S;
    uint4 u[MAXR];
#pragma unroll
    for (int j = 0; j < MAXR; ++j) {
        if (j < nr) {
            const uint4* src = nullptr;
            if (j < k) {
                if (rows[j] >= 0) src = reinterpret_cast<const uint4*>(y + (size_t)rows[j] * H) + v;
            } else {
                src = reinterpret_cast<const uint4*>(shared_y + ((size_t)(j - k) * T + t) * H) + v;
            }
            u[j] = src ? *src : make_uint4(0, 0, 0, 0);
        }
    }
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
    for (int j = 0; j < MAXR; ++j) {
        if (j < k) {
            if (rows[j] < 0) continue;
            const float wj = wts[j];
            const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u[j]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(b[i]);
                acc[2 * i] = fmaf(wj, f.x, acc[2 * i]);
                acc[2 * i + 1] = fmaf(wj, f.y, acc[2 * i + 1]);
            }
        } else if (j < nr) {
            const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u[j]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(b[i]);
                acc[2 * i] += f.x;
                acc[2 * i + 1] += f.y;
            }
        }
    }
    uint4 o;
    __nv_bfloat162* ob = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
    for (int i = 0; i < 4; ++i) ob[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
    *reinterpret_cast<uint4*>(out + (size_t)t * H + (size_t)v * 8) = o;
}

// Post-attention RMSNorm fused with the expert-input quantisation: the prologue
// in front of the router ("DeepSeek V3架构拆解：Kimi-K2-Thinking-NVFP4的MLA注意力
// 与MoE路由实现原理", 三: the decoder layer runs post_attention_layernorm then the
// MoE block; "DeepSeek-V4-Pro 架构与代码概述", 文件说明: model.py RMSNorm keeps its
// weight in fp32, kernel.py act_quant_kernel quantises the activations).
// Row t: r = 1 / sqrt(sum_h x_h^2 / H + eps) and xn_h = bf16((x_h * r) * w_h),
// every step in double and one round-to-nearest-even to bf16, so the bf16
// decision is taken at a precision where only values within ~2^-40 of a
// rounding midpoint can depend on the order of the sum. With a quantised
// activation format the same pass also writes the row's E4M3 codes and E8M0
// scales (per 32 elements; a 128-element block's code repeated over its four
// sub-blocks), by the rule pack_fp8_kernel applies, computed from the bf16 xn.
// One warp per row, two passes over it (sum of squares, then normalise); the
// second reads the row again from L2. Lane l covers 8 consecutive elements
// per 256-element step: a 128-element block is 16 lanes, a 32-element one 4.
template <int AFMT>
__global__ void __launch_bounds__(256) rmsnorm_quant_kernel(const uint4* __restrict__ x, int H,
                                                            const float4* __restrict__ w,
                                                            double eps, int T,
                                                            uint4* __restrict__ xn,
                                                            uint2* __restrict__ q,
                                                            uint8_t* __restrict__ qs) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (t >= T) return;
    const int H8 = H / 8;
    const uint4* row = x + (size_t)t * H8;
    double ss = 0.0;
    int v = lane;
    for (; v + 96 < H8; v += 128) {
        const uint4 u[4] = {row[v], row[v + 32], row[v + 64], row[v + 96]};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u[j]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(b[i]);
                ss = fma((double)f.x, (double)f.x, ss);
                ss = fma((double)f.y, (double)f.y, ss);
            }
        }
    }
    for (; v < H8; v += 32) {
        const uint4 u = row[v];
        const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(b[i]);
            ss = fma((double)f.x, (double)f.x, ss);
            ss = fma((double)f.y, (double)f.y, ss);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const double r = 1.0 / sqrt(ss / (double)H + eps);
    uint4* orow = xn + (size_t)t * H8;
    for (int base = 0; base < H8; base += 32) {  // every lane runs every step (shuffles below)
        const int vv = base + lane;
        const bool act = vv < H8;
        uint4 u = make_uint4(0, 0, 0, 0);
        float4 w0 = make_float4(0.f, 0.f, 0.f, 0.f), w1 = w0;
        if (act) {
            u = row[vv];
            w0 = w[2 * vv];
            w1 = w[2 * vv + 1];
        }
        const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
        const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u);
        uint4 o;
        __nv_bfloat16* ob = reinterpret_cast<__nv_bfloat16*>(&o);
        float f[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 p = __bfloat1622float2(b[i]);
            ob[2 * i] = __double2bfloat16(((double)p.x * r) * (double)wv[2 * i]);
            ob[2 * i + 1] = __double2bfloat16(((double)p.y * r) * (double)wv[2 * i + 1]);
            f[2 * i] = __bfloat162float(ob[2 * i]);
            f[2 * i + 1] = __bfloat162float(ob[2 * i + 1]);
        }
        if (act) orow[vv] = o;
        if (AFMT != MOE_A_BF16) {
            constexpr int LANES = (AFMT == MOE_A_FP8_E4M3_POW2_B128) ? 16 : 4;  // lanes per block
            float amax = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
            for (int off = LANES / 2; off > 0; off >>= 1)
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
            int e = (AFMT == MOE_A_FP8_E4M3_POW2_B128) ? pow2_scale_exp(amax) : mx_scale_exp(amax);
            e = min(max(e, -127), 127);
            const float inv = __uint_as_float((uint32_t)(127 - e) << 23);  // 2^-e, e in [-127, 126]
            uint32_t pk[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const __nv_fp8x2_storage_t a = __nv_cvt_float2_to_fp8x2(
                    make_float2(f[4 * h] * inv, f[4 * h + 1] * inv), __NV_SATFINITE, __NV_E4M3);
                const __nv_fp8x2_storage_t c = __nv_cvt_float2_to_fp8x2(
                    make_float2(f[4 * h + 2] * inv, f[4 * h + 3] * inv), __NV_SATFINITE, __NV_E4M3);
                pk[h] = (uint32_t)a | ((uint32_t)c << 16);
            }
            if (act) {
                q[(size_t)t * H8 + vv] = make_uint2(pk[0], pk[1]);
                if ((lane & 3) == 0) qs[(size_t)t * (H / 32) + vv / 4] = (uint8_t)(e + 127);
            }
        }
    }
}

// NVFP4 expert input rows ("DeepSeek V3架构拆解：Kimi-K2-Thinking-NVFP4的MLA注意力与
// MoE路由实现原理", 四 NVFP4 量化: the routed experts' input activations in 4-bit
// floats, groups of 16 with an FP8 scale), with tensor scale g: per group
// s = E4M3_RNE(amax / (6 g)) and q = E2M1_RNE(v / (e4m3(s) g)), saturating at
// +-6, zero codes where s is 0. The quotients are formed in double: for bf16 v
// and fp32 g they are exact enough that every code is the one the definition
// gives. One warp per token row, one 16-element group per lane per step; the
// row's codes go to q (two per byte, even element in the low nibble), its scale
// codes to qs, and, when xb is set, the bf16 row itself to xb (the shared
// experts' input).
__device__ __forceinline__ uint32_t e2m1_code_d(double v) {
    const double a = fabs(v);
    const uint32_t c = (a > 0.25) + (a >= 0.75) + (a > 1.25) + (a >= 1.75) + (a > 2.5) +
                       (a >= 3.5) + (a > 5.0);
    return c | (signbit(v) ? 8u : 0u);
}

__global__ void __launch_bounds__(256) pack_nvfp4_kernel(const uint4* __restrict__ x, int H, double g,
                                                         int T, uint2* __restrict__ q,
                                                         uint8_t* __restrict__ qs,
                                                         uint4* __restrict__ xb) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (t >= T) return;
    const int G = H / 16;  // groups per row
    const uint4* row = x + (size_t)t * (H / 8);
    for (int gi = lane; gi < G; gi += 32) {
        const uint4 u0 = row[2 * gi], u1 = row[2 * gi + 1];
        if (xb) {
            xb[(size_t)t * (H / 8) + 2 * gi] = u0;
            xb[(size_t)t * (H / 8) + 2 * gi + 1] = u1;
        }
        float v[16];
        const __nv_bfloat162* b0 = reinterpret_cast<const __nv_bfloat162*>(&u0);
        const __nv_bfloat162* b1 = reinterpret_cast<const __nv_bfloat162*>(&u1);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f0 = __bfloat1622float2(b0[i]), f1 = __bfloat1622float2(b1[i]);
            v[2 * i] = f0.x;
            v[2 * i + 1] = f0.y;
            v[8 + 2 * i] = f1.x;
            v[8 + 2 * i + 1] = f1.y;
        }
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
        const __nv_fp8_storage_t s8 =
            __nv_cvt_double_to_fp8((double)amax / (6.0 * g), __NV_SATFINITE, __NV_E4M3);
        const double sg = (double)__half2float(__nv_cvt_fp8_to_halfraw(s8, __NV_E4M3)) * g;
        uint32_t w[2] = {0u, 0u};
        if (sg > 0.0) {
#pragma unroll
            for (int i = 0; i < 16; ++i) w[i >> 3] |= e2m1_code_d((double)v[i] / sg) << (4 * (i & 7));
        }
        q[(size_t)t * G + gi] = make_uint2(w[0], w[1]);
        qs[(size_t)t * G + gi] = (uint8_t)s8;
    }
}

}  // namespace

cudaError_t launch_pack_rows(int afmt, const void* x, int H, const int32_t* sorted_pair, int N,
                             int k, int T, int n_rows, void* out, uint8_t* out_scale, int per32,
                             cudaStream_t st) {
    if (n_rows == 0) return cudaSuccess;
    if (afmt == MOE_A_BF16) {
        launch_pdl(gather_rows_kernel, (n_rows + 7) / 8, 256, 0, st, static_cast<const uint4*>(x),
            0, H / 8, nullptr, 0, sorted_pair, N, k, T, n_rows, static_cast<uint4*>(out), nullptr,
            nullptr, nullptr);
        return cudaGetLastError();
    }
    const int blk = (afmt == MOE_A_FP8_E4M3_POW2_B128) ? 128 : 32;
    const int sbytes = H / (per32 ? 32 : blk);  // scale bytes per row
    // With shared-expert rows (rows N..N+T-1 are the tokens in order), quantise
    // those T rows once and gather the routed rows from them; otherwise each
    // routed row is quantised where it is gathered.
    const bool two_pass = n_rows == N + T && T > 0 && H % 16 == 0 && sbytes % 16 == 0 &&
                          reinterpret_cast<uintptr_t>(out) % 16 == 0 &&
                          reinterpret_cast<uintptr_t>(out_scale) % 16 == 0;
    const int row0 = two_pass ? N : 0;
    const int q_rows = n_rows - row0;
    dim3 grid((q_rows + 7) / 8);
    if (afmt == MOE_A_FP8_E4M3_POW2_B128)
        launch_pdl(pack_fp8_kernel<MOE_A_FP8_E4M3_POW2_B128>, grid, 256, 0, st,
            static_cast<const __nv_bfloat16*>(x), H, sorted_pair, N, k, T, n_rows,
            static_cast<uint8_t*>(out), out_scale, per32, row0);
    else
        launch_pdl(pack_fp8_kernel<MOE_A_MXFP8>, grid, 256, 0, st,
            static_cast<const __nv_bfloat16*>(x), H, sorted_pair, N, k, T, n_rows,
            static_cast<uint8_t*>(out), out_scale, per32, row0);
    if (two_pass && N > 0) {
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        launch_pdl(gather_rows_kernel, (N + 7) / 8, 256, 0, st, static_cast<const uint4*>(out), N,
            H / 16, reinterpret_cast<const uint4*>(out_scale), sbytes / 16, sorted_pair, N, k, T, N,
            static_cast<uint4*>(out), reinterpret_cast<uint4*>(out_scale), nullptr, nullptr);
    }
    return cudaGetLastError();
}

cudaError_t launch_pack_f16_rows(const void* x, int H, const int32_t* sorted_pair, int N, int k,
                                 int T, int n_rows, void* out, int8_t* xs, cudaStream_t st) {
    if (n_rows == 0) return cudaSuccess;
    // with shared-expert rows, convert the T token rows once and gather the rest
    const bool two_pass = n_rows == N + T && T > 0;
    const int row0 = two_pass ? N : 0;
    launch_pdl(pack_f16_kernel, (n_rows - row0 + 7) / 8, 256, 0, st, static_cast<const uint4*>(x),
        H / 8, sorted_pair, N, k, T, n_rows, row0, static_cast<uint4*>(out), xs);
    if (two_pass && N > 0) {
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        launch_pdl(gather_rows_kernel, (N + 7) / 8, 256, 0, st, static_cast<const uint4*>(out), N,
            H / 8, nullptr, 0, sorted_pair, N, k, T, N, static_cast<uint4*>(out), nullptr, xs, xs);
    }
    return cudaGetLastError();
}

cudaError_t launch_rows_to_f16(void* rows, int C, int n_rows, int8_t* xs, cudaStream_t st) {
    if (n_rows == 0) return cudaSuccess;
    launch_pdl(rows_to_f16_kernel, (n_rows + 7) / 8, 256, 0, st, static_cast<uint4*>(rows), C / 8,
        n_rows, xs);
    return cudaGetLastError();
}

cudaError_t launch_combine(const void* y, const void* shared_y, int S, const int32_t* row_of,
                           const float* w, int T, int k, int H, void* out, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const unsigned grid = (unsigned)T * (unsigned)((H / 8 + 127) / 128);
    const auto* yy = static_cast<const __nv_bfloat16*>(y);
    const auto* sy = static_cast<const __nv_bfloat16*>(shared_y);
    auto* o = static_cast<__nv_bfloat16*>(out);
    // enough tokens to fill the GPU with one CTA each (the column-split CTAs
    // are latency-bound: measured slower at 16384 tokens, faster at 128)
    if (T >= 8 * num_sms()) {
        launch_pdl(combine_token_kernel, T, 128, 0, st, yy, sy, S, row_of, w, T, k, H, o);
        return cudaGetLastError();
    }
    if (k + S <= 12)
        launch_pdl(combine_kernel<12>, grid, 128, 0, st, yy, sy, S, row_of, w, T, k, H, o);
    else if (k + S <= 20)
        launch_pdl(combine_kernel<20>, grid, 128, 0, st, yy, sy, S, row_of, w, T, k, H, o);
    else
        launch_pdl(combine_kernel<36>, grid, 128, 0, st, yy, sy, S, row_of, w, T, k, H, o);
    return cudaGetLastError();
}

cudaError_t launch_rmsnorm_quant(int afmt, const void* x, int H, const float* w, float eps, int T,
                                 void* xn, void* q, uint8_t* qs, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const unsigned grid = (unsigned)((T + 7) / 8);
    const auto* xx = static_cast<const uint4*>(x);
    const auto* ww = reinterpret_cast<const float4*>(w);
    auto* o = static_cast<uint4*>(xn);
    auto* qq = static_cast<uint2*>(q);
    if (afmt == MOE_A_FP8_E4M3_POW2_B128)
        launch_pdl(rmsnorm_quant_kernel<MOE_A_FP8_E4M3_POW2_B128>, grid, 256, 0, st, xx, H, ww,
            (double)eps, T, o, qq, qs);
    else if (afmt == MOE_A_MXFP8)
        launch_pdl(rmsnorm_quant_kernel<MOE_A_MXFP8>, grid, 256, 0, st, xx, H, ww, (double)eps, T, o,
            qq, qs);
    else
        launch_pdl(rmsnorm_quant_kernel<MOE_A_BF16>, grid, 256, 0, st, xx, H, ww, (double)eps, T, o,
            qq, qs);
    return cudaGetLastError();
}

cudaError_t launch_gather_token_rows(const void* rows, const uint8_t* scales, int H,
                                     const int32_t* sorted_pair, int N, int k, int T, void* out,
                                     uint8_t* out_scale, cudaStream_t st) {
    if (N == 0) return cudaSuccess;
    launch_pdl(gather_rows_kernel, (N + 7) / 8, 256, 0, st, static_cast<const uint4*>(rows), 0,
        H / 16, reinterpret_cast<const uint4*>(scales), H / 32 / 16, sorted_pair, N, k, T, N,
        static_cast<uint4*>(out), reinterpret_cast<uint4*>(out_scale), nullptr, nullptr);
    return cudaGetLastError();
}

cudaError_t launch_pack_nvfp4(const void* x, int H, float g, int T, void* q, uint8_t* qs, void* xb,
                              cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    launch_pdl(pack_nvfp4_kernel, (unsigned)((T + 7) / 8), 256, 0, st, static_cast<const uint4*>(x),
        H, (double)g, T, static_cast<uint2*>(q), qs, static_cast<uint4*>(xb));
    return cudaGetLastError();
}

cudaError_t launch_gather_nvfp4_rows(const void* rows, const uint8_t* scales, int H,
                                     const int32_t* sorted_pair, int N, int k, int T, void* out,
                                     uint8_t* out_scale, cudaStream_t st) {
    if (N == 0) return cudaSuccess;
    launch_pdl(gather_rows_kernel, (N + 7) / 8, 256, 0, st, static_cast<const uint4*>(rows), 0,
        H / 32, reinterpret_cast<const uint4*>(scales), H / 256, sorted_pair, N, k, T, N,
        static_cast<uint4*>(out), reinterpret_cast<uint4*>(out_scale), nullptr, nullptr);
    return cudaGetLastError();
}

}  // namespace moe
