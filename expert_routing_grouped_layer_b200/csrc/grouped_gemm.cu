// grouped_gemm.cu -- per-expert SwiGLU MLP on the tcgen05 tensor cores.
//
// "DeepSeek V3架构拆解：Kimi-K2-Thinking-NVFP4的MLA注意力与MoE路由实现原理", 三.4 推理执行:
// after the argsort each expert multiplies its contiguous block of tokens by
// its gate/up/down projections with SiLU; the shared experts see every token.
// ("DeepSeek-V4-Pro 架构与代码概述", 文件说明: FFNSwiGLU is the standard SwiGLU.)
//
// Two launches per layer:
//   GEMM1: for every expert block, G = X W1^T and U = X W3^T, a = SiLU(G) * U;
//   GEMM2: Y = a W2^T.
// Both run "weights as the M operand": an MMA tile is 128 weight rows (output
// features) x up to 128 tokens (N, a multiple of 16), so a decode expert with
// a handful of tokens still issues full-height MMAs and its weights stream at
// HBM speed, and a prefill expert with ~170 tokens needs only two N tiles.
//
// Kernel structure (one persistent CTA per SM, 6 warps):
//   warp 0   TMA producer: weight tiles (128 rows x 64 K, 128B-swizzled) and
//            token tiles (16-row boxes) into a ring of shared-memory stages;
//   warp 1   MMA issuer: tcgen05.mma kind::f16 (bf16 x bf16 -> fp32 in TMEM),
//            tcgen05.commit frees each stage and publishes each accumulator;
//   warps 2-5 epilogue: tcgen05.ld the accumulator (lane = weight row,
//            column = token), SwiGLU (GEMM1), bf16 stores.
// Accumulators are double-buffered in tensor memory so the epilogue of one
// tile overlaps the main loop of the next. The tile list (expert, M tile,
// N tile) is derived on the device from expert_offsets; there is no host sync.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "internal.h"
#include "sm100.cuh"

namespace moe {

namespace {

constexpr int BM = 128;   // weight rows per tile (MMA M)
constexpr int BN = 128;   // max tokens per tile (MMA N)
constexpr int BK = 64;    // bf16 elements in one 128-byte swizzled row
constexpr int B_BOX = 16; // token rows per TMA box
constexpr int MAX_SEG = 1024 + 4;

template <int GEMM>
struct Tile {
    static constexpr int NA = (GEMM == 1) ? 2 : 1;  // A tiles per stage (gate + up)
    static constexpr int A_BYTES = BM * BK * 2;
    static constexpr int B_BYTES = BN * BK * 2;
    static constexpr int STAGE_BYTES = NA * A_BYTES + B_BYTES;
    static constexpr int STAGES = (GEMM == 1) ? 4 : 6;
    static constexpr int ACC_COLS = NA * BN;        // TMEM columns of one accumulator set
    static constexpr int TMEM_COLS = 2 * ACC_COLS;  // double-buffered
    static constexpr int BAR_BYTES = 8 * (2 * STAGES + 5) + 16;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES + 4 * (MAX_SEG + 1);
};

struct KParams {
    int nseg;  // E + S
    int E, S, T, N;
    int K;               // reduction length
    int M;               // output features per matrix
    int a_rows_per_mat;  // 2I (GEMM1) or H (GEMM2)
    int a_up_offset;     // I (GEMM1): first up-projection row
    int b_shared_base;   // first B row of the shared-expert rows
    int b_shared_stride; // B-row step per shared expert
    int bn;              // tokens per tile (MMA N upper bound)
    const int32_t* offsets;
    uint8_t* out_routed;  // output rows (element size out_esize bytes)
    uint8_t* out_shared;
    int ld_out;           // output row length in elements
    int out_esize;
    uint8_t* sc_routed;   // per-32 E8M0 scales of quantised outputs (or null)
    uint8_t* sc_shared;
    int32_t* status;
};

struct Unit {
    int seg, mt, n_valid, a_row, b_row;
    uint8_t* out;  // row of the first token, column 0
    uint8_t* sc;   // its scale row (quantised outputs only)
};

__device__ __forceinline__ int seg_rows(const KParams& p, int s) {
    return s < p.E ? (p.offsets[s + 1] - p.offsets[s]) : p.T;
}

__device__ __forceinline__ Unit decode_unit(const KParams& p, const int* pref, int u) {
    int lo = 0, hi = p.nseg - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (pref[mid] <= u) lo = mid; else hi = mid - 1;
    }
    Unit t;
    t.seg = lo;
    const int m = seg_rows(p, lo);
    const int ntiles = (m + p.bn - 1) / p.bn;
    const int local = u - pref[lo];
    t.mt = local / ntiles;
    const int nt = local - t.mt * ntiles;
    t.n_valid = min(p.bn, m - nt * p.bn);
    const int ld_sc = p.ld_out / 32;
    size_t r0;
    uint8_t *out, *sc;
    if (lo < p.E) {
        t.a_row = lo * p.a_rows_per_mat + t.mt * BM;
        r0 = (size_t)p.offsets[lo] + nt * p.bn;
        t.b_row = (int)r0;
        out = p.out_routed;
        sc = p.sc_routed;
    } else {
        const int s = lo - p.E;
        t.a_row = s * p.a_rows_per_mat + t.mt * BM;
        t.b_row = p.b_shared_base + s * p.b_shared_stride + nt * p.bn;
        r0 = (size_t)s * p.T + nt * p.bn;
        out = p.out_shared;
        sc = p.sc_shared;
    }
    t.out = out + r0 * p.ld_out * p.out_esize;
    t.sc = sc ? sc + r0 * ld_sc : nullptr;
    return t;
}

// pref[s] = index of the first tile unit of segment s; pref[nseg] = total.
// Called by one full warp.
__device__ __forceinline__ void build_schedule(const KParams& p, int* pref, int MT, int lane) {
    const int per = (p.nseg + 31) / 32;
    const int s0 = lane * per;
    const int s1 = min(p.nseg, s0 + per);
    int sum = 0;
    for (int s = s0; s < s1; ++s) sum += ((seg_rows(p, s) + p.bn - 1) / p.bn) * MT;
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    int run = incl - sum;
    for (int s = s0; s < s1; ++s) {
        pref[s] = run;
        run += ((seg_rows(p, s) + p.bn - 1) / p.bn) * MT;
    }
    if (lane == 31) pref[p.nseg] = incl;
}

// Epilogue warps (4 of them, one per TMEM lane quadrant): per unit, wait for
// the accumulator, read it 16 columns at a time (lane = output feature,
// column = token), apply SwiGLU for GEMM1, store bf16, release the buffer.
template <int GEMM, int ACC_COLS>
__device__ __forceinline__ void epilogue_loop(const KParams& p, const int* pref, int total,
                                              uint32_t tmem_base, uint64_t* tfull,
                                              uint64_t* tempty, volatile int* abort_flag,
                                              int warp, int lane) {
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    const int row = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int u = blockIdx.x; u < total; u += gridDim.x) {
        const Unit t = decode_unit(p, pref, u);
        if (!mbar_wait(&tfull[acc], acc_phase, abort_flag)) break;
        tc_fence_after();
        const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * ACC_COLS;
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(t.out) + t.mt * BM + row;
        for (int c0 = 0; c0 < t.n_valid; c0 += 16) {
            uint32_t g[16];
            tmem_ld16(taddr + c0, g);
            if (GEMM == 1) {
                uint32_t uu[16];
                tmem_ld16(taddr + ACC_COLS / 2 + c0, uu);
                tmem_ld_wait(g, uu);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    if (c0 + j < t.n_valid) {
                        const float gv = __uint_as_float(g[j]);
                        const float a = gv / (1.0f + __expf(-gv)) * __uint_as_float(uu[j]);
                        out[(size_t)(c0 + j) * p.ld_out] = __float2bfloat16_rn(a);
                    }
                }
            } else {
                tmem_ld_wait(g);
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    if (c0 + j < t.n_valid)
                        out[(size_t)(c0 + j) * p.ld_out] = __float2bfloat16_rn(__uint_as_float(g[j]));
            }
        }
        tc_fence_before();
        mbar_arrive(&tempty[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
}

template <int GEMM>
__global__ void __launch_bounds__(192, 1)
    grouped_gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA_routed,
                             const __grid_constant__ CUtensorMap tmA_shared,
                             const __grid_constant__ CUtensorMap tmB, const KParams p) {
    using C = Tile<GEMM>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
    uint64_t* empty = full + C::STAGES;
    uint64_t* tfull = empty + C::STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* mma_done = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* pref = reinterpret_cast<int*>(tmem_slot + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 128);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmA_routed);
        tma_prefetch_desc(&tmA_shared);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    // tile schedule: pref[s] = first unit of segment s
    const int MT = p.M / BM;
    if (warp == 1) build_schedule(p, pref, MT, lane);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int total = pref[p.nseg];
    const int KB = p.K / BK;

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            for (int u = blockIdx.x; u < total && !*abort_flag; u += gridDim.x) {
                const Unit t = decode_unit(p, pref, u);
                const int n_mma = (t.n_valid + 15) & ~15;
                const int nb = n_mma / B_BOX;
                const uint32_t tx = C::NA * C::A_BYTES + nb * B_BOX * BK * 2;
                const CUtensorMap* tmA = (t.seg < p.E) ? &tmA_routed : &tmA_shared;
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
                    uint8_t* st = smem + stage * C::STAGE_BYTES;
                    mbar_arrive_expect_tx(&full[stage], tx);
                    tma_load_2d(st, tmA, kb * BK, t.a_row, &full[stage]);
                    if (GEMM == 1)
                        tma_load_2d(st + C::A_BYTES, tmA, kb * BK, t.a_row + p.a_up_offset, &full[stage]);
                    uint8_t* sb = st + C::NA * C::A_BYTES;
                    for (int i = 0; i < nb; ++i)
                        tma_load_2d(sb + i * B_BOX * BK * 2, &tmB, kb * BK, t.b_row + i * B_BOX,
                                    &full[stage]);
                    ++issued;
                    if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
            }
            if (*abort_flag) {
                // let every copy this thread issued land before the CTA exits
                int s = stage;
                uint32_t ph = phase;
                for (int i = 0; i < min(issued, C::STAGES); ++i) {
                    if (--s < 0) { s = C::STAGES - 1; ph ^= 1; }
                    volatile int no_abort = 0;
                    mbar_wait(&full[s], ph, &no_abort);
                }
                status_or(p.status, MOE_DEV_TIMEOUT);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            for (int u = blockIdx.x; u < total; u += gridDim.x) {
                const Unit t = decode_unit(p, pref, u);
                const int n_mma = (t.n_valid + 15) & ~15;
                const uint32_t idesc = idesc_bf16(BM, n_mma);
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1, abort_flag)) break;
                tc_fence_after();
                const uint32_t d0 = tmem_base + acc * C::ACC_COLS;
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t st = smem_u32(smem + stage * C::STAGE_BYTES);
                    const uint32_t sb = st + C::NA * C::A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint32_t acc_flag = (kb | kk) != 0;
                        const uint64_t bd = sdesc_kmajor_sw128(sb + kk * 32);
                        mma_bf16(d0, sdesc_kmajor_sw128(st + kk * 32), bd, idesc, acc_flag);
                        if (GEMM == 1)
                            mma_bf16(d0 + BN, sdesc_kmajor_sw128(st + C::A_BYTES + kk * 32), bd, idesc,
                                     acc_flag);
                    }
                    mma_commit(&empty[stage]);
                    if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                mma_commit(&tfull[acc]);
                if (++acc == 2) { acc = 0; acc_phase ^= 1; }
            }
            // every MMA this thread issued has finished once mma_done flips
            mma_commit(mma_done);
            volatile int no_abort = 0;
            mbar_wait(mma_done, 0, &no_abort);
            if (*abort_flag) status_or(p.status, MOE_DEV_TIMEOUT);
        }
    } else {
        epilogue_loop<GEMM, C::ACC_COLS>(p, pref, total, tmem_base, tfull, tempty, abort_flag,
                                         warp, lane);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}


// ---------------------------------------------------------------- FP8 weights
// E4M3 weights with one fp32 scale per 128x128 block ("DeepSeek-V4-Pro 架构与代码概述",
// 文件说明: Linear with block-scaled FP8 weights; block 128x128). The activations
// stay bf16, so the tensor-core operands are bf16: a converter warpgroup turns
// each TMA-staged E4M3 weight tile (64-byte swizzled rows) into bf16 values
// times the tile's block scale, written straight into the 128B-swizzled
// K-major layout tcgen05.mma reads. With BK = 64 inside a 128-wide scale block
// and M tiles aligned to the 128-row blocks, one scalar scale covers a tile.
// E4M3 -> bf16 is exact; the product with the fp32 scale is rounded once to
// bf16 (relative error <= 2^-9 per weight).
constexpr int CVT_WARPS = 8;
constexpr int CVT_THREADS = CVT_WARPS * 32;
constexpr int F8_THREADS = 64 + 128 + CVT_THREADS;

template <int GEMM>
struct TileF8 {
    static constexpr int NA = (GEMM == 1) ? 2 : 1;
    static constexpr int A8_BYTES = BM * BK;      // e4m3 staging tile
    static constexpr int A_BYTES = BM * BK * 2;   // bf16 MMA tile
    static constexpr int B_BYTES = BN * BK * 2;
    static constexpr int CVT_OFF = 0;                       // NA bf16 A tiles
    static constexpr int B_OFF = NA * A_BYTES;              // token tile
    static constexpr int A8_OFF = B_OFF + B_BYTES;          // NA e4m3 tiles
    static constexpr int STAGE_BYTES = A8_OFF + NA * A8_BYTES;
    static constexpr int STAGES = (GEMM == 1) ? 3 : 5;
    static constexpr int ACC_COLS = NA * BN;
    static constexpr int TMEM_COLS = 2 * ACC_COLS;
    static constexpr int BAR_BYTES = 8 * (4 * STAGES + 5) + 16;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES + 4 * (MAX_SEG + 1);
};

// 16 E4M3 values -> 16 bf16 values of (value * scale), in element order.
__device__ __forceinline__ void e4m3x16_to_bf16_scaled(uint4 v, float scale, uint4& lo, uint4& hi) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const __nv_fp8x2_storage_t pair = (__nv_fp8x2_storage_t)((w[i] >> (16 * h)) & 0xFFFFu);
            const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
            const __nv_bfloat162 b = __floats2bfloat162_rn(f.x * scale, f.y * scale);
            o[2 * i + h] = *reinterpret_cast<const uint32_t*>(&b);
        }
    }
    lo = make_uint4(o[0], o[1], o[2], o[3]);
    hi = make_uint4(o[4], o[5], o[6], o[7]);
}

template <int GEMM>
__global__ void __launch_bounds__(F8_THREADS, 1)
    grouped_gemm_fp8w_kernel(const __grid_constant__ CUtensorMap tmA_routed,
                             const __grid_constant__ CUtensorMap tmA_shared,
                             const __grid_constant__ CUtensorMap tmB, const KParams p,
                             const float* __restrict__ scale_routed,
                             const float* __restrict__ scale_shared) {
    using C = TileF8<GEMM>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* raw_full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
    uint64_t* raw_empty = raw_full + C::STAGES;
    uint64_t* cvt_full = raw_empty + C::STAGES;
    uint64_t* cvt_empty = cvt_full + C::STAGES;
    uint64_t* tfull = cvt_empty + C::STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* mma_done = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* pref = reinterpret_cast<int*>(tmem_slot + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&raw_full[s], 1);
            mbar_init(&raw_empty[s], 1 + CVT_THREADS);  // MMA commit + every converter thread
            mbar_init(&cvt_full[s], CVT_THREADS);
            mbar_init(&cvt_empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 128);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmA_routed);
        tma_prefetch_desc(&tmA_shared);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    const int MT = p.M / BM;
    if (warp == 1) build_schedule(p, pref, MT, lane);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int total = pref[p.nseg];
    const int KB = p.K / BK;

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            for (int u = blockIdx.x; u < total && !*abort_flag; u += gridDim.x) {
                const Unit t = decode_unit(p, pref, u);
                const int n_mma = (t.n_valid + 15) & ~15;
                const int nb = n_mma / B_BOX;
                const uint32_t tx = C::NA * C::A8_BYTES + nb * B_BOX * BK * 2;
                const CUtensorMap* tmA = (t.seg < p.E) ? &tmA_routed : &tmA_shared;
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&raw_empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
                    uint8_t* st = smem + stage * C::STAGE_BYTES;
                    mbar_arrive_expect_tx(&raw_full[stage], tx);
                    tma_load_2d(st + C::A8_OFF, tmA, kb * BK, t.a_row, &raw_full[stage]);
                    if (GEMM == 1)
                        tma_load_2d(st + C::A8_OFF + C::A8_BYTES, tmA, kb * BK,
                                    t.a_row + p.a_up_offset, &raw_full[stage]);
                    for (int i = 0; i < nb; ++i)
                        tma_load_2d(st + C::B_OFF + i * B_BOX * BK * 2, &tmB, kb * BK,
                                    t.b_row + i * B_BOX, &raw_full[stage]);
                    ++issued;
                    if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
            }
            if (*abort_flag) {
                int s = stage;
                uint32_t ph = phase;
                for (int i = 0; i < min(issued, C::STAGES); ++i) {
                    if (--s < 0) { s = C::STAGES - 1; ph ^= 1; }
                    volatile int no_abort = 0;
                    mbar_wait(&raw_full[s], ph, &no_abort);
                }
                status_or(p.status, MOE_DEV_TIMEOUT);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            for (int u = blockIdx.x; u < total; u += gridDim.x) {
                const Unit t = decode_unit(p, pref, u);
                const int n_mma = (t.n_valid + 15) & ~15;
                const uint32_t idesc = idesc_bf16(BM, n_mma);
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1, abort_flag)) break;
                tc_fence_after();
                const uint32_t d0 = tmem_base + acc * C::ACC_COLS;
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&raw_full[stage], phase, abort_flag) ||
                        !mbar_wait(&cvt_full[stage], phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t st = smem_u32(smem + stage * C::STAGE_BYTES);
                    const uint32_t sb = st + C::B_OFF;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint32_t acc_flag = (kb | kk) != 0;
                        const uint64_t bd = sdesc_kmajor_sw128(sb + kk * 32);
                        mma_bf16(d0, sdesc_kmajor_sw128(st + C::CVT_OFF + kk * 32), bd, idesc, acc_flag);
                        if (GEMM == 1)
                            mma_bf16(d0 + BN, sdesc_kmajor_sw128(st + C::CVT_OFF + C::A_BYTES + kk * 32),
                                     bd, idesc, acc_flag);
                    }
                    mma_commit(&raw_empty[stage]);
                    mma_commit(&cvt_empty[stage]);
                    if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                mma_commit(&tfull[acc]);
                if (++acc == 2) { acc = 0; acc_phase ^= 1; }
            }
            mma_commit(mma_done);
            volatile int no_abort = 0;
            mbar_wait(mma_done, 0, &no_abort);
            if (*abort_flag) status_or(p.status, MOE_DEV_TIMEOUT);
        }
    } else if (warp < 6) {
        epilogue_loop<GEMM, C::ACC_COLS>(p, pref, total, tmem_base, tfull, tempty, abort_flag,
                                         warp, lane);
    } else {
        // converters: e4m3 staging tile -> scaled bf16 MMA tile
        const int ct = threadIdx.x - 192;
        const int KS = p.K / 128;  // scale blocks along K
        const int RS = p.a_rows_per_mat / 128;
        int stage = 0;
        uint32_t phase = 0;
        for (int u = blockIdx.x; u < total; u += gridDim.x) {
            const Unit t = decode_unit(p, pref, u);
            const bool routed = t.seg < p.E;
            const int mat = routed ? t.seg : t.seg - p.E;
            const float* sbase = (routed ? scale_routed : scale_shared) + (size_t)mat * RS * KS;
            const float* s_gate = sbase + (size_t)(t.mt) * KS;
            const float* s_up = sbase + (size_t)(p.a_up_offset / 128 + t.mt) * KS;
            bool ok = true;
            for (int kb = 0; kb < KB; ++kb) {
                if (!mbar_wait(&raw_full[stage], phase, abort_flag) ||
                    !mbar_wait(&cvt_empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
                uint8_t* st = smem + stage * C::STAGE_BYTES;
                const float sc[2] = {s_gate[kb >> 1], GEMM == 1 ? s_up[kb >> 1] : 0.f};
#pragma unroll
                for (int i = 0; i < C::NA * 512 / CVT_THREADS; ++i) {
                    const int task = ct + i * CVT_THREADS;
                    const int tile = task >> 9;
                    const int r = task & 127;
                    const int c = (task >> 7) & 3;
                    const uint8_t* src = st + C::A8_OFF + tile * C::A8_BYTES + r * 64 +
                                         ((c ^ ((r >> 1) & 3)) << 4);
                    uint8_t* dst = st + C::CVT_OFF + tile * C::A_BYTES + r * 128;
                    uint4 lo, hi;
                    e4m3x16_to_bf16_scaled(*reinterpret_cast<const uint4*>(src), sc[tile], lo, hi);
                    *reinterpret_cast<uint4*>(dst + (((2 * c) ^ (r & 7)) << 4)) = lo;
                    *reinterpret_cast<uint4*>(dst + (((2 * c + 1) ^ (r & 7)) << 4)) = hi;
                }
                fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor core
                mbar_arrive(&cvt_full[stage]);
                mbar_arrive(&raw_empty[stage]);
                if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
            }
            if (!ok) break;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}


// ---------------------------------------------------------------- block-scaled
// E2M1 weights with one E8M0 scale per 32 elements ("DeepSeek-V4-Pro 架构与代码概述",
// 架构: FP4 experts with UE8M0 scales, kernel.py fp4_quant_kernel block 32;
// "开源巨头开放2.8T MoE权重:架构创新与本地部署实践指南", 存储与量化策略: MXFP4 weights)
// times E4M3 activations with one E8M0 scale per 32 elements (MXFP8, or the
// per-128 power-of-two activation scale repeated over its four 32-blocks).
// tcgen05.mma kind::mxf8f6f4 applies both scales inside the MMA, so the FP4
// weights are never dequantised in software: TMA expands each packed row of
// 128 E2M1 values to the one-byte-per-value layout the MMA reads
// (16U4_ALIGN16B). Scales travel by TMA as 128 rows x 16 bytes (16 k-blocks);
// a scale warp regroups the 4 k-blocks of the current stage into the 512-byte
// order tcgen05.cp.32x128b.warpx4 expects (row m = m0 + 32*m1 at byte
// 16*m0 + 4*m1 + kb), which puts row m's scales in lane m mod 32 of every lane
// quadrant, column m / 32, one k-block per byte.
// GEMM1's epilogue quantises the SwiGLU output per 32 (MXFP8) or per 128
// (power of two) along I, exactly as the activation quantiser does.
constexpr int MX_BK = 128;        // K elements per stage (one 128-byte smem row)
constexpr int SF_TILE = 128 * 16; // scale tile: 128 rows x 16 k-blocks of 32

template <int GEMM>
struct TileMX {
    static constexpr int NA = (GEMM == 1) ? 2 : 1;
    static constexpr int BNX = (GEMM == 1) ? 64 : 128;  // tokens per tile
    static constexpr int A_BYTES = BM * MX_BK;          // one byte per E2M1 value in smem
    static constexpr int B_BYTES = BNX * MX_BK;
    static constexpr int A_OFF = 0;
    static constexpr int B_OFF = NA * A_BYTES;
    static constexpr int SFA_OFF = B_OFF + B_BYTES;
    static constexpr int SFB_OFF = SFA_OFF + NA * SF_TILE;
    static constexpr int ATOM_OFF = SFB_OFF + SF_TILE;  // regrouped scales: A gate, [A up], B
    static constexpr int STAGE_BYTES = ((ATOM_OFF + (NA + 1) * 512) + 1023) / 1024 * 1024;
    static constexpr int STAGES = (GEMM == 1) ? 4 : 5;
    static constexpr int ACC_COLS = NA * BNX;
    static constexpr int SF_COL = 2 * ACC_COLS;  // scale columns: A gate, A up, B (4 each)
    static constexpr int TMEM_COLS = 512;
    static constexpr int BAR_BYTES = 8 * (3 * STAGES + 7) + 16;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES + 4 * (MAX_SEG + 1) +
                                      2 * 4 * 16 * 4;  // + cross-warp amax exchange
};

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
    return v;
}

// exponent of the power-of-two scale: smallest e with a <= 448 * 2^e (a >= 0)
__device__ __forceinline__ int pow2_exp448(float a) {
    if (a == 0.0f) return 0;
    int adj = 0;
    uint32_t b = __float_as_uint(a);
    if ((b >> 23) == 0) {
        b = __float_as_uint(a * 0x1p64f);
        adj = -64;
    }
    const int E = (int)(b >> 23) - 127;
    return E - 8 + ((b & 0x7FFFFFu) > 0x600000u ? 1 : 0) + adj;
}

// OCP MX shared exponent for E4M3 elements: floor(log2 a) - 8
__device__ __forceinline__ int mx_exp(float a) {
    const int f = (int)(__float_as_uint(a) >> 23);
    return f == 0 ? -127 : max(f - 135, -127);
}

__device__ __forceinline__ uint8_t e4m3_sat(float v) {
    return (uint8_t)(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3));
}

template <int GEMM, int AFMT>
__global__ void __launch_bounds__(224, 1)
    grouped_gemm_mx_kernel(const __grid_constant__ CUtensorMap tmA_routed,
                           const __grid_constant__ CUtensorMap tmA_shared,
                           const __grid_constant__ CUtensorMap tmSFA_routed,
                           const __grid_constant__ CUtensorMap tmSFA_shared,
                           const __grid_constant__ CUtensorMap tmB,
                           const __grid_constant__ CUtensorMap tmSFB, const KParams p) {
    using C = TileMX<GEMM>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
    uint64_t* empty = full + C::STAGES;
    uint64_t* sf_ready = empty + C::STAGES;  // scales regrouped for the stage
    uint64_t* tfull = sf_ready + C::STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* mma_done = tempty + 2;
    uint64_t* red_bar = mma_done + 1;  // [2]: the 4 epilogue warps' amax exchange
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(red_bar + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* pref = reinterpret_cast<int*>(tmem_slot + 4);
    float* red = reinterpret_cast<float*>(pref + MAX_SEG + 1);  // [2][4 warps][16 columns]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&sf_ready[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 128);
        }
        mbar_init(mma_done, 1);
        mbar_init(&red_bar[0], 4);
        mbar_init(&red_bar[1], 4);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmA_routed);
        tma_prefetch_desc(&tmA_shared);
        tma_prefetch_desc(&tmSFA_routed);
        tma_prefetch_desc(&tmSFA_shared);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmSFB);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    const int MT = p.M / BM;
    if (warp == 1) build_schedule(p, pref, MT, lane);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int total = pref[p.nseg];
    const int KB = p.K / MX_BK;

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            for (int u = blockIdx.x; u < total && !*abort_flag; u += gridDim.x) {
                const Unit t = decode_unit(p, pref, u);
                const int n_mma = (t.n_valid + 15) & ~15;
                const int nb = n_mma / B_BOX;
                // a padded E2M1 tile occupies A_BYTES of shared memory but the copy
                // counts its packed size (4 bits per value) toward the transaction
                const uint32_t tx =
                    C::NA * (C::A_BYTES / 2 + SF_TILE) + nb * B_BOX * MX_BK + SF_TILE;
                const bool routed = t.seg < p.E;
                const CUtensorMap* tmA = routed ? &tmA_routed : &tmA_shared;
                const CUtensorMap* tmSFA = routed ? &tmSFA_routed : &tmSFA_shared;
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
                    uint8_t* st = smem + stage * C::STAGE_BYTES;
                    const int sfx = (kb >> 2) * 16;  // 16-k-block group holding this stage
                    mbar_arrive_expect_tx(&full[stage], tx);
                    tma_load_2d(st + C::A_OFF, tmA, kb * MX_BK, t.a_row, &full[stage]);
                    tma_load_2d(st + C::SFA_OFF, tmSFA, sfx, t.a_row, &full[stage]);
                    if (GEMM == 1) {
                        tma_load_2d(st + C::A_OFF + C::A_BYTES, tmA, kb * MX_BK,
                                    t.a_row + p.a_up_offset, &full[stage]);
                        tma_load_2d(st + C::SFA_OFF + SF_TILE, tmSFA, sfx, t.a_row + p.a_up_offset,
                                    &full[stage]);
                    }
                    for (int i = 0; i < nb; ++i)
                        tma_load_2d(st + C::B_OFF + i * B_BOX * MX_BK, &tmB, kb * MX_BK,
                                    t.b_row + i * B_BOX, &full[stage]);
                    tma_load_2d(st + C::SFB_OFF, &tmSFB, sfx, t.b_row, &full[stage]);
                    ++issued;
                    if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
            }
            if (*abort_flag) {
                int s = stage;
                uint32_t ph = phase;
                for (int i = 0; i < min(issued, C::STAGES); ++i) {
                    if (--s < 0) { s = C::STAGES - 1; ph ^= 1; }
                    volatile int no_abort = 0;
                    mbar_wait(&full[s], ph, &no_abort);
                }
                status_or(p.status, MOE_DEV_TIMEOUT);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            const uint32_t sfa_gate = tmem_base + C::SF_COL;
            const uint32_t sfa_up = tmem_base + C::SF_COL + 4;
            const uint32_t sfb = tmem_base + C::SF_COL + 8;
            for (int u = blockIdx.x; u < total; u += gridDim.x) {
                const Unit t = decode_unit(p, pref, u);
                const int n_mma = (t.n_valid + 15) & ~15;
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1, abort_flag)) break;
                tc_fence_after();
                const uint32_t d0 = tmem_base + acc * C::ACC_COLS;
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&full[stage], phase, abort_flag) ||
                        !mbar_wait(&sf_ready[stage], phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t st = smem_u32(smem + stage * C::STAGE_BYTES);
                    tmem_cp_32x128b_x4(sfa_gate, sdesc_kmajor_noswizzle_rows16(st + C::ATOM_OFF));
                    if (GEMM == 1)
                        tmem_cp_32x128b_x4(sfa_up,
                                           sdesc_kmajor_noswizzle_rows16(st + C::ATOM_OFF + 512));
                    tmem_cp_32x128b_x4(sfb, sdesc_kmajor_noswizzle_rows16(st + C::ATOM_OFF +
                                                                          C::NA * 512));
#pragma unroll
                    for (int kk = 0; kk < MX_BK / 32; ++kk) {
                        const uint32_t acc_flag = (kb | kk) != 0;
                        const uint32_t idesc = idesc_mx_e2m1_e4m3(BM, n_mma, kk, kk);
                        const uint32_t sub = (uint32_t)kk << 30;  // k-block byte in each column
                        const uint64_t bd = sdesc_kmajor_sw128(st + C::B_OFF + kk * 32);
                        mma_mx(d0, sdesc_kmajor_sw128(st + C::A_OFF + kk * 32), bd, idesc,
                               sfa_gate | sub, sfb | sub, acc_flag);
                        if (GEMM == 1)
                            mma_mx(d0 + C::BNX, sdesc_kmajor_sw128(st + C::A_OFF + C::A_BYTES + kk * 32),
                                   bd, idesc, sfa_up | sub, sfb | sub, acc_flag);
                    }
                    mma_commit(&empty[stage]);
                    if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                mma_commit(&tfull[acc]);
                if (++acc == 2) { acc = 0; acc_phase ^= 1; }
            }
            mma_commit(mma_done);
            volatile int no_abort = 0;
            mbar_wait(mma_done, 0, &no_abort);
            if (*abort_flag) status_or(p.status, MOE_DEV_TIMEOUT);
        }
    } else if (warp == 6) {
        // scale warp: regroup this stage's 4 k-blocks of every 128 x 16-byte scale
        // tile into the tcgen05.cp 32x128b order (lane m0 gathers rows m0 + 32*m1)
        int stage = 0;
        uint32_t phase = 0;
        for (int u = blockIdx.x; u < total; u += gridDim.x) {
            bool ok = true;
            for (int kb = 0; kb < KB; ++kb) {
                if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
                uint8_t* st = smem + stage * C::STAGE_BYTES;
                const int j4 = (kb & 3) * 4;  // byte offset of this stage's k-blocks in a row
#pragma unroll
                for (int tile = 0; tile < C::NA + 1; ++tile) {
                    const uint8_t* src = st + (tile < C::NA ? C::SFA_OFF + tile * SF_TILE : C::SFB_OFF);
                    uint4 v;
                    v.x = *reinterpret_cast<const uint32_t*>(src + 16 * (lane + 0) + j4);
                    v.y = *reinterpret_cast<const uint32_t*>(src + 16 * (lane + 32) + j4);
                    v.z = *reinterpret_cast<const uint32_t*>(src + 16 * (lane + 64) + j4);
                    v.w = *reinterpret_cast<const uint32_t*>(src + 16 * (lane + 96) + j4);
                    *reinterpret_cast<uint4*>(st + C::ATOM_OFF + tile * 512 + 16 * lane) = v;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sf_ready[stage]);
                if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
            }
            if (!ok) break;
        }
    } else if (GEMM == 2) {
        epilogue_loop<2, C::ACC_COLS>(p, pref, total, tmem_base, tfull, tempty, abort_flag, warp,
                                      lane);
    } else {
        // GEMM1 epilogue: SwiGLU, then E4M3 + E8M0 block quantisation along I
        const int q = warp & 3;
        const int row = q * 32 + lane;
        int acc = 0;
        uint32_t acc_phase = 0;
        int chunk = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
            const Unit t = decode_unit(p, pref, u);
            if (!mbar_wait(&tfull[acc], acc_phase, abort_flag)) break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * C::ACC_COLS;
            const int feat = t.mt * BM + row;  // output feature (column of h)
            uint8_t* out = t.out + feat;
            uint8_t* sc = t.sc + (t.mt * BM + q * 32) / 32;
            const int ld_sc = p.ld_out / 32;
            for (int c0 = 0; c0 < t.n_valid; c0 += 16, ++chunk) {
                uint32_t g[16], uu[16];
                tmem_ld16(taddr + c0, g);
                tmem_ld16(taddr + C::BNX + c0, uu);
                tmem_ld_wait(g, uu);
                float a[16], wmax[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float gv = __uint_as_float(g[j]);
                    a[j] = gv / (1.0f + __expf(-gv)) * __uint_as_float(uu[j]);
                    wmax[j] = warp_max(fabsf(a[j]));
                }
                int e[16];
                if (AFMT == MOE_A_MXFP8) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) e[j] = mx_exp(wmax[j]);
                } else {
                    // block of 128 features = the 4 epilogue warps: exchange warp maxima
                    const int par = chunk & 1;
                    float* r = red + par * 64;
                    if (lane < 16) {
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            if (j == lane) r[q * 16 + j] = wmax[j];
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&red_bar[par]);
                    if (!mbar_wait(&red_bar[par], (chunk >> 1) & 1, abort_flag)) { ok = false; break; }
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float m = fmaxf(fmaxf(r[j], r[16 + j]), fmaxf(r[32 + j], r[48 + j]));
                        e[j] = pow2_exp448(m);
                    }
                }
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    if (c0 + j < t.n_valid) {
                        const int ej = min(max(e[j], -127), 127);
                        const float inv = __uint_as_float((uint32_t)(127 - ej) << 23);
                        out[(size_t)(c0 + j) * p.ld_out] = e4m3_sat(a[j] * inv);
                        if (lane == 0) sc[(size_t)(c0 + j) * ld_sc] = (uint8_t)(ej + 127);
                    }
                }
            }
            if (!ok) break;
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
            if (++acc == 2) { acc = 0; acc_phase ^= 1; }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// 2-D row-major bf16 tensor [rows][cols], box = box_rows x 64 columns, 128B swizzle.
bool make_tmap_bf16(CUtensorMap* tm, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 2-D row-major uint8 tensor [rows][cols], box = box_rows x 64 bytes, 64B swizzle.
bool make_tmap_u8_sw64(CUtensorMap* tm, const void* ptr, uint64_t rows, uint64_t cols,
                       uint32_t box_rows) {
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols};
    cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Problem geometry shared by every variant of the two GEMMs.
KParams make_params(const GroupedGemmArgs& a, int GEMM, uint64_t* b_rows) {
    KParams p;
    p.nseg = a.E + a.S;
    p.E = a.E;
    p.S = a.S;
    p.T = a.T;
    p.N = a.N;
    p.offsets = a.offsets;
    p.status = a.status;
    if (GEMM == 1) {
        p.K = a.H;
        p.M = a.I;
        p.a_rows_per_mat = 2 * a.I;
        p.a_up_offset = a.I;
        p.b_shared_base = a.N;
        p.b_shared_stride = 0;
        p.ld_out = a.I;
        *b_rows = (uint64_t)a.N + a.T;
    } else {
        p.K = a.I;
        p.M = a.H;
        p.a_rows_per_mat = a.H;
        p.a_up_offset = 0;
        p.b_shared_base = a.N;
        p.b_shared_stride = a.T;
        p.ld_out = a.H;
        *b_rows = (uint64_t)a.N + (uint64_t)a.S * a.T;
    }
    p.bn = BN;
    p.out_routed = static_cast<uint8_t*>(a.out_routed);
    p.out_shared = static_cast<uint8_t*>(a.out_shared);
    p.out_esize = 2;
    p.sc_routed = p.sc_shared = nullptr;
    return p;
}

int grid_for(const KParams& p) {
    // upper bound on tiles: sum_e ceil(m_e/BN) <= N/BN + min(E, N), plus shared
    const long MT = p.M / BM;
    const long routed_tiles = (long)p.N / p.bn + std::min<long>(p.E, p.N);
    const long shared_tiles = (long)p.S * ((p.T + p.bn - 1) / p.bn);
    const long units_max = (routed_tiles + shared_tiles) * MT;
    return (int)std::max<long>(1, std::min<long>(num_sms(), units_max));
}


// 2-D tensor map helper: `dtype` elements, rows x cols, box_cols x box_rows.
bool make_tmap_2d(CUtensorMap* tm, CUtensorMapDataType dtype, const void* ptr, uint64_t rows,
                  uint64_t cols, uint64_t row_bytes, uint32_t box_cols, uint32_t box_rows,
                  CUtensorMapSwizzle swz) {
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(tm, dtype, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int GEMM, int AFMT>
cudaError_t launch_mx(const GroupedGemmArgs& a, cudaStream_t st) {
    using C = TileMX<GEMM>;
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(grouped_gemm_mx_kernel<GEMM, AFMT>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    });
    if (attr_err != cudaSuccess) return attr_err;
    uint64_t b_rows;
    KParams p = make_params(a, GEMM, &b_rows);
    p.bn = C::BNX;
    if (GEMM == 1) {
        p.out_esize = 1;  // E4M3 intermediate
        p.sc_routed = a.out_routed_scale;
        p.sc_shared = a.out_shared_scale;
    }
    const int S = a.S;
    const uint64_t K = p.K, rowsA = (uint64_t)a.E * p.a_rows_per_mat;
    const uint64_t rowsAs = (uint64_t)(S > 0 ? S : a.E) * p.a_rows_per_mat;
    const void* wA = a.w_routed;
    const void* wAs = S > 0 ? a.w_shared : a.w_routed;
    const void* sA = a.w_routed_scale;
    const void* sAs = S > 0 ? a.w_shared_scale : a.w_routed_scale;
    CUtensorMap tmA, tmAs, tmSFA, tmSFAs, tmB, tmSFB;
    if (!make_tmap_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, wA, rowsA, K, K / 2, MX_BK, BM,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_2d(&tmAs, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, wAs, rowsAs, K, K / 2, MX_BK, BM,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_2d(&tmSFA, CU_TENSOR_MAP_DATA_TYPE_UINT8, sA, rowsA, K / 32, K / 32, 16, 128,
                      CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_tmap_2d(&tmSFAs, CU_TENSOR_MAP_DATA_TYPE_UINT8, sAs, rowsAs, K / 32, K / 32, 16, 128,
                      CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    if (b_rows == 0) return cudaSuccess;
    if (!make_tmap_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.b_rows, b_rows, K, K, MX_BK, B_BOX,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_2d(&tmSFB, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.b_scale, b_rows, K / 32, K / 32, 16,
                      128, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    grouped_gemm_mx_kernel<GEMM, AFMT><<<grid_for(p), 224, C::SMEM_BYTES, st>>>(
        tmA, tmAs, tmSFA, tmSFAs, tmB, tmSFB, p);
    return cudaGetLastError();
}

template <int GEMM>
cudaError_t launch_fp8w(const GroupedGemmArgs& a, cudaStream_t st) {
    using C = TileF8<GEMM>;
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(grouped_gemm_fp8w_kernel<GEMM>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    });
    if (attr_err != cudaSuccess) return attr_err;
    uint64_t b_rows;
    const KParams p = make_params(a, GEMM, &b_rows);
    CUtensorMap tmAr, tmAs, tmB;
    const int S = a.S;
    if (!make_tmap_u8_sw64(&tmAr, a.w_routed, (uint64_t)a.E * p.a_rows_per_mat, p.K, BM))
        return cudaErrorInvalidValue;
    if (!make_tmap_u8_sw64(&tmAs, S > 0 ? a.w_shared : a.w_routed,
                           (uint64_t)(S > 0 ? S : a.E) * p.a_rows_per_mat, p.K, BM))
        return cudaErrorInvalidValue;
    if (b_rows == 0) return cudaSuccess;
    if (!make_tmap_bf16(&tmB, a.b_rows, b_rows, p.K, B_BOX)) return cudaErrorInvalidValue;
    grouped_gemm_fp8w_kernel<GEMM><<<grid_for(p), F8_THREADS, C::SMEM_BYTES, st>>>(
        tmAr, tmAs, tmB, p, static_cast<const float*>(a.w_routed_scale),
        static_cast<const float*>(S > 0 ? a.w_shared_scale : a.w_routed_scale));
    return cudaGetLastError();
}

template <int GEMM>
cudaError_t launch_bf16(const GroupedGemmArgs& a, cudaStream_t st) {
    using C = Tile<GEMM>;
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(grouped_gemm_bf16_kernel<GEMM>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    });
    if (attr_err != cudaSuccess) return attr_err;

    uint64_t b_rows;
    const KParams p = make_params(a, GEMM, &b_rows);
    const int E = a.E, S = a.S;
    CUtensorMap tmAr, tmAs, tmB;
    if (!make_tmap_bf16(&tmAr, a.w_routed, (uint64_t)E * p.a_rows_per_mat, p.K, BM))
        return cudaErrorInvalidValue;
    if (!make_tmap_bf16(&tmAs, S > 0 ? a.w_shared : a.w_routed,
                        (uint64_t)(S > 0 ? S : E) * p.a_rows_per_mat, p.K, BM))
        return cudaErrorInvalidValue;
    if (b_rows == 0) return cudaSuccess;
    if (!make_tmap_bf16(&tmB, a.b_rows, b_rows, p.K, B_BOX)) return cudaErrorInvalidValue;
    const int grid = grid_for(p);
    grouped_gemm_bf16_kernel<GEMM><<<grid, 192, C::SMEM_BYTES, st>>>(tmAr, tmAs, tmB, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_grouped_gemm(const GroupedGemmArgs& a, cudaStream_t st) {
    if (a.wfmt == MOE_W_FP4_E2M1_UE8M0_B32 || a.wfmt == MOE_W_MXFP4) {
        if (a.afmt == MOE_A_MXFP8)
            return a.gemm == 1 ? launch_mx<1, MOE_A_MXFP8>(a, st) : launch_mx<2, MOE_A_MXFP8>(a, st);
        if (a.afmt == MOE_A_FP8_E4M3_POW2_B128)
            return a.gemm == 1 ? launch_mx<1, MOE_A_FP8_E4M3_POW2_B128>(a, st)
                               : launch_mx<2, MOE_A_FP8_E4M3_POW2_B128>(a, st);
        return cudaErrorNotSupported;
    }
    if (a.afmt != MOE_A_BF16) return cudaErrorNotSupported;
    if (a.wfmt == MOE_W_BF16) return a.gemm == 1 ? launch_bf16<1>(a, st) : launch_bf16<2>(a, st);
    if (a.wfmt == MOE_W_FP8_E4M3_B128x128)
        return a.gemm == 1 ? launch_fp8w<1>(a, st) : launch_fp8w<2>(a, st);
    return cudaErrorNotSupported;
}

}  // namespace moe
