// gemm_bf16.cu -- per-expert SwiGLU MLP on the tcgen05 tensor cores, bf16 weights.
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
//            token tiles into a ring of shared-memory stages. Token tiles come
//            as 16-row boxes when experts hold a few tokens each (decode: one
//            box per tile), or, for launches of many tokens per expert (the
//            shared experts of the NVFP4 layer alone), as one box per set bit of
//            the tile's 16-row count (16 to 128 rows). Measured: the large boxes
//            took the decode down projection from 0.74 to 0.83 ms and the NVFP4
//            layer's bf16 shared-expert launches from ~0.53 to ~0.46 ms;
//   warp 1   MMA issuer: tcgen05.mma kind::f16 (bf16 x bf16 -> fp32 in TMEM),
//            tcgen05.commit frees each stage and publishes each accumulator;
//   warps 2-5 epilogue: tcgen05.ld the accumulator (lane = weight row,
//            column = token), SwiGLU (GEMM1), bf16 stores.
// Accumulators are double-buffered in tensor memory so the epilogue of one
// tile overlaps the main loop of the next. The tile list (expert, M tile,
// N tile) is derived on the device from expert_offsets; there is no host sync.
#include <type_traits>

#include "gemm_common.cuh"

namespace moe {
namespace gemm {
namespace {

// token-tile maps: four box heights (wide) or the 16-row box alone
template <bool WIDE_B>
using BParam = typename std::conditional<WIDE_B, BMaps, CUtensorMap>::type;

template <int GEMM, bool WIDE_B, int NA>
__global__ void __launch_bounds__(192, 1)
    grouped_gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA_routed,
                             const __grid_constant__ CUtensorMap tmA_shared,
                             const __grid_constant__ BParam<WIDE_B> tmB, const KParams p) {
    pdl_wait();
    pdl_trigger();
    using C = Tile<GEMM, NA>;
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
        if constexpr (WIDE_B) prefetch_bmaps(tmB);
        else tma_prefetch_desc(&tmB);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    // tile schedule: pref[s] = first unit of segment s
    const int MT = p.M / p.tile_rows;
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
                    if (C::NA == 2)  // gate/up: the up tile; down: the next 128-row block
                        tma_load_2d(st + C::A_BYTES, tmA, kb * BK, t.a_row + p.a_up_offset, &full[stage]);
                    uint8_t* sb = st + C::NA * C::A_BYTES;
                    if constexpr (WIDE_B) {
                        load_b_rows(sb, tmB, kb * BK, t.b_row, n_mma, BK * 2, &full[stage]);
                    } else {
                        for (int i = 0; i < nb; ++i)
                            tma_load_2d(sb + i * B_BOX * BK * 2, &tmB, kb * BK, t.b_row + i * B_BOX,
                                        &full[stage]);
                    }
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
                        if (C::NA == 2)
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
        epilogue_loop<GEMM, C::ACC_COLS, 2, (GEMM == 2 ? NA : 1)>(p, pref, total, tmem_base, tfull,
                                                                  tempty, abort_flag, warp, lane);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}


}  // namespace

template <int GEMM, bool WIDE_B, int NA>
cudaError_t launch_bf16(const GroupedGemmArgs& a, cudaStream_t st) {
    using C = Tile<GEMM, NA>;
    const cudaError_t attr_err = ensure_smem_limit(
        reinterpret_cast<const void*>(grouped_gemm_bf16_kernel<GEMM, WIDE_B, NA>), C::SMEM_BYTES);
    if (attr_err != cudaSuccess) return attr_err;

    uint64_t b_rows;
    KParams p = make_params(a, GEMM, &b_rows);
    if (GEMM == 2 && NA == 2) {  // two consecutive 128-row blocks of W2 per unit
        if (p.M % (2 * BM)) return cudaErrorInvalidValue;
        p.tile_rows = 2 * BM;
        p.a_up_offset = BM;
    }
    const int E = a.E, S = a.S;
    CUtensorMap tmAr, tmAs;
    BParam<WIDE_B> tmB;
    if (!make_tmap_bf16(&tmAs, S > 0 ? a.w_shared : a.w_routed,
                        (uint64_t)(S > 0 ? S : E) * p.a_rows_per_mat, p.K, BM))
        return cudaErrorInvalidValue;
    // a launch of shared experts alone (E == 0) never reads the routed map
    if (E == 0) tmAr = tmAs;
    else if (!make_tmap_bf16(&tmAr, a.w_routed, (uint64_t)E * p.a_rows_per_mat, p.K, BM))
        return cudaErrorInvalidValue;
    if (b_rows == 0) return cudaSuccess;
    if constexpr (WIDE_B) {
        if (!make_bmaps(&tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.b_rows, b_rows, p.K, BK))
            return cudaErrorInvalidValue;
    } else {
        if (!make_tmap_bf16(&tmB, a.b_rows, b_rows, p.K, B_BOX)) return cudaErrorInvalidValue;
    }
    const int grid = grid_for(p);
    launch_pdl(grouped_gemm_bf16_kernel<GEMM, WIDE_B, NA>, grid, 192, C::SMEM_BYTES, st, tmAr, tmAs, tmB, p);
    return cudaGetLastError();
}

cudaError_t launch_gemm_bf16(const GroupedGemmArgs& a, cudaStream_t st) {
    // wide token boxes for many tokens per expert (at least 64 on average)
    const bool wide = (long)(a.N + (long)a.S * a.T) >= 64L * (a.E + a.S);
    if (a.gemm == 1) return wide ? launch_bf16<1, true, 2>(a, st) : launch_bf16<1, false, 2>(a, st);
    // down: two 128-row blocks of W2 per unit (twice the weight bytes per stage and
    // half the units) when H allows it
    if (a.H % (2 * BM) == 0)
        return wide ? launch_bf16<2, true, 2>(a, st) : launch_bf16<2, false, 2>(a, st);
    return wide ? launch_bf16<2, true, 1>(a, st) : launch_bf16<2, false, 1>(a, st);
}

}  // namespace gemm
}  // namespace moe
