// gemm_mx_pair.cu -- the block-scaled (E2M1 x E4M3) down projection on CTA
// pairs: tcgen05.mma.cta_group::2 with M = 256 weight rows (output features)
// spread over the two SMs of a cluster, each SM loading its own 128 weight rows
// and half of the 224-token tile. Against the one-SM kernel (gemm_mx.cu) each
// SM fetches half the token rows per weight row, the larger share of a down
// stage's copies (K = 1024 leaves little else per unit). Measured on the
// 896-expert layer: down projection 3.48 -> 3.24 ms. (The same pairing of the
// gate/up GEMM measured 4.19 -> 4.42 ms: its two accumulators leave no room
// to double-buffer, and each stage waits on both SMs; it stays on one SM.)
//
// Arithmetic as in gemm_mx.cu ("DeepSeek-V4-Pro 架构与代码概述", 架构: FP4
// experts with UE8M0 scales; "开源巨头开放2.8T MoE权重:架构创新与本地部署实践指南",
// 存储与量化策略: MXFP4 weights, MXFP8 activations): kind::mxf8f6f4 applies one
// E8M0 scale per 32 elements of K to every row of A and of B.
//
// Pair protocol (rank 0 leads; every wait is bounded as in the other kernels):
//  - Each SM's TMA loads its 128 weight rows and its half of the token rows
//    with .cta_group::2, completing on the leader's full barrier; the leader's
//    expect-tx arrival covers both SMs' bytes (the peer only copies).
//  - Each SM's four scale warps store its own weight rows' scales and the whole
//    token tile's scales (duplicated) into its own tensor memory, then arrive
//    on the leader's sf_ready barrier.
//  - The leader's MMA thread issues the pair MMAs and commits to the empty and
//    tfull barriers of both SMs (multicast commit).
//  - Each SM's epilogue drains its own 128 rows of the accumulator (double
//    buffered) and arrives on the leader's tempty barrier.
//  - Tensor memory is allocated and freed by warp 0 of both SMs with
//    .cta_group::2; a cluster barrier brackets the kernel so that neither SM
//    leaves while the other may still touch its barriers or tensor memory.
// No load uses .multicast::cluster: each SM loads its own rows.
#include "gemm_common.cuh"

namespace moe {
namespace gemm {
namespace {

constexpr int P_BK = 128;      // K elements per stage (one 128-byte smem row)
constexpr int P_SF_KB = 32;    // k-blocks of 32 per scale box row (eight stages)
constexpr int P_SF_STAGES = P_SF_KB / 4;
constexpr int P_SF_TILE = 128 * P_SF_KB;

// One accumulator per SM (its 128 output features x the pair's 224 tokens),
// double-buffered; BNX tokens per pair tile, BNX / 2 rows of it in each SM.
struct TileP {
    static constexpr int BNX = 224;
    static constexpr int BHALF = BNX / 2;
    static constexpr int ACCB = 2;
    static constexpr int SCALE_WARP = 6;  // warps: 0 TMA, 1 MMA, 2-5 and 10-13 epilogue, 6-9 scales
    static constexpr int EPI_WARPS = 8;   // two groups of four, alternate 16-token chunks
    static constexpr int THREADS = 32 * 14;
    static constexpr int EPI_BYTES = EPI_WARPS * 2 * 16 * 32 * 2 + 128;  // per warp two [16][32] bf16 chunks
    static constexpr int SFB_ROWS = (BNX + 127) / 128 * 128;
    static constexpr int SFB_ATOMS = SFB_ROWS / 128;
    static constexpr int NOPS = 1 + SFB_ATOMS;  // scale operands: the weight rows, the token rows
    static constexpr int A_BYTES = BM * P_BK;
    static constexpr int B_BYTES = BHALF * P_BK;
    static constexpr int A_OFF = 0;
    static constexpr int B_OFF = A_BYTES;
    static constexpr int RAW_BYTES = NOPS * P_SF_TILE;
    static constexpr int RING_BYTES = 2 * RAW_BYTES;
    static constexpr int NBARS = 3 * 6 + 13;
    static constexpr int FIXED_BYTES = 1024 + 8 * NBARS + 16 + 4 * (MAX_SEG + 1) + EPI_BYTES;
    static constexpr int STAGE_BYTES = (B_OFF + B_BYTES + 1023) / 1024 * 1024;
    static constexpr int STAGES = stages_for(STAGE_BYTES, FIXED_BYTES + RING_BYTES, 6);
    static constexpr int ACC_COLS = BNX;
    static constexpr int TMEM_COLS = 512;
    static constexpr int SF_COL = ACCB * ACC_COLS;
    static constexpr int SET_COLS = 4 * NOPS;
    static constexpr int NSETS_FIT = (TMEM_COLS - SF_COL) / SET_COLS;
    static constexpr int NSETS = NSETS_FIT < STAGES ? NSETS_FIT : STAGES;
    static_assert(NSETS >= 2, "tensor memory budget: two scale sets");
    static constexpr int BAR_BYTES = 8 * (3 * STAGES + 13) + 16;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + RING_BYTES + BAR_BYTES +
                                      4 * (MAX_SEG + 1) + EPI_BYTES;
    static_assert(STAGES >= 3 && SMEM_BYTES <= 232448, "shared memory budget");
    static_assert(BHALF % 16 == 0, "half tiles of whole 16-row boxes");
};

// ------------------------------------------------------------ pair helpers
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Address in the shared::cluster window of the same variable in CTA `rank`.
__device__ __forceinline__ uint32_t peer_addr(const void* p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
    return r;
}

__device__ __forceinline__ void cluster_barrier() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}

// Arrival on a barrier of the other SM. Relaxed: the arriving warps signal that
// their tcgen05 stores completed (scale warps, after tcgen05.wait::st) or that
// their tensor-memory reads are done (epilogue), both ordered by
// tcgen05.fence::before_thread_sync; the waiter reads no generic memory they
// wrote. (Release semantics made every arrival a cluster-wide memory fence,
// which held the pair's stages back.)
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
                 : "memory");
}

// Tiled load into this SM's shared memory, completing on the leader's barrier.
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const void* tmap, int32_t x,
                                                 int32_t y, uint32_t leader_bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(leader_bar)
        : "memory");
}

__device__ __forceinline__ void load_b_rows_pair(uint8_t* dst, const BMaps& bm, int x, int row, int n,
                                                 int row_bytes, uint32_t leader_bar) {
    const int blocks = n >> 4;
    int off = 0;
#pragma unroll
    for (int i = B_HEIGHTS - 1; i >= 0; --i) {
        if ((blocks >> i) & 1) {
            tma_load_2d_pair(dst + off * row_bytes, &bm.m[i], x, row + off, leader_bar);
            off += 16 << i;
        }
    }
}

__device__ __forceinline__ void mma_mx_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem),
        "r"(sfb_tmem)
        : "memory");
}

// Arrive on `bar` (the same offset) in both SMs of the pair once this
// thread's tcgen05 operations have completed.
__device__ __forceinline__ void mma_commit_pair(uint64_t* bar) {
    const uint16_t mask = 3;
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(smem_u32(bar)),
        "h"(mask)
        : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* smem_slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(smem_slot)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ uint32_t word_of_p(const uint4& u, int w) {
    return w == 0 ? u.x : (w == 1 ? u.y : (w == 2 ? u.z : u.w));
}

__device__ __forceinline__ bool warp_wait_p(uint64_t* bar, uint32_t parity, volatile int* abort, int lane) {
    int ok = 1;
    if (lane == 0) ok = mbar_wait(bar, parity, abort) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}

__global__ void __launch_bounds__(TileP::THREADS, 1)
    grouped_gemm_mx_pair_down_kernel(const __grid_constant__ CUtensorMap tmA_routed,
                                const __grid_constant__ CUtensorMap tmA_shared,
                                const __grid_constant__ CUtensorMap tmSFA_routed,
                                const __grid_constant__ CUtensorMap tmSFA_shared,
                                const __grid_constant__ BMaps tmB,
                                const __grid_constant__ CUtensorMap tmSFB, const KParams p) {
    pdl_wait();
    pdl_trigger();
    using C = TileP;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* sf_ring = smem + C::STAGES * C::STAGE_BYTES;
    uint64_t* full = reinterpret_cast<uint64_t*>(sf_ring + C::RING_BYTES);
    uint64_t* empty = full + C::STAGES;
    uint64_t* sf_ready = empty + C::STAGES;
    uint64_t* tfull = sf_ready + C::STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* mma_done = tempty + 2;
    uint64_t* sf_full = mma_done + 1;
    uint64_t* sf_empty = sf_full + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sf_empty + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* pref = reinterpret_cast<int*>(tmem_slot + 4);
    __nv_bfloat16* ep_buf = reinterpret_cast<__nv_bfloat16*>(
        (reinterpret_cast<uintptr_t>(pref + MAX_SEG + 1) + 127) & ~static_cast<uintptr_t>(127));

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();  // 0 leads the pair
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);          // the leader's expect-tx arrival covers both SMs' copies
            mbar_init(&empty[s], 1);         // the leader's multicast commit
            mbar_init(&sf_ready[s], 8);      // four scale warps per SM (leader's copy used)
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 2 * 32 * C::EPI_WARPS);  // both SMs' epilogues (leader's copy used)
        }
        mbar_init(mma_done, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sf_full[i], 1);
            mbar_init(&sf_empty[i], 4);
        }
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmA_routed);
        tma_prefetch_desc(&tmA_shared);
        tma_prefetch_desc(&tmSFA_routed);
        tma_prefetch_desc(&tmSFA_shared);
        prefetch_bmaps(tmB);
        tma_prefetch_desc(&tmSFB);
    }
    if (warp == 0) {
        tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
        tmem_relinquish_pair();
    }
    const int MT = p.M / p.tile_rows;
    if (warp == 1) build_schedule(p, pref, MT, lane);
    tc_fence_before();
    __syncthreads();
    cluster_barrier();  // both SMs' barriers are initialised before any remote arrival
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int total = pref[p.nseg];
    const int KB = p.K / P_BK;

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            int sfs = 0, sf_issued = 0;
            uint32_t sf_phase = 0;
            for (int u = pair; u < total && !*abort_flag; u += npairs) {
                const Unit t = decode_unit(p, pref, u);
                const int n_mma = (t.n_valid + 31) & ~31;  // pair MMA N: two 16-row halves
                const int n_half = n_mma >> 1;
                // padded E2M1 tiles count their packed size toward the transaction;
                // the leader expects both SMs' bytes
                const uint32_t tx = 2 * (C::A_BYTES / 2 + n_half * P_BK);
                const bool routed = t.seg < p.E;
                const CUtensorMap* tmA = routed ? &tmA_routed : &tmA_shared;
                const CUtensorMap* tmSFA = routed ? &tmSFA_routed : &tmSFA_shared;
                const int a_row = t.a_row + (int)rank * BM;  // this SM's 128 rows of the 256
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb) {
                    if (kb % P_SF_STAGES == 0) {  // this SM's A scales and all token scales
                        if (!mbar_wait(&sf_empty[sfs], sf_phase ^ 1, abort_flag)) { ok = false; break; }
                        uint8_t* sl = sf_ring + sfs * C::RAW_BYTES;
                        const int sfx = kb * 4;
                        mbar_arrive_expect_tx(&sf_full[sfs], C::RAW_BYTES);
                        tma_load_2d(sl, tmSFA, sfx, a_row, &sf_full[sfs]);
                        tma_load_2d(sl + P_SF_TILE, &tmSFB, sfx, t.b_row, &sf_full[sfs]);
                        ++sf_issued;
                        if (++sfs == 2) { sfs = 0; sf_phase ^= 1; }
                    }
                    if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
                    uint8_t* st = smem + stage * C::STAGE_BYTES;
                    const uint32_t lfull = peer_addr(&full[stage], 0);
                    if (rank == 0) mbar_arrive_expect_tx(&full[stage], tx);
                    tma_load_2d_pair(st + C::A_OFF, tmA, kb * P_BK, a_row, lfull);
                    load_b_rows_pair(st + C::B_OFF, tmB, kb * P_BK, t.b_row + (int)rank * n_half,
                                     n_half, P_BK, lfull);
                    ++issued;
                    if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
            }
            if (*abort_flag) {
                // this SM's scale copies complete on its own barriers; the tile
                // copies complete on the leader's, which the leader drains
                volatile int no_abort = 0;
                int s = sfs;
                uint32_t ph = sf_phase;
                for (int i = 0; i < min(sf_issued, 2); ++i) {
                    if (--s < 0) { s = 1; ph ^= 1; }
                    mbar_wait(&sf_full[s], ph, &no_abort);
                }
                if (rank == 0) {
                    s = stage;
                    ph = phase;
                    for (int i = 0; i < min(issued, C::STAGES); ++i) {
                        if (--s < 0) { s = C::STAGES - 1; ph ^= 1; }
                        mbar_wait(&full[s], ph, &no_abort);
                    }
                }
                status_or(p.status, MOE_DEV_TIMEOUT);
            }
        }
    } else if (warp == 1) {
        // the leader's MMA thread issues the pair MMAs
        if (lane == 0 && rank == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int set = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            for (int u = pair; u < total; u += npairs) {
                const Unit t = decode_unit(p, pref, u);
                const int n_mma = (t.n_valid + 31) & ~31;
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1, abort_flag)) break;
                tc_fence_after();
                const uint32_t d0 = tmem_base + acc * C::ACC_COLS;
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&full[stage], phase, abort_flag) ||
                        !mbar_wait(&sf_ready[stage], phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t st = smem_u32(smem + stage * C::STAGE_BYTES);
                    const uint32_t sfs = tmem_base + C::SF_COL + set * C::SET_COLS;
                    const uint32_t sfa = sfs;
                    const uint32_t sfb = sfs + 4;
#pragma unroll
                    for (int kk = 0; kk < P_BK / 32; ++kk) {
                        const uint32_t acc_flag = (kb | kk) != 0;
                        const uint32_t idesc = idesc_mx_e2m1_e4m3(2 * BM, n_mma, kk, kk);
                        const uint32_t sub = (uint32_t)kk << 30;
                        mma_mx_pair(d0, sdesc_kmajor_sw128(st + C::A_OFF + kk * 32),
                                    sdesc_kmajor_sw128(st + C::B_OFF + kk * 32), idesc, sfa | sub,
                                    sfb | sub, acc_flag);
                    }
                    mma_commit_pair(&empty[stage]);
                    if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
                    if (++set == C::NSETS) set = 0;
                }
                if (!ok) break;
                mma_commit_pair(&tfull[acc]);
                if (++acc == C::ACCB) { acc = 0; acc_phase ^= 1; }
            }
            mma_commit(mma_done);
            volatile int no_abort = 0;
            mbar_wait(mma_done, 0, &no_abort);
            if (*abort_flag) status_or(p.status, MOE_DEV_TIMEOUT);
        }
    } else if (warp >= C::SCALE_WARP && warp < C::SCALE_WARP + 4) {
        // scale warps: as in gemm_mx.cu (this SM's A rows, all token rows, 32-byte
        // swizzled boxes), arriving on the leader's sf_ready
        const uint32_t lane_cols = tmem_base + ((uint32_t)((warp & 3) * 32) << 16) + C::SF_COL;
        uint4 cache[C::NOPS][4];
        int stage = 0;
        int set = 0;
        int g = 0;
        int sfs = 0;
        uint32_t sf_phase = 0;
        bool ok = true;
        for (int u = pair; u < total && ok; u += npairs) {
            for (int kb = 0; kb < KB; ++kb) {
                if (kb % P_SF_STAGES == 0 && !warp_wait_p(&sf_full[sfs], sf_phase, abort_flag, lane)) {
                    ok = false;
                    break;
                }
                if (g >= C::NSETS) {
                    const int gp = g - C::NSETS;
                    if (!warp_wait_p(&empty[gp % C::STAGES], (uint32_t)(gp / C::STAGES) & 1u, abort_flag,
                                     lane)) {
                        ok = false;
                        break;
                    }
                }
                if ((kb & 3) == 0) {
                    const uint8_t* raw = sf_ring + sfs * C::RAW_BYTES;
                    const int sf_swz = 16 * (((kb % P_SF_STAGES) >> 2) ^ ((lane >> 2) & 1));
#pragma unroll
                    for (int i = 0; i < C::NOPS; ++i)
#pragma unroll
                        for (int r = 0; r < 4; ++r)
                            cache[i][r] = *reinterpret_cast<const uint4*>(
                                raw + i * P_SF_TILE + P_SF_KB * (lane + 32 * r) + sf_swz);
                    if (kb % P_SF_STAGES == P_SF_STAGES - 4 || kb + 4 >= KB) {
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&sf_empty[sfs]);
                        if (++sfs == 2) { sfs = 0; sf_phase ^= 1; }
                    }
                }
                const int w = kb & 3;
                uint4 v[C::NOPS];
#pragma unroll
                for (int i = 0; i < C::NOPS; ++i)
                    v[i] = make_uint4(word_of_p(cache[i][0], w), word_of_p(cache[i][1], w),
                                      word_of_p(cache[i][2], w), word_of_p(cache[i][3], w));
#pragma unroll
                for (int i = 0; i < C::NOPS; ++i) tmem_st4(lane_cols + set * C::SET_COLS + 4 * i, v[i]);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (rank == 0) mbar_arrive(&sf_ready[stage]);
                    else mbar_arrive_remote(peer_addr(&sf_ready[stage], 0));
                }
                if (++stage == C::STAGES) stage = 0;
                if (++set == C::NSETS) set = 0;
                ++g;
            }
        }
    } else if ((warp >= 2 && warp < 6) || warp >= 10) {
        // this SM's 128 output features of the pair's 256, bf16. Group grp (warps
        // 2-5 or 10-13) takes the 16-token chunks grp, grp + 2, ...; per chunk each
        // warp converts its 32 features into its own shared [16 tokens][32] tile
        // (two, alternating) and writes each token row's 64 bytes of them as four
        // 16-byte pieces, two per lane; no barrier between warps.
        const int q = warp & 3;
        const int grp = warp >= 10 ? 1 : 0;
        __nv_bfloat16* wbuf = ep_buf + (warp < 6 ? warp - 2 : warp - 6) * 2 * 16 * 32;
        int acc = 0;
        uint32_t acc_phase = 0;
        int chunk = 0;
        for (int u = pair; u < total; u += npairs) {
            const Unit t = decode_unit(p, pref, u);
            if (!mbar_wait(&tfull[acc], acc_phase, abort_flag)) break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * C::ACC_COLS;
            __nv_bfloat16* out =
                reinterpret_cast<__nv_bfloat16*>(t.out) + t.mt * p.tile_rows + (int)rank * BM + q * 32;
            for (int c0 = 16 * grp; c0 < t.n_valid; c0 += 32, ++chunk) {
                uint32_t gq[16];
                tmem_ld16(taddr + c0, gq);
                tmem_ld_wait(gq);
                __nv_bfloat16* buf = wbuf + (chunk & 1) * 16 * 32;
#pragma unroll
                for (int j = 0; j < 16; ++j) buf[j * 32 + lane] = __float2bfloat16_rn(__uint_as_float(gq[j]));
                __syncwarp();
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int i = lane + 32 * h;  // 16 token rows x 4 pieces of 8 features
                    const int r = i >> 2, pc = i & 3;
                    if (c0 + r < t.n_valid)
                        *reinterpret_cast<uint4*>(out + (size_t)(c0 + r) * p.ld_out + pc * 8) =
                            *reinterpret_cast<const uint4*>(buf + r * 32 + pc * 8);
                }
            }
            tc_fence_before();
            if (rank == 0) mbar_arrive(&tempty[acc]);
            else mbar_arrive_remote(peer_addr(&tempty[acc], 0));
            if (++acc == C::ACCB) { acc = 0; acc_phase ^= 1; }
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_barrier();  // neither SM leaves while the pair may still use its memory
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    }
}

// Cluster launch (two CTAs per cluster) with programmatic stream serialization.
template <typename... KArgs, typename... Args>
cudaError_t launch_pair(void (*kernel)(KArgs...), int pairs, int threads, size_t smem, cudaStream_t st,
                        Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

}  // namespace

cudaError_t launch_gemm_mx_pair_down(const GroupedGemmArgs& a, cudaStream_t st) {
    using C = TileP;
    auto kernel = grouped_gemm_mx_pair_down_kernel;
    const cudaError_t attr_err = ensure_smem_limit(reinterpret_cast<const void*>(kernel), C::SMEM_BYTES);
    if (attr_err != cudaSuccess) return attr_err;
    uint64_t b_rows;
    KParams p = make_params(a, 2, &b_rows);
    p.bn = C::BNX;
    p.tile_rows = 2 * BM;  // 256 output features per pair unit
    if (p.M % p.tile_rows) return cudaErrorInvalidValue;
    const int S = a.S;
    const uint64_t K = p.K, rowsA = (uint64_t)a.E * p.a_rows_per_mat;
    const uint64_t rowsAs = (uint64_t)(S > 0 ? S : a.E) * p.a_rows_per_mat;
    const void* wA = a.w_routed;
    const void* wAs = S > 0 ? a.w_shared : a.w_routed;
    const void* sA = a.w_routed_scale;
    const void* sAs = S > 0 ? a.w_shared_scale : a.w_routed_scale;
    CUtensorMap tmA, tmAs, tmSFA, tmSFAs, tmSFB;
    BMaps tmB;
    if (!make_tmap_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, wA, rowsA, K, K / 2, P_BK, BM,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_2d(&tmAs, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, wAs, rowsAs, K, K / 2, P_BK, BM,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_2d(&tmSFA, CU_TENSOR_MAP_DATA_TYPE_UINT8, sA, rowsA, K / 32, K / 32, P_SF_KB, 128,
                      CU_TENSOR_MAP_SWIZZLE_32B) ||
        !make_tmap_2d(&tmSFAs, CU_TENSOR_MAP_DATA_TYPE_UINT8, sAs, rowsAs, K / 32, K / 32, P_SF_KB, 128,
                      CU_TENSOR_MAP_SWIZZLE_32B))
        return cudaErrorInvalidValue;
    if (b_rows == 0) return cudaSuccess;
    if (!make_bmaps(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.b_rows, b_rows, K, P_BK) ||
        !make_tmap_2d(&tmSFB, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.b_scale, b_rows, K / 32, K / 32, P_SF_KB,
                      C::SFB_ROWS, CU_TENSOR_MAP_SWIZZLE_32B))
        return cudaErrorInvalidValue;
    const int pairs = std::max(1, grid_for(p) / 2);
    launch_pair(kernel, pairs, C::THREADS, C::SMEM_BYTES, st, tmA, tmAs, tmSFA, tmSFAs, tmB, tmSFB, p);
    return cudaGetLastError();
}

}  // namespace gemm
}  // namespace moe
