// gemm_mx.cu -- per-expert SwiGLU MLP with E2M1 weights and E4M3 activations,
// both block-scaled per 32 elements, on tcgen05 kind::mxf8f6f4. The expert
// structure and tile schedule are those of gemm_bf16.cu.
#include "gemm_common.cuh"

namespace moe {
namespace gemm {
namespace {

// ---------------------------------------------------------------- block-scaled
// E2M1 weights with one E8M0 scale per 32 elements ("DeepSeek-V4-Pro 架构与代码概述",
// 架构: FP4 experts with UE8M0 scales, kernel.py fp4_quant_kernel block 32;
// "开源巨头开放2.8T MoE权重:架构创新与本地部署实践指南", 存储与量化策略: MXFP4 weights)
// times E4M3 activations with one E8M0 scale per 32 elements (MXFP8, or the
// per-128 power-of-two activation scale repeated over its four 32-blocks).
// tcgen05.mma kind::mxf8f6f4 applies both scales inside the MMA, so the FP4
// weights are never dequantised in software: TMA expands each packed row of
// 128 E2M1 values to the one-byte-per-value layout the MMA reads
// (16U4_ALIGN16B). Scales travel by TMA as 128 rows x 32 bytes (32 k-blocks,
// 32-byte swizzle) into a two-slot ring. The MMA reads row m's scale (m = m0 + 32*m1) from
// TMEM lane m0 of every lane quadrant, column m1, one k-block per byte. Four
// scale warps, one per lane quadrant, store each stage's 4 k-blocks in that
// order (tcgen05.st) into a ring of TMEM column sets: a tcgen05.cp issued by
// the MMA thread costs the tensor pipe about as much as two small MMAs, a
// store from another warp next to nothing.
// The TMA unit keeps a bounded number of row requests in flight, and a row
// fetched from HBM holds its slot for the whole DRAM latency whatever its
// width: the scale boxes are therefore 32 bytes (eight stages) wide, so that
// the narrow scale rows take as few of those slots as the ring allows.
// A unit's NA weight tiles (gate and up for GEMM1; two consecutive 128-row
// blocks of the down projection when NA = 2) share its token tile, and each
// has its own MMA-issuing thread and accumulator: one thread issuing small
// block-scaled MMAs with per-stage commits sustains ~72 cycles per MMA, two
// threads ~48 at 64 tokens and the full rate from 112 tokens.
// GEMM1's epilogue quantises the SwiGLU output per 32 (MXFP8) or per 128
// (power of two) along I, exactly as the activation quantiser does.
constexpr int MX_BK = 128;        // K elements per stage (one 128-byte smem row)
constexpr int SF_KB = 32;         // k-blocks of 32 per scale box row (8 stages)
constexpr int SF_STAGES = SF_KB / 4;
constexpr int SF_TILE = 128 * SF_KB;  // scale tile: 128 rows x 32 k-blocks

// GEMM: 1 gate/up, 2 down. NA: weight tiles per unit (= MMA threads). BNX_:
// tokens per tile. ACCB: accumulator buffers in tensor memory (2 overlaps a
// tile's epilogue with the next tile's main loop; 1 lets gate/up use
// 224-token tiles). Warps: 0 TMA, 1 MMA (tile 0), then EG groups of 4
// epilogue warps (one per TMEM lane quadrant), then the 4 scale warps, then
// the MMA warp of tile 1. Wide tiles take two epilogue groups on alternating
// 16-token chunks (the single-buffered gate/up drain is not overlapped with
// the next tile's main loop).
template <int GEMM, int NA_, int BNX_, int ACCB_>
struct TileMX {
    static constexpr int NA = NA_;
    // epilogue groups: two for the wide tiles (single-buffered gate/up, double-buffered down)
    static constexpr int EG = (ACCB_ == 1 || BNX_ > 128) ? 2 : 1;
    static constexpr int SCALE_WARP = 2 + 4 * EG;     // first of the 4 scale warps
    static constexpr int MMA2_WARP = SCALE_WARP + 4;  // MMA thread of tile 1 (NA == 2)
    static constexpr int THREADS = 32 * (MMA2_WARP + (NA == 2 ? 1 : 0));
    static constexpr int RED_BYTES = EG * 2 * 4 * 16 * 4;  // [group][parity][warp][16 columns]
    // staged epilogue chunks, per group and parity: down [16 tokens][128] bf16;
    // gate/up [16][128] E4M3 bytes, then [16][4] E8M0 codes
    static constexpr int G1_STAGE = 16 * BM + 16 * 4;
    static constexpr int EPI_BYTES = (GEMM == 2 ? EG * 2 * 16 * BM * 2 : EG * 2 * G1_STAGE) + 128;
    static constexpr int BNX = BNX_;
    static constexpr int ACCB = ACCB_;
    static constexpr int SFB_ROWS = (BNX + 127) / 128 * 128;  // token rows of the scale tile
    static constexpr int SFB_ATOMS = SFB_ROWS / 128;
    static constexpr int NOPS = NA + SFB_ATOMS;  // scale operands: A tiles, B rows 0-127, [128-255]
    static constexpr int A_BYTES = BM * MX_BK;   // one byte per E2M1 value in smem
    static constexpr int B_BYTES = BNX * MX_BK;
    static constexpr int A_OFF = 0;
    static constexpr int B_OFF = NA * A_BYTES;
    static constexpr int RAW_BYTES = NOPS * SF_TILE;  // one scale ring slot: operand i at i*SF_TILE
    static constexpr int RING_BYTES = 2 * RAW_BYTES;
    static constexpr int FIXED_BYTES =
        1024 + 8 * (3 * 6 + 9 + 4 * EG) + 16 + 4 * (MAX_SEG + 1) + RED_BYTES + EPI_BYTES;
    static constexpr int STAGE_BYTES = (B_OFF + B_BYTES + 1023) / 1024 * 1024;
    static constexpr int STAGES = stages_for(STAGE_BYTES, FIXED_BYTES + RING_BYTES, 6);
    static constexpr int ACC_COLS = NA * BNX;
    static constexpr int TMEM_COLS = 512;
    static constexpr int SF_COL = ACCB * ACC_COLS;  // scale sets: set s, operand i at SF_COL + s*SET_COLS + 4*i
    static constexpr int SET_COLS = 4 * NOPS;
    static constexpr int NSETS_FIT = (TMEM_COLS - SF_COL) / SET_COLS;
    static constexpr int NSETS = NSETS_FIT < STAGES ? NSETS_FIT : STAGES;
    static_assert(NSETS >= 2, "tensor memory budget: two scale sets");
    static constexpr int BAR_BYTES = 8 * (3 * STAGES + 9 + 4 * EG) + 16;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + RING_BYTES + BAR_BYTES +
                                      4 * (MAX_SEG + 1) + RED_BYTES + EPI_BYTES;
    static_assert(STAGES >= 2 && SMEM_BYTES <= 232448, "shared memory budget");
    static_assert(NA == 1 || NA == 2, "one or two weight tiles per unit");
    static_assert(GEMM == 2 || NA == 2, "gate/up units hold both projections");
};

// Max over the warp of non-negative floats: their bit patterns order like the
// values, so one integer max reduction does it.
__device__ __forceinline__ float warp_max_nonneg(float v) {
    return __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(v)));
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

// Two floats to E4M3 (saturating, nearest-even) in one conversion: byte 0 = a,
// byte 1 = b (the instruction puts its first source in the upper byte).
__device__ __forceinline__ uint32_t e4m3x2_sat(float a, float b) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(b), "f"(a));
    return r;
}

// Word w (0..3) of a 16-byte vector.
__device__ __forceinline__ uint32_t word_of(const uint4& u, int w) {
    return w == 0 ? u.x : (w == 1 ? u.y : (w == 2 ? u.z : u.w));
}

// Wait by lane 0 only, the outcome shared with the warp.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int lane) {
    int ok = 1;
    if (lane == 0) ok = mbar_wait(bar, parity, abort) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}


template <int GEMM, int AFMT, int NA_, int BNX_, int ACCB_>
__global__ void __launch_bounds__(TileMX<GEMM, NA_, BNX_, ACCB_>::THREADS, 1)
    grouped_gemm_mx_kernel(const __grid_constant__ CUtensorMap tmA_routed,
                           const __grid_constant__ CUtensorMap tmA_shared,
                           const __grid_constant__ CUtensorMap tmSFA_routed,
                           const __grid_constant__ CUtensorMap tmSFA_shared,
                           const __grid_constant__ BMaps tmB,
                           const __grid_constant__ CUtensorMap tmSFB, const KParams p) {
    pdl_wait();
    pdl_trigger();
    using C = TileMX<GEMM, NA_, BNX_, ACCB_>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* sf_ring = smem + C::STAGES * C::STAGE_BYTES;  // [2][RAW_BYTES]
    uint64_t* full = reinterpret_cast<uint64_t*>(sf_ring + C::RING_BYTES);
    uint64_t* empty = full + C::STAGES;
    uint64_t* sf_ready = empty + C::STAGES;  // the stage's scales are in their TMEM set
    uint64_t* tfull = sf_ready + C::STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* mma_done = tempty + 2;
    uint64_t* sf_full = mma_done + 1;  // [2] scale ring slots
    uint64_t* sf_empty = sf_full + 2;  // [2] released by the 4 scale warps
    uint64_t* red_bar = sf_empty + 2;  // [group][parity]: the amax exchange of a group's 4 warps
    uint64_t* ep_bar = red_bar + 2 * C::EG;  // [group][parity]: an epilogue group's staged chunk
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ep_bar + 2 * C::EG);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* pref = reinterpret_cast<int*>(tmem_slot + 4);
    float* red = reinterpret_cast<float*>(pref + MAX_SEG + 1);  // [group][parity][4 warps][16]
    __nv_bfloat16* ep_buf = reinterpret_cast<__nv_bfloat16*>(  // [group][2][16][128], 128-byte aligned
        (reinterpret_cast<uintptr_t>(red + C::RED_BYTES / 4) + 127) & ~static_cast<uintptr_t>(127));

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], C::NA);  // one commit per MMA thread
            mbar_init(&sf_ready[s], 4);   // one arrival per scale warp
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], C::NA);
            mbar_init(&tempty[a], 128 * C::EG);
        }
        mbar_init(mma_done, C::NA);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sf_full[i], 1);
            mbar_init(&sf_empty[i], 4);
        }
        for (int i = 0; i < 2 * C::EG; ++i) mbar_init(&red_bar[i], 4);
        for (int i = 0; i < 2 * C::EG; ++i) mbar_init(&ep_bar[i], 4);
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
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    const int MT = p.M / p.tile_rows;
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
            int sfs = 0, sf_issued = 0;  // scale ring slot and loads issued into the ring
            uint32_t sf_phase = 0;
            for (int u = blockIdx.x; u < total && !*abort_flag; u += gridDim.x) {
                const Unit t = decode_unit(p, pref, u);
                const int n_mma = (t.n_valid + 15) & ~15;
                // a padded E2M1 tile occupies A_BYTES of shared memory but the copy
                // counts its packed size (4 bits per value) toward the transaction
                const uint32_t tx = C::NA * (C::A_BYTES / 2) + n_mma * MX_BK;
                const bool routed = t.seg < p.E;
                const CUtensorMap* tmA = routed ? &tmA_routed : &tmA_shared;
                const CUtensorMap* tmSFA = routed ? &tmSFA_routed : &tmSFA_shared;
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb) {
                    if (kb % SF_STAGES == 0) {  // the scales of this stage and the next seven
                        if (!mbar_wait(&sf_empty[sfs], sf_phase ^ 1, abort_flag)) { ok = false; break; }
                        uint8_t* sl = sf_ring + sfs * C::RAW_BYTES;
                        const int sfx = kb * 4;  // first k-block of the box
                        mbar_arrive_expect_tx(&sf_full[sfs], C::RAW_BYTES);
#pragma unroll
                        for (int j = 0; j < C::NA; ++j)
                            tma_load_2d(sl + j * SF_TILE, tmSFA, sfx, t.a_row + j * p.a_up_offset,
                                        &sf_full[sfs]);
                        tma_load_2d(sl + C::NA * SF_TILE, &tmSFB, sfx, t.b_row, &sf_full[sfs]);
                        ++sf_issued;
                        if (++sfs == 2) { sfs = 0; sf_phase ^= 1; }
                    }
                    if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
                    uint8_t* st = smem + stage * C::STAGE_BYTES;
                    mbar_arrive_expect_tx(&full[stage], tx);
#pragma unroll
                    for (int j = 0; j < C::NA; ++j)
                        tma_load_2d(st + C::A_OFF + j * C::A_BYTES, tmA, kb * MX_BK,
                                    t.a_row + j * p.a_up_offset, &full[stage]);
                    load_b_rows(st + C::B_OFF, tmB, kb * MX_BK, t.b_row, n_mma, MX_BK, &full[stage]);
                    ++issued;
                    if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
            }
            if (*abort_flag) {
                // wait (bounded) for this thread's copies still in flight
                volatile int no_abort = 0;
                int s = stage;
                uint32_t ph = phase;
                for (int i = 0; i < min(issued, C::STAGES); ++i) {
                    if (--s < 0) { s = C::STAGES - 1; ph ^= 1; }
                    mbar_wait(&full[s], ph, &no_abort);
                }
                s = sfs;
                ph = sf_phase;
                for (int i = 0; i < min(sf_issued, 2); ++i) {
                    if (--s < 0) { s = 1; ph ^= 1; }
                    mbar_wait(&sf_full[s], ph, &no_abort);
                }
                status_or(p.status, MOE_DEV_TIMEOUT);
            }
        }
    } else if (warp == 1 || (C::NA == 2 && warp == C::MMA2_WARP)) {
        // MMA thread of weight tile w: its own accumulator, the shared token tile
        if (lane == 0) {
            const int w = (warp == 1) ? 0 : 1;
            int stage = 0;
            uint32_t phase = 0;
            int set = 0;  // TMEM scale set of the stage
            int acc = 0;
            uint32_t acc_phase = 0;
            for (int u = blockIdx.x; u < total; u += gridDim.x) {
                const Unit t = decode_unit(p, pref, u);
                const int n_mma = (t.n_valid + 15) & ~15;
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1, abort_flag)) break;
                tc_fence_after();
                const uint32_t d0 = tmem_base + acc * C::ACC_COLS + w * C::BNX;
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&full[stage], phase, abort_flag) ||
                        !mbar_wait(&sf_ready[stage], phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t st = smem_u32(smem + stage * C::STAGE_BYTES);
                    const uint32_t sfs = tmem_base + C::SF_COL + set * C::SET_COLS;
                    const uint32_t sfa = sfs + 4 * w;
                    const uint32_t sfb = sfs + 4 * C::NA;
#pragma unroll
                    for (int kk = 0; kk < MX_BK / 32; ++kk) {
                        const uint32_t acc_flag = (kb | kk) != 0;
                        const uint32_t idesc = idesc_mx_e2m1_e4m3(BM, n_mma, kk, kk);
                        const uint32_t sub = (uint32_t)kk << 30;  // k-block byte in each column
                        mma_mx(d0, sdesc_kmajor_sw128(st + C::A_OFF + w * C::A_BYTES + kk * 32),
                               sdesc_kmajor_sw128(st + C::B_OFF + kk * 32), idesc, sfa | sub,
                               sfb | sub, acc_flag);
                    }
                    mma_commit(&empty[stage]);
                    if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
                    if (++set == C::NSETS) set = 0;
                }
                if (!ok) break;
                mma_commit(&tfull[acc]);
                if (++acc == C::ACCB) { acc = 0; acc_phase ^= 1; }
            }
            mma_commit(mma_done);
            volatile int no_abort = 0;
            mbar_wait(mma_done, 0, &no_abort);
            if (*abort_flag) status_or(p.status, MOE_DEV_TIMEOUT);
        }
    } else if (warp >= C::SCALE_WARP && warp < C::SCALE_WARP + 4) {
        // scale warps. Per stage, lane m0 of quadrant q gathers for every operand
        // the stage's 4 k-block bytes of rows m0, m0+32, m0+64, m0+96 from the
        // ring slot and stores them to columns 0..3 of the operand in the
        // stage's TMEM set. A set is rewritten only after the MMAs that read it
        // completed (the empty barrier of the stage that last used it). A ring
        // slot serves eight stages (fewer at the end of a unit): every four stages
        // each lane loads the 16 bytes covering them of each of its rows (one
        // vector load per row instead of one 4-byte load per row per stage), and
        // the slot is released after the group's last such load.
        const uint32_t lane_cols = tmem_base + ((uint32_t)((warp & 3) * 32) << 16) + C::SF_COL;
        uint4 cache[C::NOPS][4];  // rows lane + 32 r: 16 bytes, the k-blocks of four stages
        int stage = 0;
        int set = 0;
        int g = 0;  // stages processed
        int sfs = 0;
        uint32_t sf_phase = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
            for (int kb = 0; kb < KB; ++kb) {
                if (kb % SF_STAGES == 0 && !warp_wait(&sf_full[sfs], sf_phase, abort_flag, lane)) {
                    ok = false;
                    break;
                }
                if (g >= C::NSETS) {
                    const int gp = g - C::NSETS;
                    if (!warp_wait(&empty[gp % C::STAGES], (uint32_t)(gp / C::STAGES) & 1u, abort_flag, lane)) {
                        ok = false;
                        break;
                    }
                }
                if ((kb & 3) == 0) {
                    // the next four stages' bytes of this lane's four rows, one 16-byte
                    // load per row; after the group's last such load the slot is free.
                    // The boxes arrive with a 32-byte swizzle: 16-byte piece c of row m
                    // sits at piece c ^ ((m >> 2) & 1), so the eight lanes of a load
                    // phase hit distinct banks (rows 32 bytes apart unswizzled put
                    // lanes m and m + 4 on one bank).
                    const uint8_t* raw = sf_ring + sfs * C::RAW_BYTES;
                    const int sf_swz = 16 * (((kb % SF_STAGES) >> 2) ^ ((lane >> 2) & 1));
#pragma unroll
                    for (int i = 0; i < C::NOPS; ++i)
#pragma unroll
                        for (int r = 0; r < 4; ++r)
                            cache[i][r] = *reinterpret_cast<const uint4*>(
                                raw + i * SF_TILE + SF_KB * (lane + 32 * r) + sf_swz);
                    if (kb % SF_STAGES == SF_STAGES - 4 || kb + 4 >= KB) {
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&sf_empty[sfs]);
                        if (++sfs == 2) { sfs = 0; sf_phase ^= 1; }
                    }
                }
                const int w = kb & 3;  // this stage's word: its 4 k-block bytes
                uint4 v[C::NOPS];
#pragma unroll
                for (int i = 0; i < C::NOPS; ++i)
                    v[i] = make_uint4(word_of(cache[i][0], w), word_of(cache[i][1], w), word_of(cache[i][2], w),
                                      word_of(cache[i][3], w));
#pragma unroll
                for (int i = 0; i < C::NOPS; ++i) tmem_st4(lane_cols + set * C::SET_COLS + 4 * i, v[i]);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sf_ready[stage]);
                if (++stage == C::STAGES) stage = 0;
                if (++set == C::NSETS) set = 0;
                ++g;
            }
        }
    } else if (GEMM == 2) {
        // down epilogue: NA accumulators of BNX columns, lane = output feature.
        // Group grp takes the 16-token chunks grp, grp + EG, ... Per chunk each
        // warp converts its 32 features to bf16 into its own shared [16 tokens]
        // [32 features] tile (two, alternating) and writes each token row's 64
        // bytes of them as four 16-byte pieces, two per lane; no barrier between
        // warps.
        const int q = warp & 3;
        const int grp = (warp - 2) >> 2;
        __nv_bfloat16* wbuf = ep_buf + (warp - 2) * 2 * 16 * 32;
        int acc = 0;
        uint32_t acc_phase = 0;
        int chunk = 0;
        for (int u = blockIdx.x; u < total; u += gridDim.x) {
            const Unit t = decode_unit(p, pref, u);
            if (!mbar_wait(&tfull[acc], acc_phase, abort_flag)) break;
            tc_fence_after();
#pragma unroll 1
            for (int w = 0; w < C::NA; ++w) {
                const uint32_t taddr =
                    tmem_base + ((uint32_t)(q * 32) << 16) + acc * C::ACC_COLS + w * C::BNX;
                __nv_bfloat16* out =
                    reinterpret_cast<__nv_bfloat16*>(t.out) + t.mt * p.tile_rows + w * BM + q * 32;
                for (int c0 = 16 * grp; c0 < t.n_valid; c0 += 16 * C::EG, ++chunk) {
                    uint32_t g[16];
                    tmem_ld16(taddr + c0, g);
                    tmem_ld_wait(g);
                    __nv_bfloat16* buf = wbuf + (chunk & 1) * 16 * 32;
#pragma unroll
                    for (int j = 0; j < 16; ++j) buf[j * 32 + lane] = __float2bfloat16_rn(__uint_as_float(g[j]));
                    __syncwarp();
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int i2 = lane + 32 * h;  // 16 token rows x 4 pieces of 8 features
                        const int r = i2 >> 2, pc = i2 & 3;
                        if (c0 + r < t.n_valid)
                            *reinterpret_cast<uint4*>(out + (size_t)(c0 + r) * p.ld_out + pc * 8) =
                                *reinterpret_cast<const uint4*>(buf + r * 32 + pc * 8);
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
            if (++acc == C::ACCB) { acc = 0; acc_phase ^= 1; }
        }
    } else {
        // GEMM1 epilogue: SwiGLU, then E4M3 + E8M0 block quantisation along I.
        // Group grp takes the 16-column chunks grp, grp + EG, ... Each chunk's
        // bytes and codes are staged in shared memory; after the group's four
        // warps meet, every lane writes one 16-byte piece of a 128-byte token row
        // (one-byte stores had made the single accumulator's drain stall the
        // tensor cores), and 16 lanes the rows' four scale codes.
        const int q = warp & 3;
        const int grp = (warp - 2) >> 2;
        const int row = q * 32 + lane;
        uint8_t* gstage = reinterpret_cast<uint8_t*>(ep_buf) + grp * 2 * C::G1_STAGE;
        uint64_t* gbar = ep_bar + 2 * grp;
        float* red_g = red + grp * 128;
        uint64_t* red_bar_g = red_bar + 2 * grp;
        int acc = 0;
        uint32_t acc_phase = 0;
        int chunk = 0;  // chunks this group has processed (amax exchange parity)
        bool ok = true;
        for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
            const Unit t = decode_unit(p, pref, u);
            if (!mbar_wait(&tfull[acc], acc_phase, abort_flag)) break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * C::ACC_COLS;
            uint8_t* hrow = t.out + t.mt * BM;     // first feature of the tile, row of the first token
            uint8_t* srow = t.sc + t.mt * BM / 32;  // its four 32-feature codes
            const int ld_sc = p.ld_out / 32;
            for (int c0 = 16 * grp; c0 < t.n_valid; c0 += 16 * C::EG, ++chunk) {
                uint32_t g[16], uu[16];
                tmem_ld16(taddr + c0, g);
                tmem_ld16(taddr + C::BNX + c0, uu);
                tmem_ld_wait(g, uu);
                // each step runs over all 16 token columns, branch-free, so the
                // columns' exp / reduction chains overlap
                float a[16], wmax[16];
                const bool lim = p.swiglu_limit > 0.0f;  // optional limit: min(g, L), clamp(u, -L, L)
                const float L = p.swiglu_limit;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float g0 = __uint_as_float(g[j]), u0 = __uint_as_float(uu[j]);
                    const float gv = lim ? fminf(g0, L) : g0;
                    const float uv = lim ? fminf(fmaxf(u0, -L), L) : u0;
                    a[j] = __fdividef(gv, 1.0f + __expf(-gv)) * uv;
                }
#pragma unroll
                for (int j = 0; j < 16; ++j) wmax[j] = warp_max_nonneg(fabsf(a[j]));
                int e[16];
                if (AFMT == MOE_A_MXFP8) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) e[j] = mx_exp(wmax[j]);
                } else {
                    // block of 128 features = the group's 4 warps: exchange warp maxima
                    const int par = chunk & 1;
                    float* r = red_g + par * 64;
                    if (lane < 16) {
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            if (j == lane) r[q * 16 + j] = wmax[j];
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&red_bar_g[par]);
                    if (!mbar_wait(&red_bar_g[par], (chunk >> 1) & 1, abort_flag)) { ok = false; break; }
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float m = fmaxf(fmaxf(r[j], r[16 + j]), fmaxf(r[32 + j], r[48 + j]));
                        e[j] = pow2_exp448(m);
                    }
                }
                uint8_t* b = gstage + (chunk & 1) * C::G1_STAGE;
#pragma unroll
                for (int j = 0; j < 16; j += 2) {
                    e[j] = min(max(e[j], -127), 127);
                    e[j + 1] = min(max(e[j + 1], -127), 127);
                    const uint32_t pr = e4m3x2_sat(a[j] * __uint_as_float((uint32_t)(127 - e[j]) << 23),
                                                   a[j + 1] * __uint_as_float((uint32_t)(127 - e[j + 1]) << 23));
                    b[j * BM + row] = (uint8_t)pr;
                    b[(j + 1) * BM + row] = (uint8_t)(pr >> 8);
                }
                if (lane == 0) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) b[16 * BM + j * 4 + q] = (uint8_t)(e[j] + 127);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&gbar[chunk & 1]);
                if (!mbar_wait(&gbar[chunk & 1], (uint32_t)(chunk >> 1) & 1u, abort_flag)) { ok = false; break; }
                const int f = q * 32 + lane;  // 16 token rows x 8 pieces of 16 bytes
                const int r = f >> 3, pc = f & 7;
                if (c0 + r < t.n_valid)
                    *reinterpret_cast<uint4*>(hrow + (size_t)(c0 + r) * p.ld_out + pc * 16) =
                        *reinterpret_cast<const uint4*>(b + r * BM + pc * 16);
                if (q == 0 && lane < 16 && c0 + lane < t.n_valid)
                    *reinterpret_cast<uint32_t*>(srow + (size_t)(c0 + lane) * ld_sc) =
                        *reinterpret_cast<const uint32_t*>(b + 16 * BM + lane * 4);
            }
            if (!ok) break;
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
            if (++acc == C::ACCB) { acc = 0; acc_phase ^= 1; }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace

template <int GEMM, int AFMT, int NA_, int BNX_, int ACCB_>
cudaError_t launch_mx(const GroupedGemmArgs& a, cudaStream_t st) {
    using C = TileMX<GEMM, NA_, BNX_, ACCB_>;
    const cudaError_t attr_err = ensure_smem_limit(
        reinterpret_cast<const void*>(grouped_gemm_mx_kernel<GEMM, AFMT, NA_, BNX_, ACCB_>), C::SMEM_BYTES);
    if (attr_err != cudaSuccess) return attr_err;
    uint64_t b_rows;
    KParams p = make_params(a, GEMM, &b_rows);
    p.bn = C::BNX;
    if (GEMM == 1) {
        p.out_esize = 1;  // E4M3 intermediate
        p.sc_routed = a.out_routed_scale;
        p.sc_shared = a.out_shared_scale;
    } else if (C::NA == 2) {
        // two consecutive 128-row blocks of the down projection per unit
        if (p.M % (2 * BM)) return cudaErrorInvalidValue;
        p.tile_rows = 2 * BM;
        p.a_up_offset = BM;
    }
    const int S = a.S;
    const uint64_t K = p.K, rowsA = (uint64_t)a.E * p.a_rows_per_mat;
    const uint64_t rowsAs = (uint64_t)(S > 0 ? S : a.E) * p.a_rows_per_mat;
    const void* wA = a.w_routed;
    const void* wAs = S > 0 ? a.w_shared : a.w_routed;
    const void* sA = a.w_routed_scale;
    const void* sAs = S > 0 ? a.w_shared_scale : a.w_routed_scale;
    CUtensorMap tmA, tmAs, tmSFA, tmSFAs, tmSFB;
    BMaps tmB;
    if (!make_tmap_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, wA, rowsA, K, K / 2, MX_BK, BM,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_2d(&tmAs, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, wAs, rowsAs, K, K / 2, MX_BK, BM,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_2d(&tmSFA, CU_TENSOR_MAP_DATA_TYPE_UINT8, sA, rowsA, K / 32, K / 32, SF_KB, 128,
                      CU_TENSOR_MAP_SWIZZLE_32B) ||
        !make_tmap_2d(&tmSFAs, CU_TENSOR_MAP_DATA_TYPE_UINT8, sAs, rowsAs, K / 32, K / 32, SF_KB, 128,
                      CU_TENSOR_MAP_SWIZZLE_32B))
        return cudaErrorInvalidValue;
    if (b_rows == 0) return cudaSuccess;
    if (!make_bmaps(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.b_rows, b_rows, K, MX_BK) ||
        !make_tmap_2d(&tmSFB, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.b_scale, b_rows, K / 32, K / 32, SF_KB,
                      C::SFB_ROWS, CU_TENSOR_MAP_SWIZZLE_32B))
        return cudaErrorInvalidValue;
    launch_pdl(grouped_gemm_mx_kernel<GEMM, AFMT, NA_, BNX_, ACCB_>, grid_for(p), C::THREADS,
        C::SMEM_BYTES, st, tmA, tmAs, tmSFA, tmSFAs, tmB, tmSFB, p);
    return cudaGetLastError();
}

cudaError_t launch_gemm_mx_pair_down(const GroupedGemmArgs& a, cudaStream_t st);

template <int AFMT>
cudaError_t launch_mx_tiles(const GroupedGemmArgs& a, cudaStream_t st) {
    // When experts average many tokens: 224-token tiles (gate/up single-buffered
    // with two epilogue groups; the down projection on CTA pairs, gemm_mx_pair.cu,
    // M = 256 over two SMs each loading half the token tile).
    // Otherwise 112-token tiles with double-buffered accumulators, so the
    // epilogue overlaps the next tile, and two weight tiles (two MMA threads)
    // per unit in both GEMMs.
    const bool wide = a.N >= 128L * a.E;
    if (a.gemm == 1)
        return wide ? launch_mx<1, AFMT, 2, 224, 1>(a, st) : launch_mx<1, AFMT, 2, 112, 2>(a, st);
    return wide ? launch_gemm_mx_pair_down(a, st) : launch_mx<2, AFMT, 2, 112, 2>(a, st);
}

cudaError_t launch_gemm_mx(const GroupedGemmArgs& a, cudaStream_t st) {
    if (a.afmt == MOE_A_MXFP8) return launch_mx_tiles<MOE_A_MXFP8>(a, st);
    return launch_mx_tiles<MOE_A_FP8_E4M3_POW2_B128>(a, st);
}

}  // namespace gemm
}  // namespace moe
