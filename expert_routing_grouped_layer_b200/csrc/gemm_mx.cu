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
// (16U4_ALIGN16B). Scales travel by TMA as 128 rows x 16 bytes (16 k-blocks).
// The MMA reads row m's scale (m = m0 + 32*m1) from TMEM lane m0 of every
// lane quadrant, column m1, one k-block per byte. A scale warp regroups the 4
// k-blocks of the current stage into that order (row m at byte
// 16*m0 + 4*m1 + kb of a 512-byte atom), in place over the staged scale
// tiles, and two operands' atoms share one 128-lane x 256-bit copy (each atom
// repeated for the 4 lane quadrants), so a stage issues half as many
// tensor-memory copies as operands.
// GEMM1's epilogue quantises the SwiGLU output per 32 (MXFP8) or per 128
// (power of two) along I, exactly as the activation quantiser does.
constexpr int MX_BK = 128;        // K elements per stage (one 128-byte smem row)
constexpr int SF_TILE = 128 * 16; // scale tile: 128 rows x 16 k-blocks of 32

// GEMM: 1 gate/up, 2 down. BNX_: tokens per tile. ACCB: accumulator buffers
// in tensor memory (2 overlaps a tile's epilogue with the next tile's main
// loop; 1 lets gate/up use 240-token tiles). Warps: 0 TMA, 1 MMA, then EG
// groups of 4 epilogue warps (one per TMEM lane quadrant), then the scale
// warp. Single-buffered gate/up tiles take three epilogue groups (measured
// faster than two), since there the quantising epilogue is not overlapped
// with the next tile's main loop.
template <int GEMM, int BNX_, int ACCB_>
struct TileMX {
    static constexpr int EG = (GEMM == 1 && ACCB_ == 1) ? 3 : 1;
    static constexpr int THREADS = 64 + 128 * EG + 32;
    static constexpr int SCALE_WARP = 2 + 4 * EG;
    static constexpr int RED_BYTES = EG * 2 * 4 * 16 * 4;  // [group][parity][warp][16 columns]
    static constexpr int NA = (GEMM == 1) ? 2 : 1;
    static constexpr int BNX = BNX_;
    static constexpr int ACCB = ACCB_;
    static constexpr int SFB_ROWS = (BNX + 127) / 128 * 128;  // token rows of the scale tile
    static constexpr int SFB_ATOMS = SFB_ROWS / 128;
    static constexpr int NOPS = NA + SFB_ATOMS;  // scale operands: A gate, [A up], B rows 0-127, [128-255]
    static constexpr int NPAIR = NOPS / 2;       // operand pairs copied by one 128x256b copy
    static constexpr int A_BYTES = BM * MX_BK;                // one byte per E2M1 value in smem
    static constexpr int B_BYTES = BNX * MX_BK;
    static constexpr int A_OFF = 0;
    static constexpr int B_OFF = NA * A_BYTES;
    static constexpr int SF_OFF = B_OFF + B_BYTES;  // regrouped scale atoms of the stage
    static constexpr int RAW_BYTES = NOPS * SF_TILE;  // staged scale tiles, operand i at i*SF_TILE
    static constexpr int ATOM_BYTES = NPAIR * 2 * SF_TILE + (NOPS & 1) * 512;
    // A scale box covers 16 k-blocks, four stages. Normally the boxes go to a
    // two-slot ring, loaded once per four stages, and the scale warp writes the
    // atoms into the stage. Where that ring would cost a pipeline stage (wide
    // gate/up tiles), each stage loads the boxes itself and the atoms overwrite
    // them in place.
    static constexpr int FIXED_BYTES =
        1024 + 8 * (3 * 6 + 9 + 2 * EG) + 16 + 4 * (MAX_SEG + 1) + RED_BYTES;
    static constexpr int STAGE_RING = (SF_OFF + ATOM_BYTES + 1023) / 1024 * 1024;
    static constexpr int STAGES_RING = stages_for(STAGE_RING, FIXED_BYTES + 2 * RAW_BYTES, 6);
    static constexpr int STAGE_INPLACE = (SF_OFF + RAW_BYTES + 1023) / 1024 * 1024;
    static constexpr int STAGES_INPLACE = stages_for(STAGE_INPLACE, FIXED_BYTES, 6);
    static constexpr bool SF_RING = STAGES_RING >= 4 || STAGES_RING >= STAGES_INPLACE;
    static constexpr int STAGE_BYTES = SF_RING ? STAGE_RING : STAGE_INPLACE;
    static constexpr int STAGES = SF_RING ? STAGES_RING : STAGES_INPLACE;
    static constexpr int RING_BYTES = SF_RING ? 2 * RAW_BYTES : 0;
    static constexpr int ACC_COLS = NA * BNX;
    static constexpr int SF_COL = ACCB * ACC_COLS;  // scale columns: operand i at SF_COL + 4*i
    static constexpr int TMEM_COLS = 512;
    static_assert(SF_COL % 8 == 0, "256-bit scale copies start on a multiple of 8 columns");
    static_assert(SF_COL + 4 * NOPS <= TMEM_COLS, "tensor memory budget");
    static constexpr int BAR_BYTES = 8 * (3 * STAGES + 9 + 2 * EG) + 16;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + RING_BYTES + BAR_BYTES +
                                      4 * (MAX_SEG + 1) + RED_BYTES;  // + cross-warp amax exchange
    static_assert(STAGES >= 2 && SMEM_BYTES <= 232448, "shared memory budget");
};

// 128 lanes x 256 bits from shared memory (two 16-byte halves 2048 bytes apart,
// rows 16 bytes apart) to 8 TMEM columns.
__device__ __forceinline__ void tmem_cp_128x256b(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.128x256b [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

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

__device__ __forceinline__ uint8_t e4m3_sat(float v) {
    return (uint8_t)(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3));
}

template <int GEMM, int AFMT, int BNX_, int ACCB_>
__global__ void __launch_bounds__(TileMX<GEMM, BNX_, ACCB_>::THREADS, 1)
    grouped_gemm_mx_kernel(const __grid_constant__ CUtensorMap tmA_routed,
                           const __grid_constant__ CUtensorMap tmA_shared,
                           const __grid_constant__ CUtensorMap tmSFA_routed,
                           const __grid_constant__ CUtensorMap tmSFA_shared,
                           const __grid_constant__ BMaps tmB,
                           const __grid_constant__ CUtensorMap tmSFB, const KParams p) {
    using C = TileMX<GEMM, BNX_, ACCB_>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* sf_ring = smem + C::STAGES * C::STAGE_BYTES;  // [2][RAW_BYTES] (ring variant)
    uint64_t* full = reinterpret_cast<uint64_t*>(sf_ring + C::RING_BYTES);
    uint64_t* empty = full + C::STAGES;
    uint64_t* sf_ready = empty + C::STAGES;  // scales regrouped for the stage
    uint64_t* tfull = sf_ready + C::STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* mma_done = tempty + 2;
    uint64_t* sf_full = mma_done + 1;  // [2] scale ring slots
    uint64_t* sf_empty = sf_full + 2;  // [2]
    uint64_t* red_bar = sf_empty + 2;  // [group][parity]: the amax exchange of a group's 4 warps
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(red_bar + 2 * C::EG);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* pref = reinterpret_cast<int*>(tmem_slot + 4);
    float* red = reinterpret_cast<float*>(pref + MAX_SEG + 1);  // [group][parity][4 warps][16]

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
            mbar_init(&tempty[a], 128 * C::EG);
        }
        mbar_init(mma_done, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sf_full[i], 1);
            mbar_init(&sf_empty[i], 1);
        }
        for (int i = 0; i < 2 * C::EG; ++i) mbar_init(&red_bar[i], 4);
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
            int sfs = 0, sf_issued = 0;  // scale ring slot and loads issued into the ring
            uint32_t sf_phase = 0;
            for (int u = blockIdx.x; u < total && !*abort_flag; u += gridDim.x) {
                const Unit t = decode_unit(p, pref, u);
                const int n_mma = (t.n_valid + 15) & ~15;
                // a padded E2M1 tile occupies A_BYTES of shared memory but the copy
                // counts its packed size (4 bits per value) toward the transaction
                const uint32_t tx = C::NA * (C::A_BYTES / 2) + n_mma * MX_BK +
                                    (C::SF_RING ? 0 : C::RAW_BYTES);
                const bool routed = t.seg < p.E;
                const CUtensorMap* tmA = routed ? &tmA_routed : &tmA_shared;
                const CUtensorMap* tmSFA = routed ? &tmSFA_routed : &tmSFA_shared;
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb) {
                    const int sfx = (kb >> 2) * 16;  // 16-k-block group holding this stage
                    if (C::SF_RING && (kb & 3) == 0) {
                        if (!mbar_wait(&sf_empty[sfs], sf_phase ^ 1, abort_flag)) { ok = false; break; }
                        uint8_t* sl = sf_ring + sfs * C::RAW_BYTES;
                        mbar_arrive_expect_tx(&sf_full[sfs], C::RAW_BYTES);
                        tma_load_2d(sl, tmSFA, sfx, t.a_row, &sf_full[sfs]);
                        if (GEMM == 1)
                            tma_load_2d(sl + SF_TILE, tmSFA, sfx, t.a_row + p.a_up_offset, &sf_full[sfs]);
                        tma_load_2d(sl + C::NA * SF_TILE, &tmSFB, sfx, t.b_row, &sf_full[sfs]);
                        ++sf_issued;
                        if (++sfs == 2) { sfs = 0; sf_phase ^= 1; }
                    }
                    if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
                    uint8_t* st = smem + stage * C::STAGE_BYTES;
                    mbar_arrive_expect_tx(&full[stage], tx);
                    tma_load_2d(st + C::A_OFF, tmA, kb * MX_BK, t.a_row, &full[stage]);
                    if (GEMM == 1)
                        tma_load_2d(st + C::A_OFF + C::A_BYTES, tmA, kb * MX_BK,
                                    t.a_row + p.a_up_offset, &full[stage]);
                    load_b_rows(st + C::B_OFF, tmB, kb * MX_BK, t.b_row, n_mma, MX_BK, &full[stage]);
                    if (!C::SF_RING) {
                        tma_load_2d(st + C::SF_OFF, tmSFA, sfx, t.a_row, &full[stage]);
                        if (GEMM == 1)
                            tma_load_2d(st + C::SF_OFF + SF_TILE, tmSFA, sfx, t.a_row + p.a_up_offset,
                                        &full[stage]);
                        tma_load_2d(st + C::SF_OFF + C::NA * SF_TILE, &tmSFB, sfx, t.b_row,
                                    &full[stage]);
                    }
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
    } else if (warp == 1) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            const uint32_t sfa_gate = tmem_base + C::SF_COL;
            const uint32_t sfa_up = tmem_base + C::SF_COL + 4;
            const uint32_t sfb = tmem_base + C::SF_COL + 4 * C::NA;
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
#pragma unroll
                    for (int pr = 0; pr < C::NPAIR; ++pr)
                        tmem_cp_128x256b(sfa_gate + 8 * pr,
                                         sdesc_kmajor_noswizzle_rows16(st + C::SF_OFF + pr * 2 * SF_TILE));
                    if (C::NOPS & 1)
                        tmem_cp_32x128b_x4(sfa_gate + 8 * C::NPAIR, sdesc_kmajor_noswizzle_rows16(
                                                                     st + C::SF_OFF + 2 * C::NPAIR * SF_TILE));
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
                if (++acc == C::ACCB) { acc = 0; acc_phase ^= 1; }
            }
            mma_commit(mma_done);
            volatile int no_abort = 0;
            mbar_wait(mma_done, 0, &no_abort);
            if (*abort_flag) status_or(p.status, MOE_DEV_TIMEOUT);
        }
    } else if (warp == C::SCALE_WARP) {
        // scale warp: regroup this stage's 4 k-blocks of every staged 128 x 16-byte
        // scale tile (lane m0 gathers rows m0 + 32*m1) into the stage's atoms.
        // Operand pair pr becomes a 128-row x 32-byte copy source: operand 2pr in
        // the first 16-byte half, 2pr+1 in the second (2048 bytes on), each atom
        // written for rows m0, m0+32, m0+64, m0+96. An odd last operand stays one
        // 512-byte atom. A ring slot serves four stages, then is released.
        int stage = 0;
        uint32_t phase = 0;
        int sfs = 0;
        uint32_t sf_phase = 0;
        for (int u = blockIdx.x; u < total; u += gridDim.x) {
            bool ok = true;
            for (int kb = 0; kb < KB; ++kb) {
                if (C::SF_RING && (kb & 3) == 0 && !mbar_wait(&sf_full[sfs], sf_phase, abort_flag)) {
                    ok = false;
                    break;
                }
                if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
                uint8_t* atoms = smem + stage * C::STAGE_BYTES + C::SF_OFF;
                const uint8_t* raw = C::SF_RING ? sf_ring + sfs * C::RAW_BYTES : atoms;
                const int j4 = (kb & 3) * 4;  // byte offset of this stage's k-blocks in a row
                uint4 v[C::NOPS];
#pragma unroll
                for (int i = 0; i < C::NOPS; ++i) {
                    const uint8_t* src = raw + i * SF_TILE;
                    v[i].x = *reinterpret_cast<const uint32_t*>(src + 16 * (lane + 0) + j4);
                    v[i].y = *reinterpret_cast<const uint32_t*>(src + 16 * (lane + 32) + j4);
                    v[i].z = *reinterpret_cast<const uint32_t*>(src + 16 * (lane + 64) + j4);
                    v[i].w = *reinterpret_cast<const uint32_t*>(src + 16 * (lane + 96) + j4);
                }
                __syncwarp();  // in place: every lane has read the tiles before they are overwritten
                if (C::SF_RING && (kb & 3) == 3) {
                    if (lane == 0) mbar_arrive(&sf_empty[sfs]);
                    if (++sfs == 2) { sfs = 0; sf_phase ^= 1; }
                }
#pragma unroll
                for (int i = 0; i < 2 * C::NPAIR; ++i) {
                    uint8_t* dst = atoms + (i >> 1) * 2 * SF_TILE + (i & 1) * SF_TILE;
#pragma unroll
                    for (int r = 0; r < 4; ++r)
                        *reinterpret_cast<uint4*>(dst + 16 * (lane + 32 * r)) = v[i];
                }
                if (C::NOPS & 1)
                    *reinterpret_cast<uint4*>(atoms + 2 * C::NPAIR * SF_TILE + 16 * lane) =
                        v[C::NOPS - 1];
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sf_ready[stage]);
                if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
            }
            if (!ok) break;
        }
    } else if (GEMM == 2) {
        epilogue_loop<2, C::ACC_COLS, C::ACCB>(p, pref, total, tmem_base, tfull, tempty, abort_flag,
                                               warp, lane);
    } else {
        // GEMM1 epilogue: SwiGLU, then E4M3 + E8M0 block quantisation along I.
        // Group grp takes the 16-column chunks grp, grp + EG, ...
        const int q = warp & 3;
        const int grp = (warp - 2) >> 2;
        const int row = q * 32 + lane;
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
            const int feat = t.mt * BM + row;  // output feature (column of h)
            uint8_t* out = t.out + feat;
            uint8_t* sc = t.sc + (t.mt * BM + q * 32) / 32;
            const int ld_sc = p.ld_out / 32;
            for (int c0 = 16 * grp; c0 < t.n_valid; c0 += 16 * C::EG, ++chunk) {
                uint32_t g[16], uu[16];
                tmem_ld16(taddr + c0, g);
                tmem_ld16(taddr + C::BNX + c0, uu);
                tmem_ld_wait(g, uu);
                float a[16], wmax[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    float gv = __uint_as_float(g[j]), uv = __uint_as_float(uu[j]);
                    if (p.swiglu_limit > 0.0f) {  // optional limit: min(g, L), clamp(u, -L, L)
                        gv = fminf(gv, p.swiglu_limit);
                        uv = fminf(fmaxf(uv, -p.swiglu_limit), p.swiglu_limit);
                    }
                    a[j] = __fdividef(gv, 1.0f + __expf(-gv)) * uv;
                    wmax[j] = warp_max_nonneg(fabsf(a[j]));
                }
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

template <int GEMM, int AFMT, int BNX_, int ACCB_>
cudaError_t launch_mx(const GroupedGemmArgs& a, cudaStream_t st) {
    using C = TileMX<GEMM, BNX_, ACCB_>;
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(grouped_gemm_mx_kernel<GEMM, AFMT, BNX_, ACCB_>,
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
    CUtensorMap tmA, tmAs, tmSFA, tmSFAs, tmSFB;
    BMaps tmB;
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
    if (!make_bmaps(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.b_rows, b_rows, K, MX_BK) ||
        !make_tmap_2d(&tmSFB, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.b_scale, b_rows, K / 32, K / 32, 16,
                      C::SFB_ROWS, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    grouped_gemm_mx_kernel<GEMM, AFMT, BNX_, ACCB_><<<grid_for(p), C::THREADS, C::SMEM_BYTES, st>>>(
        tmA, tmAs, tmSFA, tmSFAs, tmB, tmSFB, p);
    return cudaGetLastError();
}

template <int AFMT>
cudaError_t launch_mx_tiles(const GroupedGemmArgs& a, cudaStream_t st) {
    // When experts average many tokens: 240-token tiles (gate/up single-buffered
    // with two epilogue groups, down double-buffered). Otherwise gate/up takes
    // 112-token tiles with double-buffered accumulators, so the quantising
    // epilogue overlaps the next tile, and down 128-token tiles with a deeper ring.
    const bool wide = a.N >= 128L * a.E;
    if (a.gemm == 1)
        return wide ? launch_mx<1, AFMT, 240, 1>(a, st) : launch_mx<1, AFMT, 112, 2>(a, st);
    return wide ? launch_mx<2, AFMT, 240, 2>(a, st) : launch_mx<2, AFMT, 128, 2>(a, st);
}

cudaError_t launch_gemm_mx(const GroupedGemmArgs& a, cudaStream_t st) {
    if (a.afmt == MOE_A_MXFP8) return launch_mx_tiles<MOE_A_MXFP8>(a, st);
    return launch_mx_tiles<MOE_A_FP8_E4M3_POW2_B128>(a, st);
}

}  // namespace gemm
}  // namespace moe
