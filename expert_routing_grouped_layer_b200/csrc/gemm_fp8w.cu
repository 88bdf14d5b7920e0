// gemm_fp8w.cu -- per-expert SwiGLU MLP with FP8 (E4M3, 128x128 block-scaled)
// weights and bf16 activations on the tcgen05 tensor cores. The expert
// structure and tile schedule are those of gemm_bf16.cu.
#include <cuda_fp16.h>

#include "gemm_common.cuh"

namespace moe {
namespace gemm {
namespace {

// ---------------------------------------------------------------- FP8 weights
// E4M3 weights with one fp32 scale per 128x128 block ("DeepSeek-V4-Pro 架构与代码概述",
// 文件说明: Linear with block-scaled FP8 weights; block 128x128). There is no
// tensor-core instruction for E4M3 times bf16, so a converter warpgroup turns
// each TMA-staged E4M3 weight tile into 16-bit values times the tile's block
// scale, written straight into the 128B-swizzled K-major layout tcgen05.mma
// reads. A staged tile spans two MMA stages of BK = 64 (128-byte swizzled
// rows): the TMA unit keeps a bounded number of row requests in flight and an
// HBM row holds its slot for the DRAM latency whatever its width, so full
// 128-byte rows halve the weight stream's cost there against 64-byte ones.
// With a staged tile inside one 128-wide scale block and M tiles aligned to
// the 128-row blocks, one scalar scale covers a tile.
// Both GEMMs run on f16 operands (see the f16 path below): one cvt and one
// f16x2 multiply per two weights. Token rows come in as f16 with a power-of-two
// row scale, and so does the SwiGLU output h (the gate/up call rewrites its
// bf16 rows in place).
constexpr int CVT_WARPS = 8;
constexpr int CVT_THREADS = CVT_WARPS * 32;
constexpr int B_WARP = 6 + CVT_WARPS;  // token-tile loader, after the converters
constexpr int EPI2_WARP = B_WARP + 1;  // second epilogue group (gate/up), after the loader
static_assert(512 % CVT_THREADS == 0, "converter tasks: whole tiles per round");

// Gate/up with the converted weight tiles in shared memory (the narrow-tile
// variant; wide tiles keep them in tensor memory, below). GEMM: 1 (gate/up).
// BNF_: tokens per tile. ACCB_: accumulator buffers in tensor memory (2
// overlaps a tile's epilogue with the next main loop). Two rings: the raw ring
// holds the TMA-staged e4m3 weight tiles and is freed as soon as the converters
// have read a slot, so it can run many stages ahead of the tensor cores; the
// MMA ring holds the converted f16 weight tiles and the token tile, freed by
// the MMA commit.
template <int GEMM, int BNF_, int ACCB_, int MST_>
struct TileF8 {
    static_assert(GEMM == 1, "the shared-memory variant serves the gate/up GEMM");
    // a second group of 4 epilogue warps halves the drain of the accumulator
    static constexpr int EG = 2;
    static constexpr int THREADS = 64 + 128 + CVT_THREADS + 32 + 128 * (EG - 1);
    static constexpr int NA = 2;
    static constexpr int BNF = BNF_;
    static constexpr int ACCB = ACCB_;
    static constexpr int RK = 2 * BK;             // K of a staged e4m3 tile (two MMA stages)
    static constexpr int A8_BYTES = BM * RK;      // e4m3 staging tile, 128-byte rows
    static constexpr int A_BYTES = BM * BK * 2;   // f16 MMA tile
    static constexpr int B_BYTES = BNF * BK * 2;
    static constexpr int CVT_OFF = 0;                       // NA f16 A tiles
    static constexpr int B_OFF = NA * A_BYTES;              // token tile
    static constexpr int MSLOT_BYTES = (B_OFF + B_BYTES + 1023) / 1024 * 1024;
    static constexpr int RSLOT_BYTES = NA * A8_BYTES;       // NA e4m3 tiles (two MMA stages)
    static constexpr int MSTAGES = MST_;
    static constexpr int FIXED_BYTES = 1024 + 8 * (2 * 8 + 3 * MSTAGES + 5) + 16 + 4 * (MAX_SEG + 1);
    static constexpr int RSTAGES_FIT = (232448 - FIXED_BYTES - MSTAGES * MSLOT_BYTES) / RSLOT_BYTES;
    static constexpr int RSTAGES = RSTAGES_FIT < 8 ? RSTAGES_FIT : 8;
    static constexpr int ACC_COLS = NA * BNF;
    static constexpr int TMEM_COLS = 512;
    static_assert(ACCB * ACC_COLS <= TMEM_COLS, "tensor memory budget");
    static constexpr int RING_BYTES = MSTAGES * MSLOT_BYTES + RSTAGES * RSLOT_BYTES;
    static constexpr int BAR_BYTES = 8 * (2 * RSTAGES + 3 * MSTAGES + 5) + 16;
    static constexpr int SMEM_BYTES = 1024 + RING_BYTES + BAR_BYTES + 4 * (MAX_SEG + 1);
    static_assert(RSTAGES >= 2 && SMEM_BYTES <= 232448, "shared memory budget");
};

// ---- f16 path of the gate/up GEMM. The tensor-core operands are f16: token
// rows arrive as x * 2^-e (exact, see pack_f16_kernel) and each weight tile is
// E4M3 (exact in f16) times m = s * 2^-E rounded to f16, where s is the tile's
// 128x128 block scale and 2^E the largest power of two not above the largest
// block scale of the 128 rows' K range (|m| < 2; weight products round once in
// f16, <= 2^-11 relative, plus <= 2^-12 for m). The epilogue multiplies the
// accumulator by 2^E * 2^e exactly. Conversion is one cvt and one f16x2
// multiply per two weights.

// Exponent E of a 128-row tile: max over its KS block scales of floor(log2 s),
// kept in [-126, 126]. Every lane of the warp returns the same value.
__device__ __forceinline__ int tile_exp(const float* __restrict__ srow, int KS, int lane) {
    int e = -126;
    for (int j = lane; j < KS; j += 32) {
        const float sj = srow[j];
        if (sj > 0.f) e = max(e, ilogbf(sj));
    }
    e = __reduce_max_sync(0xffffffffu, e);
    return min(e, 126);
}

__device__ __forceinline__ float pow2f(int e) {  // 2^e for e in [-126, 127]
    return __uint_as_float((uint32_t)(127 + e) << 23);
}

// 16 E4M3 values times the f16 pair (m, m) -> 16 f16 values, in element order.
__device__ __forceinline__ void e4m3x16_to_f16_scaled(uint4 v, __half2 m2, uint4& lo, uint4& hi) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const __nv_fp8x2_storage_t pair = (__nv_fp8x2_storage_t)((w[i] >> (16 * h)) & 0xFFFFu);
            const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);
            const __half2 p = __hmul2(*reinterpret_cast<const __half2*>(&hr), m2);
            o[2 * i + h] = *reinterpret_cast<const uint32_t*>(&p);
        }
    }
    lo = make_uint4(o[0], o[1], o[2], o[3]);
    hi = make_uint4(o[4], o[5], o[6], o[7]);
}

// Instruction descriptor, kind::f16 with f16 A and B (format 0), fp32 accumulate.
__host__ __device__ __forceinline__ uint32_t idesc_f16(uint32_t M, uint32_t N) {
    return (1u << 4) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

// Gate/up epilogue of the f16 path: per unit, wait for the accumulator, read it
// 16 token columns at a time (lane = output feature; group g of GROUPS takes
// chunks g, g + GROUPS, ...), restore 2^E (gate and up tiles) and 2^e (token
// row), apply SwiGLU, store bf16, release the buffer (128 * GROUPS arrivals).
template <int ACC_COLS, int ACCB, int GROUPS>
__device__ __forceinline__ void epilogue_f16_gate_up(const KParams& p, const int* pref, int total,
                                                     uint32_t tmem_base, uint64_t* tfull,
                                                     uint64_t* tempty, volatile int* abort_flag,
                                                     int warp, int lane, int group,
                                                     const float* __restrict__ scale_routed,
                                                     const float* __restrict__ scale_shared,
                                                     const int8_t* __restrict__ row_exp) {
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int KS = p.K / 128;
    const int RS = p.a_rows_per_mat / 128;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int u = blockIdx.x; u < total; u += gridDim.x) {
        const Unit t = decode_unit(p, pref, u);
        const bool routed = t.seg < p.E;
        const int mat = routed ? t.seg : t.seg - p.E;
        const float* sbase = (routed ? scale_routed : scale_shared) + (size_t)mat * RS * KS;
        const float fg = pow2f(tile_exp(sbase + (size_t)t.mt * KS, KS, lane));
        const float fu = pow2f(tile_exp(sbase + (size_t)(p.a_up_offset / 128 + t.mt) * KS, KS, lane));
        if (!mbar_wait(&tfull[acc], acc_phase, abort_flag)) break;
        tc_fence_after();
        const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * ACC_COLS;
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(t.out) + t.mt * BM + row;
        for (int c0 = 16 * group; c0 < t.n_valid; c0 += 16 * GROUPS) {
            uint32_t g[16], uu[16];
            tmem_ld16(taddr + c0, g);
            tmem_ld16(taddr + ACC_COLS / 2 + c0, uu);
            // 2^e of this lane's token column (e in [-127, 114]; 2^-127 is subnormal)
            const int ex_l = (lane < 16 && c0 + lane < t.n_valid) ? row_exp[t.b_row + c0 + lane] : 0;
            const float fe_l = ex_l >= -126 ? pow2f(ex_l) : __uint_as_float(0x00400000u);
            tmem_ld_wait(g, uu);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float fe = __shfl_sync(0xffffffffu, fe_l, j);
                if (c0 + j < t.n_valid) {
                    const float gv = __uint_as_float(g[j]) * fg * fe;  // exact power-of-two factors
                    const float uv = __uint_as_float(uu[j]) * fu * fe;
                    const float a = swiglu(gv, uv, p.swiglu_limit);
                    out[(size_t)(c0 + j) * p.ld_out] = __float2bfloat16_rn(a);
                }
            }
        }
        tc_fence_before();
        mbar_arrive(&tempty[acc]);
        if (++acc == ACCB) { acc = 0; acc_phase ^= 1; }
    }
}

// Down epilogue of the f16 path: per unit, wait for the accumulator, read it 16
// token columns at a time (lane = output feature), restore 2^E (the W2 tile) and
// 2^e (the token's h row), and store bf16. Each warp stages its 16 x 32 chunk in
// its own shared [16 tokens][32 features] tile (two, alternating) and writes
// every token row's 64 bytes as four 16-byte pieces (two per lane), instead of
// one 2-byte store per element; then it releases the buffer.
template <int ACC_COLS, int ACCB>
__device__ __forceinline__ void epilogue_f16_down(const KParams& p, const int* pref, int total,
                                                  uint32_t tmem_base, uint64_t* tfull, uint64_t* tempty,
                                                  volatile int* abort_flag, int warp, int lane,
                                                  const float* __restrict__ scale_routed,
                                                  const float* __restrict__ scale_shared,
                                                  const int8_t* __restrict__ row_exp,
                                                  __nv_bfloat16* wbuf) {
    const int q = warp & 3;
    const int KS = p.K / 128;
    const int RS = p.a_rows_per_mat / 128;
    int acc = 0;
    uint32_t acc_phase = 0;
    int chunk = 0;
    for (int u = blockIdx.x; u < total; u += gridDim.x) {
        const Unit t = decode_unit(p, pref, u);
        const bool routed = t.seg < p.E;
        const int mat = routed ? t.seg : t.seg - p.E;
        const float* sbase = (routed ? scale_routed : scale_shared) + (size_t)mat * RS * KS;
        const float fw = pow2f(tile_exp(sbase + (size_t)t.mt * KS, KS, lane));
        if (!mbar_wait(&tfull[acc], acc_phase, abort_flag)) break;
        tc_fence_after();
        const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * ACC_COLS;
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(t.out) + t.mt * BM + q * 32;
        for (int c0 = 0; c0 < t.n_valid; c0 += 16, ++chunk) {
            uint32_t g[16];
            tmem_ld16(taddr + c0, g);
            // 2^e of this lane's token column (e in [-127, 114]; 2^-127 is subnormal)
            const int ex_l = (lane < 16 && c0 + lane < t.n_valid) ? row_exp[t.b_row + c0 + lane] : 0;
            const float fe_l = ex_l >= -126 ? pow2f(ex_l) : __uint_as_float(0x00400000u);
            tmem_ld_wait(g);
            __nv_bfloat16* b = wbuf + (chunk & 1) * 16 * 32;
#pragma unroll
            for (int j = 0; j < 16; ++j) {  // exact power-of-two factors
                const float fe = __shfl_sync(0xffffffffu, fe_l, j);
                b[j * 32 + lane] = __float2bfloat16_rn(__uint_as_float(g[j]) * fw * fe);
            }
            __syncwarp();
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int i = lane + 32 * k;  // 16 token rows x 4 pieces of 8 features
                const int r = i >> 2, pc = i & 3;
                if (c0 + r < t.n_valid)
                    *reinterpret_cast<uint4*>(out + (size_t)(c0 + r) * p.ld_out + pc * 8) =
                        *reinterpret_cast<const uint4*>(b + r * 32 + pc * 8);
            }
        }
        tc_fence_before();
        mbar_arrive(&tempty[acc]);
        if (++acc == ACCB) { acc = 0; acc_phase ^= 1; }
    }
}

template <int GEMM, int BNF_, int ACCB_, int MST_>
__global__ void __launch_bounds__(TileF8<GEMM, BNF_, ACCB_, MST_>::THREADS, 1)
    grouped_gemm_fp8w_kernel(const __grid_constant__ CUtensorMap tmA_routed,
                             const __grid_constant__ CUtensorMap tmA_shared,
                             const __grid_constant__ BMaps tmB, const KParams p,
                             const float* __restrict__ scale_routed,
                             const float* __restrict__ scale_shared,
                             const int8_t* __restrict__ row_exp) {
    pdl_wait();
    pdl_trigger();
    using C = TileF8<GEMM, BNF_, ACCB_, MST_>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* mring = smem;                                    // [MSTAGES][MSLOT_BYTES]
    uint8_t* rring = smem + C::MSTAGES * C::MSLOT_BYTES;      // [RSTAGES][RSLOT_BYTES]
    uint64_t* raw_full = reinterpret_cast<uint64_t*>(smem + C::RING_BYTES);
    uint64_t* raw_empty = raw_full + C::RSTAGES;
    uint64_t* b_full = raw_empty + C::RSTAGES;   // token tile landed in the MMA slot
    uint64_t* cvt_full = b_full + C::MSTAGES;    // weight tiles converted into the MMA slot
    uint64_t* m_empty = cvt_full + C::MSTAGES;   // MMA slot consumed
    uint64_t* tfull = m_empty + C::MSTAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* mma_done = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* pref = reinterpret_cast<int*>(tmem_slot + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::RSTAGES; ++s) {
            mbar_init(&raw_full[s], 1);
            mbar_init(&raw_empty[s], CVT_THREADS);
        }
        for (int s = 0; s < C::MSTAGES; ++s) {
            mbar_init(&b_full[s], 1);
            mbar_init(&cvt_full[s], CVT_THREADS);
            mbar_init(&m_empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 128 * C::EG);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmA_routed);
        tma_prefetch_desc(&tmA_shared);
        prefetch_bmaps(tmB);
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
        // producer: e4m3 weight tiles (RK each) into the raw ring
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            for (int u = blockIdx.x; u < total && !*abort_flag; u += gridDim.x) {
                const Unit t = decode_unit(p, pref, u);
                const CUtensorMap* tmA = (t.seg < p.E) ? &tmA_routed : &tmA_shared;
                bool ok = true;
                for (int kr = 0; kr < KB / 2; ++kr) {
                    if (!mbar_wait(&raw_empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
                    uint8_t* rs = rring + stage * C::RSLOT_BYTES;
                    mbar_arrive_expect_tx(&raw_full[stage], C::RSLOT_BYTES);
                    tma_load_2d(rs, tmA, kr * C::RK, t.a_row, &raw_full[stage]);
                    tma_load_2d(rs + C::A8_BYTES, tmA, kr * C::RK, t.a_row + p.a_up_offset, &raw_full[stage]);
                    ++issued;
                    if (++stage == C::RSTAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
            }
            if (*abort_flag) {
                int s = stage;
                uint32_t ph = phase;
                for (int i = 0; i < min(issued, C::RSTAGES); ++i) {
                    if (--s < 0) { s = C::RSTAGES - 1; ph ^= 1; }
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
                const uint32_t idesc = idesc_f16(BM, n_mma);
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1, abort_flag)) break;
                tc_fence_after();
                const uint32_t d0 = tmem_base + acc * C::ACC_COLS;
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&b_full[stage], phase, abort_flag) ||
                        !mbar_wait(&cvt_full[stage], phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t st = smem_u32(mring + stage * C::MSLOT_BYTES);
                    const uint32_t sb = st + C::B_OFF;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint32_t acc_flag = (kb | kk) != 0;
                        const uint64_t bd = sdesc_kmajor_sw128(sb + kk * 32);
                        mma_bf16(d0, sdesc_kmajor_sw128(st + C::CVT_OFF + kk * 32), bd, idesc, acc_flag);
                        mma_bf16(d0 + C::BNF, sdesc_kmajor_sw128(st + C::CVT_OFF + C::A_BYTES + kk * 32), bd,
                                 idesc, acc_flag);
                    }
                    mma_commit(&m_empty[stage]);
                    if (++stage == C::MSTAGES) { stage = 0; phase ^= 1; }
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
    } else if (warp == B_WARP) {
        // token-tile loader: fills each MMA slot's token tile as soon as it is free
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            for (int u = blockIdx.x; u < total && !*abort_flag; u += gridDim.x) {
                const Unit t = decode_unit(p, pref, u);
                const int n_mma = (t.n_valid + 15) & ~15;
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&m_empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
                    mbar_arrive_expect_tx(&b_full[stage], (uint32_t)(n_mma * BK * 2));
                    load_b_rows(mring + stage * C::MSLOT_BYTES + C::B_OFF, tmB, kb * BK, t.b_row, n_mma,
                                BK * 2, &b_full[stage]);
                    ++issued;
                    if (++stage == C::MSTAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
            }
            if (*abort_flag) {
                int s = stage;
                uint32_t ph = phase;
                for (int i = 0; i < min(issued, C::MSTAGES); ++i) {
                    if (--s < 0) { s = C::MSTAGES - 1; ph ^= 1; }
                    volatile int no_abort = 0;
                    mbar_wait(&b_full[s], ph, &no_abort);
                }
            }
        }
    } else if (warp < 6 || warp >= EPI2_WARP) {
        epilogue_f16_gate_up<C::ACC_COLS, C::ACCB, C::EG>(p, pref, total, tmem_base, tfull, tempty,
                                                          abort_flag, warp, lane, warp < 6 ? 0 : 1,
                                                          scale_routed, scale_shared, row_exp);
    } else {
        // converters: e4m3 raw slot -> scaled f16 tiles of the MMA slot
        const int ct = threadIdx.x - 192;
        const int KS = p.K / 128;  // scale blocks along K
        const int RS = p.a_rows_per_mat / 128;
        int rstage = 0, mstage = 0;
        uint32_t rphase = 0, mphase = 0;
        for (int u = blockIdx.x; u < total; u += gridDim.x) {
            const Unit t = decode_unit(p, pref, u);
            const bool routed = t.seg < p.E;
            const int mat = routed ? t.seg : t.seg - p.E;
            const float* sbase = (routed ? scale_routed : scale_shared) + (size_t)mat * RS * KS;
            const float* s_gate = sbase + (size_t)(t.mt) * KS;
            const float* s_up = sbase + (size_t)(p.a_up_offset / 128 + t.mt) * KS;
            // block scales relative to the tile's power of two
            const float inv_g = pow2f(-tile_exp(s_gate, KS, lane));
            const float inv_u = pow2f(-tile_exp(s_up, KS, lane));
            // the scales of K block j serve stages 2j and 2j+1; the next block's are
            // loaded two stages ahead so the load never stalls a conversion
            float g_cur = s_gate[0], u_cur = s_up[0];
            float g_nxt = KS > 1 ? s_gate[1] : 0.f, u_nxt = KS > 1 ? s_up[1] : 0.f;
            bool ok = true;
            for (int kb = 0; kb < KB; ++kb) {
                if (kb > 0 && (kb & 1) == 0) {
                    g_cur = g_nxt;
                    u_cur = u_nxt;
                    const int nj = (kb >> 1) + 1;
                    if (nj < KS) {
                        g_nxt = s_gate[nj];
                        u_nxt = s_up[nj];
                    }
                }
                const int h = kb & 1;  // half of the staged 128-K tile
                if (!mbar_wait(&m_empty[mstage], mphase ^ 1, abort_flag)) { ok = false; break; }
                if (h == 0 && !mbar_wait(&raw_full[rstage], rphase, abort_flag)) { ok = false; break; }
                uint8_t* ms = mring + mstage * C::MSLOT_BYTES;
                const uint8_t* rs = rring + rstage * C::RSLOT_BYTES;
                const __half2 m2[2] = {__float2half2_rn(g_cur * inv_g), __float2half2_rn(u_cur * inv_u)};
#pragma unroll
                for (int i = 0; i < C::NA * 512 / CVT_THREADS; ++i) {
                    const int task = ct + i * CVT_THREADS;
                    const int tile = (i * CVT_THREADS) >> 9;  // 512 tasks per tile, ct < CVT_THREADS
                    const int r = task & 127;
                    const int c = (task >> 7) & 3;
                    const uint8_t* src = rs + tile * C::A8_BYTES + r * 128 + (((4 * h + c) ^ (r & 7)) << 4);
                    uint8_t* dst = ms + C::CVT_OFF + tile * C::A_BYTES + r * 128;
                    uint4 lo, hi;
                    e4m3x16_to_f16_scaled(*reinterpret_cast<const uint4*>(src), m2[tile], lo, hi);
                    *reinterpret_cast<uint4*>(dst + (((2 * c) ^ (r & 7)) << 4)) = lo;
                    *reinterpret_cast<uint4*>(dst + (((2 * c + 1) ^ (r & 7)) << 4)) = hi;
                }
                if (h == 1) mbar_arrive(&raw_empty[rstage]);
                fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor core
                mbar_arrive(&cvt_full[mstage]);
                if (h == 1 && ++rstage == C::RSTAGES) { rstage = 0; rphase ^= 1; }
                if (++mstage == C::MSTAGES) { mstage = 0; mphase ^= 1; }
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


// ---------------------------------------------------------------- weights in TMEM
// tcgen05.mma can read its A operand from tensor memory (row i in lane i, two K
// elements per 32-bit column). In this variant the converter warps turn each
// E4M3 weight row into f16 values times m, as in the f16 path above, and store
// them there with tcgen05.st, so the converted tiles never cross shared memory.
// Per MMA stage that takes the converters' stores and the tensor core's A
// reads (32 KB each for gate/up, 16 KB for down) off the shared-memory traffic
// that bounds the shared-memory variant (for wide gate/up ~186 KB against ~128
// bytes per cycle per 960-cycle stage). TMEM holds the accumulators and two A
// stages:
//  * gate/up: gate and up accumulators (2 x 192 columns, single-buffered), A
//    stages of 64 columns (gate 32, up 32); converter warps 6..9 take gate
//    rows, 10..13 up rows, one thread per row.
//  * down (every tile width): two accumulators of up to 224 columns (double-
//    buffered), A stages of 32 columns; converter warps 6..9 take the first 32
//    K of a row, 10..13 the last 32. Its token rows are the f16 h rows (h times
//    2^-e, e per row), restored by the epilogue with the tile's 2^E.
// The staged E4M3 tiles span two MMA stages (128-byte rows); shared memory
// holds only those and the token tiles.

// D[tmem] (+)= A[tmem] * B[smem]^T, kind::f16.
__device__ __forceinline__ void mma_f16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Registers -> tensor memory: thread i of the warp writes r[0..31] to columns
// col..col+31 of lane (base lane + i).
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31]) : "memory");
}

// Gate/up epilogue of the f16 path, staged: as epilogue_f16_gate_up, but each
// 16-token chunk goes as bf16 into the group's shared [16 tokens][128
// features] tile (two, alternating), the group's four warps meet at an
// mbarrier, and warp q writes token rows 4q..4q+3 as 256 contiguous bytes
// each, 16 bytes per lane (scalar 2-byte stores had made the drain of the
// single accumulator stall the tensor cores).
template <int ACC_COLS, int GROUPS>
__device__ __forceinline__ void epilogue_f16_gate_up_staged(
    const KParams& p, const int* pref, int total, uint32_t tmem_base, uint64_t* tfull,
    uint64_t* tempty, volatile int* abort_flag, int warp, int lane, int group,
    const float* __restrict__ scale_routed, const float* __restrict__ scale_shared,
    const int8_t* __restrict__ row_exp, __nv_bfloat16* buf2, uint64_t* bar2) {
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int KS = p.K / 128;
    const int RS = p.a_rows_per_mat / 128;
    uint32_t acc_phase = 0;
    int chunk = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
        const Unit t = decode_unit(p, pref, u);
        const bool routed = t.seg < p.E;
        const int mat = routed ? t.seg : t.seg - p.E;
        const float* sbase = (routed ? scale_routed : scale_shared) + (size_t)mat * RS * KS;
        const float fg = pow2f(tile_exp(sbase + (size_t)t.mt * KS, KS, lane));
        const float fu = pow2f(tile_exp(sbase + (size_t)(p.a_up_offset / 128 + t.mt) * KS, KS, lane));
        if (!mbar_wait(&tfull[0], acc_phase, abort_flag)) break;
        tc_fence_after();
        const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16);
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(t.out) + t.mt * BM;
        const bool lim = p.swiglu_limit > 0.0f;  // optional limit: min(g, L), clamp(u, -L, L)
        const float L = p.swiglu_limit;
        for (int c0 = 16 * group; c0 < t.n_valid; c0 += 16 * GROUPS, ++chunk) {
            uint32_t g[16], uu[16];
            tmem_ld16(taddr + c0, g);
            tmem_ld16(taddr + ACC_COLS / 2 + c0, uu);
            // 2^e of this lane's token column (e in [-127, 114]; 2^-127 is subnormal)
            const int ex_l = (lane < 16 && c0 + lane < t.n_valid) ? row_exp[t.b_row + c0 + lane] : 0;
            const float fe_l = ex_l >= -126 ? pow2f(ex_l) : __uint_as_float(0x00400000u);
            tmem_ld_wait(g, uu);
            __nv_bfloat16* b = buf2 + (chunk & 1) * 16 * BM;
            // each step over all 16 token columns, branch-free, so that the
            // columns' exp / division chains overlap
            float a[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float fe = __shfl_sync(0xffffffffu, fe_l, j);
                const float g0 = __uint_as_float(g[j]) * fg * fe;  // exact power-of-two factors
                const float u0 = __uint_as_float(uu[j]) * fu * fe;
                const float gv = lim ? fminf(g0, L) : g0;
                const float uv = lim ? fminf(fmaxf(u0, -L), L) : u0;
                a[j] = __fdividef(gv, 1.0f + __expf(-gv)) * uv;
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) b[j * BM + row] = __float2bfloat16_rn(a[j]);
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar2[chunk & 1]);
            if (!mbar_wait(&bar2[chunk & 1], (uint32_t)(chunk >> 1) & 1u, abort_flag)) {
                ok = false;
                break;
            }
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                const int r = 4 * q + 2 * h2 + (lane >> 4);  // token row of the chunk
                const int col = (lane & 15) * 8;             // first of 8 features
                if (c0 + r < t.n_valid)
                    *reinterpret_cast<uint4*>(out + (size_t)(c0 + r) * p.ld_out + col) =
                        *reinterpret_cast<const uint4*>(b + r * BM + col);
            }
        }
        if (!ok) break;
        tc_fence_before();
        mbar_arrive(&tempty[0]);
        acc_phase ^= 1;
    }
}

template <int GEMM, int BNT_, int MST_>
struct TileTA {
    static constexpr int NA = (GEMM == 1) ? 2 : 1;
    static constexpr int EG = (GEMM == 1) ? 2 : 1;
    static constexpr int ACCB = (GEMM == 1) ? 1 : 2;
    static constexpr int BNT = BNT_;
    static constexpr int THREADS = 64 + 128 + CVT_THREADS + 32 + 128 * (EG - 1);  // warps as in TileF8
    static constexpr int RK = 2 * BK;                  // K of a staged e4m3 tile (two MMA stages)
    static constexpr int A8_BYTES = BM * RK;           // one staged tile, 128-byte rows
    static constexpr int RSLOT_BYTES = NA * A8_BYTES;
    static constexpr int B_BYTES = BNT * BK * 2;
    static constexpr int MSLOT_BYTES = (B_BYTES + 1023) / 1024 * 1024;
    static constexpr int MSTAGES = MST_;
    // gate/up: each epilogue group stages 16-token chunks of h, [2][16][128] bf16;
    // down: each epilogue warp its 16 x 32 chunks of y, [4 warps][2][16][32] bf16
    static constexpr int EPI_BYTES = (GEMM == 1 ? EG * 2 * 16 * BM * 2 : 4 * 2 * 16 * 32 * 2) + 128;
    static constexpr int FIXED_BYTES =
        1024 + 8 * (2 * 8 + 3 * MSTAGES + 5 + 2 * EG) + 16 + 4 * (MAX_SEG + 1) + EPI_BYTES;
    static constexpr int RSTAGES_FIT = (232448 - FIXED_BYTES - MSTAGES * MSLOT_BYTES) / RSLOT_BYTES;
    static constexpr int RSTAGES = RSTAGES_FIT < 8 ? RSTAGES_FIT : 8;
    static constexpr int ACC_COLS = NA * BNT;       // gate at 0, up at BNT (gate/up)
    static constexpr int A_COL = ACCB * ACC_COLS;   // A stage s at A_COL + s * A_STAGE_COLS
    static constexpr int A_STAGE_COLS = 32 * NA;    // 64 K of 16-bit values per weight tile
    static constexpr int TMEM_COLS = 512;
    // converted weight stages in tensor memory: as many as fit, up to the MMA ring's depth
    static constexpr int ASTAGES_FIT = (TMEM_COLS - A_COL) / A_STAGE_COLS;
    static constexpr int ASTAGES = ASTAGES_FIT < MST_ ? ASTAGES_FIT : MST_;
    static_assert(ASTAGES >= 2, "tensor memory budget");
    static constexpr int RING_BYTES = MSTAGES * MSLOT_BYTES + RSTAGES * RSLOT_BYTES;
    static constexpr int BAR_BYTES = 8 * (2 * RSTAGES + 3 * MSTAGES + 5 + 2 * EG) + 16;
    static constexpr int SMEM_BYTES = 1024 + RING_BYTES + BAR_BYTES + 4 * (MAX_SEG + 1) + EPI_BYTES;
    static_assert(RSTAGES >= 2 && MSTAGES >= 2 && SMEM_BYTES <= 232448, "shared memory budget");
};

// Registers -> tensor memory: thread i of the warp writes r[0..15] to columns
// col..col+15 of lane (base lane + i).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]) : "memory");
}

template <int GEMM, int BNT_, int MST_>
__global__ void __launch_bounds__(TileTA<GEMM, BNT_, MST_>::THREADS, 1)
    grouped_gemm_fp8w_ta_kernel(const __grid_constant__ CUtensorMap tmA_routed,
                                const __grid_constant__ CUtensorMap tmA_shared,
                                const __grid_constant__ BMaps tmB, const KParams p,
                                const float* __restrict__ scale_routed,
                                const float* __restrict__ scale_shared,
                                const int8_t* __restrict__ row_exp) {
    pdl_wait();
    pdl_trigger();
    using C = TileTA<GEMM, BNT_, MST_>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* mring = smem;                                // [MSTAGES][MSLOT_BYTES]: token tiles
    uint8_t* rring = smem + C::MSTAGES * C::MSLOT_BYTES;  // [RSTAGES][RSLOT_BYTES]: e4m3 tiles
    uint64_t* raw_full = reinterpret_cast<uint64_t*>(smem + C::RING_BYTES);
    uint64_t* raw_empty = raw_full + C::RSTAGES;
    uint64_t* b_full = raw_empty + C::RSTAGES;  // token tile landed
    uint64_t* cvt_full = b_full + C::MSTAGES;   // the stage's weight tiles are in their TMEM stage
    uint64_t* m_empty = cvt_full + C::MSTAGES;  // the stage's MMAs completed
    uint64_t* tfull = m_empty + C::MSTAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* mma_done = tempty + 2;
    uint64_t* ep_bar = mma_done + 1;  // [group][parity]: a gate/up epilogue group's staged chunk
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ep_bar + 2 * C::EG);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* pref = reinterpret_cast<int*>(tmem_slot + 4);
    __nv_bfloat16* ep_buf = reinterpret_cast<__nv_bfloat16*>(  // [group][2][16][128], 128-byte aligned
        (reinterpret_cast<uintptr_t>(pref + MAX_SEG + 1) + 127) & ~static_cast<uintptr_t>(127));

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::RSTAGES; ++s) {
            mbar_init(&raw_full[s], 1);
            mbar_init(&raw_empty[s], CVT_THREADS);
        }
        for (int s = 0; s < C::MSTAGES; ++s) {
            mbar_init(&b_full[s], 1);
            mbar_init(&cvt_full[s], CVT_THREADS);
            mbar_init(&m_empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 128 * C::EG);
        }
        mbar_init(mma_done, 1);
        for (int i = 0; i < 2 * C::EG; ++i) mbar_init(&ep_bar[i], 4);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmA_routed);
        tma_prefetch_desc(&tmA_shared);
        prefetch_bmaps(tmB);
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
        // producer: e4m3 weight tiles (gate and up, or one down tile; 128 K each) into the raw ring
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            for (int u = blockIdx.x; u < total && !*abort_flag; u += gridDim.x) {
                const Unit t = decode_unit(p, pref, u);
                const CUtensorMap* tmA = (t.seg < p.E) ? &tmA_routed : &tmA_shared;
                bool ok = true;
                for (int kr = 0; kr < KB / 2; ++kr) {
                    if (!mbar_wait(&raw_empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
                    uint8_t* rs = rring + stage * C::RSLOT_BYTES;
                    mbar_arrive_expect_tx(&raw_full[stage], C::RSLOT_BYTES);
                    tma_load_2d(rs, tmA, kr * C::RK, t.a_row, &raw_full[stage]);
                    if (GEMM == 1)
                        tma_load_2d(rs + C::A8_BYTES, tmA, kr * C::RK, t.a_row + p.a_up_offset,
                                    &raw_full[stage]);
                    ++issued;
                    if (++stage == C::RSTAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
            }
            if (*abort_flag) {
                int s = stage;
                uint32_t ph = phase;
                for (int i = 0; i < min(issued, C::RSTAGES); ++i) {
                    if (--s < 0) { s = C::RSTAGES - 1; ph ^= 1; }
                    volatile int no_abort = 0;
                    mbar_wait(&raw_full[s], ph, &no_abort);
                }
                status_or(p.status, MOE_DEV_TIMEOUT);
            }
        }
    } else if (warp == 1) {
        // MMA thread: A from the stage's TMEM columns, B from the token tile
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int g = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            for (int u = blockIdx.x; u < total; u += gridDim.x) {
                const Unit t = decode_unit(p, pref, u);
                const int n_mma = (t.n_valid + 15) & ~15;
                const uint32_t idesc = idesc_f16(BM, n_mma);
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1, abort_flag)) break;
                tc_fence_after();
                const uint32_t d0 = tmem_base + acc * C::ACC_COLS;
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb, ++g) {
                    if (!mbar_wait(&b_full[stage], phase, abort_flag) ||
                        !mbar_wait(&cvt_full[stage], phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a0 = tmem_base + C::A_COL + C::A_STAGE_COLS * (g % C::ASTAGES);
                    const uint32_t sb = smem_u32(mring + stage * C::MSLOT_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint32_t acc_flag = (kb | kk) != 0;
                        const uint64_t bd = sdesc_kmajor_sw128(sb + kk * 32);
                        mma_f16_tmem_a(d0, a0 + 8 * kk, bd, idesc, acc_flag);
                        if (GEMM == 1) mma_f16_tmem_a(d0 + C::BNT, a0 + 32 + 8 * kk, bd, idesc, acc_flag);
                    }
                    mma_commit(&m_empty[stage]);
                    if (++stage == C::MSTAGES) { stage = 0; phase ^= 1; }
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
    } else if (warp == B_WARP) {
        // token-tile loader: fills each slot's token tile as soon as it is free
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            for (int u = blockIdx.x; u < total && !*abort_flag; u += gridDim.x) {
                const Unit t = decode_unit(p, pref, u);
                const int n_mma = (t.n_valid + 15) & ~15;
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&m_empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
                    mbar_arrive_expect_tx(&b_full[stage], (uint32_t)(n_mma * BK * 2));
                    load_b_rows(mring + stage * C::MSLOT_BYTES, tmB, kb * BK, t.b_row, n_mma, BK * 2,
                                &b_full[stage]);
                    ++issued;
                    if (++stage == C::MSTAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
            }
            if (*abort_flag) {
                int s = stage;
                uint32_t ph = phase;
                for (int i = 0; i < min(issued, C::MSTAGES); ++i) {
                    if (--s < 0) { s = C::MSTAGES - 1; ph ^= 1; }
                    volatile int no_abort = 0;
                    mbar_wait(&b_full[s], ph, &no_abort);
                }
            }
        }
    } else if (warp < 6 || warp >= EPI2_WARP) {
        if (GEMM == 1) {
            const int grp = warp < 6 ? 0 : 1;
            epilogue_f16_gate_up_staged<C::ACC_COLS, C::EG>(
                p, pref, total, tmem_base, tfull, tempty, abort_flag, warp, lane, grp, scale_routed,
                scale_shared, row_exp, ep_buf + grp * 2 * 16 * BM, ep_bar + 2 * grp);
        }
        else
            epilogue_f16_down<C::ACC_COLS, C::ACCB>(p, pref, total, tmem_base, tfull, tempty, abort_flag,
                                                    warp, lane, scale_routed, scale_shared, row_exp,
                                                    ep_buf + (warp & 3) * 2 * 16 * 32);
    } else {
        // converters, thread = one weight row of its lane quadrant. gate/up: warps
        // 6..9 gate rows, 10..13 up rows, 64 K each; down: warps 6..9 the first
        // 32 K of a row, 10..13 the last 32. The TMEM stage of MMA stage g was
        // last read by stage g - ASTAGES, whose completion (its slot's empty
        // barrier) is awaited first.
        const int tile = (warp - 6) >> 2;  // gate/up: which tile; down: which half of the row
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lane_cols = tmem_base + ((uint32_t)((warp & 3) * 32) << 16) + C::A_COL +
                                   (GEMM == 1 ? 32 : 16) * tile;
        const int KS = p.K / 128;  // scale blocks along K
        const int RS = p.a_rows_per_mat / 128;
        int rstage = 0, mstage = 0, g = 0;
        uint32_t rphase = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
            const Unit t = decode_unit(p, pref, u);
            const bool routed = t.seg < p.E;
            const int mat = routed ? t.seg : t.seg - p.E;
            const float* sbase = (routed ? scale_routed : scale_shared) + (size_t)mat * RS * KS;
            const float* srow =
                sbase + (size_t)((GEMM == 1 && tile == 1) ? p.a_up_offset / 128 + t.mt : t.mt) * KS;
            // block scales relative to the tile's power of two. The scale of K
            // block j serves stages 2j and 2j+1, the next one is loaded ahead
            const float inv = pow2f(-tile_exp(srow, KS, lane));
            float s_cur = srow[0];
            float s_nxt = KS > 1 ? srow[1] : 0.f;
            for (int kb = 0; kb < KB; ++kb, ++g) {
                if (kb > 0 && (kb & 1) == 0) {
                    s_cur = s_nxt;
                    const int nj = (kb >> 1) + 1;
                    if (nj < KS) s_nxt = srow[nj];
                }
                const int h = kb & 1;  // half of the staged 128-K tile
                if (h == 0 && !mbar_wait(&raw_full[rstage], rphase, abort_flag)) { ok = false; break; }
                if (g >= C::ASTAGES) {
                    const int gp = g - C::ASTAGES;
                    if (!mbar_wait(&m_empty[gp % C::MSTAGES], (uint32_t)(gp / C::MSTAGES) & 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                }
                tc_fence_after();
                const __half2 m2 = __float2half2_rn(s_cur * inv);
                if (GEMM == 1) {
                    const uint8_t* src = rring + rstage * C::RSLOT_BYTES + tile * C::A8_BYTES + row * 128;
                    uint32_t v[32];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint4 lo, hi;
                        e4m3x16_to_f16_scaled(
                            *reinterpret_cast<const uint4*>(src + (((4 * h + c) ^ (row & 7)) << 4)), m2, lo, hi);
                        v[8 * c + 0] = lo.x; v[8 * c + 1] = lo.y; v[8 * c + 2] = lo.z; v[8 * c + 3] = lo.w;
                        v[8 * c + 4] = hi.x; v[8 * c + 5] = hi.y; v[8 * c + 6] = hi.z; v[8 * c + 7] = hi.w;
                    }
                    if (h == 1) mbar_arrive(&raw_empty[rstage]);
                    tmem_st32(lane_cols + C::A_STAGE_COLS * (g % C::ASTAGES), v);
                } else {
                    const uint8_t* src = rring + rstage * C::RSLOT_BYTES + row * 128;
                    uint32_t v[16];
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        const int c = 2 * tile + i;  // 16-K chunk of the stage
                        uint4 lo, hi;
                        e4m3x16_to_f16_scaled(
                            *reinterpret_cast<const uint4*>(src + (((4 * h + c) ^ (row & 7)) << 4)), m2, lo, hi);
                        v[8 * i + 0] = lo.x; v[8 * i + 1] = lo.y; v[8 * i + 2] = lo.z; v[8 * i + 3] = lo.w;
                        v[8 * i + 4] = hi.x; v[8 * i + 5] = hi.y; v[8 * i + 6] = hi.z; v[8 * i + 7] = hi.w;
                    }
                    if (h == 1) mbar_arrive(&raw_empty[rstage]);
                    tmem_st16(lane_cols + C::A_STAGE_COLS * (g % C::ASTAGES), v);
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&cvt_full[mstage]);
                if (h == 1 && ++rstage == C::RSTAGES) { rstage = 0; rphase ^= 1; }
                if (++mstage == C::MSTAGES) mstage = 0;
            }
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

template <int GEMM, int BNF_, int ACCB_, int MST_>
cudaError_t launch_fp8w(const GroupedGemmArgs& a, cudaStream_t st) {
    using C = TileF8<GEMM, BNF_, ACCB_, MST_>;
    const cudaError_t attr_err = ensure_smem_limit(
        reinterpret_cast<const void*>(grouped_gemm_fp8w_kernel<GEMM, BNF_, ACCB_, MST_>), C::SMEM_BYTES);
    if (attr_err != cudaSuccess) return attr_err;
    uint64_t b_rows;
    KParams p = make_params(a, GEMM, &b_rows);
    p.bn = C::BNF;
    CUtensorMap tmAr, tmAs;
    BMaps tmB;
    const int S = a.S;
    if (!make_tmap_2d(&tmAr, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.w_routed, (uint64_t)a.E * p.a_rows_per_mat,
                      p.K, p.K, C::RK, BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_2d(&tmAs, CU_TENSOR_MAP_DATA_TYPE_UINT8, S > 0 ? a.w_shared : a.w_routed,
                      (uint64_t)(S > 0 ? S : a.E) * p.a_rows_per_mat, p.K, p.K, C::RK, BM,
                      CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (b_rows == 0) return cudaSuccess;
    // f16 token rows (x * 2^-e)
    if (!make_bmaps(&tmB, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.b_rows, b_rows, p.K, BK))
        return cudaErrorInvalidValue;
    launch_pdl(grouped_gemm_fp8w_kernel<GEMM, BNF_, ACCB_, MST_>, grid_for(p), C::THREADS,
        C::SMEM_BYTES, st, tmAr, tmAs, tmB, p, static_cast<const float*>(a.w_routed_scale),
        static_cast<const float*>(S > 0 ? a.w_shared_scale : a.w_routed_scale), reinterpret_cast<const int8_t*>(a.b_scale));
    return cudaGetLastError();
}

template <int GEMM, int BNT_, int MST_>
cudaError_t launch_fp8w_ta(const GroupedGemmArgs& a, cudaStream_t st) {
    using C = TileTA<GEMM, BNT_, MST_>;
    const cudaError_t attr_err = ensure_smem_limit(
        reinterpret_cast<const void*>(grouped_gemm_fp8w_ta_kernel<GEMM, BNT_, MST_>), C::SMEM_BYTES);
    if (attr_err != cudaSuccess) return attr_err;
    uint64_t b_rows;
    KParams p = make_params(a, GEMM, &b_rows);
    p.bn = C::BNT;
    CUtensorMap tmAr, tmAs;
    BMaps tmB;
    const int S = a.S;
    if (!make_tmap_2d(&tmAr, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.w_routed, (uint64_t)a.E * p.a_rows_per_mat,
                      p.K, p.K, C::RK, BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_2d(&tmAs, CU_TENSOR_MAP_DATA_TYPE_UINT8, S > 0 ? a.w_shared : a.w_routed,
                      (uint64_t)(S > 0 ? S : a.E) * p.a_rows_per_mat, p.K, p.K, C::RK, BM,
                      CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (b_rows == 0) return cudaSuccess;
    // f16 rows: token rows x * 2^-e (gate/up), SwiGLU output rows h * 2^-e (down)
    if (!make_bmaps(&tmB, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.b_rows, b_rows, p.K, BK))
        return cudaErrorInvalidValue;
    launch_pdl(grouped_gemm_fp8w_ta_kernel<GEMM, BNT_, MST_>, grid_for(p), C::THREADS,
        C::SMEM_BYTES, st, tmAr, tmAs, tmB, p, static_cast<const float*>(a.w_routed_scale),
        static_cast<const float*>(S > 0 ? a.w_shared_scale : a.w_routed_scale), reinterpret_cast<const int8_t*>(a.b_scale));
    return cudaGetLastError();
}

cudaError_t launch_gemm_fp8w(const GroupedGemmArgs& a, cudaStream_t st) {
    // many tokens per expert: wide token tiles (each weight tile converted once
    // per expert); few tokens per expert: narrower double-buffered tiles. The
    // last argument is the MMA-ring depth; the raw ring takes the rest of
    // shared memory (up to 8 slots of two MMA stages each).
    // Wide tiles run the variant with the weight tiles in tensor memory
    // (gate/up: 192-token tiles, down: 224; four token slots).
    const bool wide = a.N >= 128L * a.E;
    if (a.gemm == 1)
        return wide ? launch_fp8w_ta<1, 192, 4>(a, st) : launch_fp8w<1, 128, 2, 3>(a, st);
    return wide ? launch_fp8w_ta<2, 224, 4>(a, st) : launch_fp8w_ta<2, 128, 4>(a, st);
}

}  // namespace gemm
}  // namespace moe
