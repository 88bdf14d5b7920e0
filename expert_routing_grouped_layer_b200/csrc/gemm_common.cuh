// gemm_common.cuh -- pieces shared by the grouped expert GEMM kernels: tile
// constants, the device-side ragged tile schedule, the bf16 epilogue, and the
// host helpers that build TMA descriptors and launch geometry.
#pragma once

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
namespace gemm {


constexpr int BM = 128;   // weight rows per tile (MMA M)
constexpr int BN = 128;   // max tokens per tile (MMA N)
constexpr int BK = 64;    // bf16 elements in one 128-byte swizzled row
constexpr int B_BOX = 16; // token rows per TMA box
constexpr int MAX_SEG = 1024 + 4;

// NA_: weight tiles per stage sharing the token tile (GEMM1: gate and up;
// GEMM2: one 128-row block, or two consecutive ones)
template <int GEMM, int NA_ = (GEMM == 1 ? 2 : 1)>
struct Tile {
    static constexpr int NA = NA_;
    static constexpr int A_BYTES = BM * BK * 2;
    static constexpr int B_BYTES = BN * BK * 2;
    static constexpr int STAGE_BYTES = NA * A_BYTES + B_BYTES;
    static constexpr int STAGES = (NA == 2) ? 4 : 6;
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
    int a_up_offset;     // row offset of a unit's second weight tile (GEMM1: I, the up projection)
    int tile_rows;       // weight rows (output features) per tile unit
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
    float swiglu_limit;   // gate/up: 0 = off, else clamp g from above and u to +-limit
};

// SwiGLU with the optional limit: SiLU(min(g, L)) * clamp(u, -L, L) for L > 0.
__device__ __forceinline__ float swiglu(float g, float u, float limit) {
    if (limit > 0.0f) {
        g = fminf(g, limit);
        u = fminf(fmaxf(u, -limit), limit);
    }
    return g / (1.0f + __expf(-g)) * u;
}

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
        t.a_row = lo * p.a_rows_per_mat + t.mt * p.tile_rows;
        r0 = (size_t)p.offsets[lo] + nt * p.bn;
        t.b_row = (int)r0;
        out = p.out_routed;
        sc = p.sc_routed;
    } else {
        const int s = lo - p.E;
        t.a_row = s * p.a_rows_per_mat + t.mt * p.tile_rows;
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
// GEMM2 units may hold ND consecutive 128-row blocks (accumulators BN columns
// apart).
template <int GEMM, int ACC_COLS, int ACCB = 2, int ND = 1>
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
        const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + acc * ACC_COLS;
#pragma unroll 1
        for (int w = 0; w < (GEMM == 1 ? 1 : ND); ++w) {
        const uint32_t taddr = tbase + w * BN;
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(t.out) + t.mt * p.tile_rows + w * BM + row;
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
                        const float a =
                            swiglu(__uint_as_float(g[j]), __uint_as_float(uu[j]), p.swiglu_limit);
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
        }
        tc_fence_before();
        mbar_arrive(&tempty[acc]);
        if (++acc == ACCB) { acc = 0; acc_phase ^= 1; }
    }
}

// Token rows of the B operand are fetched with tensor maps whose boxes are
// 16, 32, 64 and 128 rows high: a tile of n rows (n a multiple of 16, below
// 256) takes one copy per set bit of n / 16, largest first, so every copy
// starts on a 16-row (2 KB for 128-byte rows) boundary of the swizzled tile.
// One TMA instruction per 16 rows kept the single producer thread busy for
// longer than the tensor cores needed per stage.
constexpr int B_HEIGHTS = 4;
struct BMaps {
    CUtensorMap m[B_HEIGHTS];  // m[i]: box of 16 << i rows
};

__device__ __forceinline__ void prefetch_bmaps(const BMaps& bm) {
#pragma unroll
    for (int i = 0; i < B_HEIGHTS; ++i) tma_prefetch_desc(&bm.m[i]);
}

__device__ __forceinline__ void load_b_rows(uint8_t* dst, const BMaps& bm, int x, int row, int n,
                                            int row_bytes, uint64_t* bar) {
    const int blocks = n >> 4;
    int off = 0;
#pragma unroll
    for (int i = B_HEIGHTS - 1; i >= 0; --i) {
        if ((blocks >> i) & 1) {
            tma_load_2d(dst + off * row_bytes, &bm.m[i], x, row + off, bar);
            off += 16 << i;
        }
    }
}

// Pipeline depth that fits the shared-memory budget (at most `cap` stages).
constexpr int stages_for(int stage_bytes, int fixed_bytes, int cap) {
    return ((232448 - fixed_bytes) / stage_bytes) < cap ? ((232448 - fixed_bytes) / stage_bytes) : cap;
}


// ---------------------------------------------------------------- host helpers
inline PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
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
inline bool make_tmap_bf16(CUtensorMap* tm, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
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

// The four B maps of one row-major tensor [rows][cols] of esize-byte elements,
// box = box_x elements x (16 << i) rows, 128-byte swizzle.
inline bool make_bmaps(BMaps* bm, CUtensorMapDataType dtype, int esize, const void* ptr,
                       uint64_t rows, uint64_t cols, uint32_t box_x) {
    auto enc = get_encode();
    if (!enc) return false;
    for (int i = 0; i < B_HEIGHTS; ++i) {
        cuuint64_t dims[2] = {cols, rows};
        cuuint64_t strides[1] = {cols * (uint64_t)esize};
        cuuint32_t box[2] = {box_x, (cuuint32_t)(16 << i)};
        cuuint32_t estr[2] = {1, 1};
        CUresult r = enc(&bm->m[i], dtype, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return false;
    }
    return true;
}

// Problem geometry shared by every variant of the two GEMMs.
inline KParams make_params(const GroupedGemmArgs& a, int GEMM, uint64_t* b_rows) {
    KParams p;
    p.nseg = a.E + a.S;
    p.E = a.E;
    p.S = a.S;
    p.T = a.T;
    p.N = a.N;
    p.offsets = a.offsets;
    p.status = a.status;
    p.swiglu_limit = a.swiglu_limit;
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
    p.tile_rows = BM;
    p.out_routed = static_cast<uint8_t*>(a.out_routed);
    p.out_shared = static_cast<uint8_t*>(a.out_shared);
    p.out_esize = 2;
    p.sc_routed = p.sc_shared = nullptr;
    return p;
}

inline int grid_for(const KParams& p) {
    // upper bound on tiles: sum_e ceil(m_e/BN) <= N/BN + min(E, N), plus shared
    const long MT = p.M / p.tile_rows;
    const long routed_tiles = (long)p.N / p.bn + std::min<long>(p.E, p.N);
    const long shared_tiles = (long)p.S * ((p.T + p.bn - 1) / p.bn);
    const long units_max = (routed_tiles + shared_tiles) * MT;
    return (int)std::max<long>(1, std::min<long>(num_sms(), units_max));
}


// 2-D tensor map helper: `dtype` elements, rows x cols, box_cols x box_rows.
inline bool make_tmap_2d(CUtensorMap* tm, CUtensorMapDataType dtype, const void* ptr, uint64_t rows,
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


}  // namespace gemm
}  // namespace moe
