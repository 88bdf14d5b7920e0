// router_tc.cu -- router logits on the tcgen05 tensor cores with fp32 accuracy.
//
// "DeepSeek V3架构拆解：Kimi-K2-Thinking-NVFP4的MLA注意力与MoE路由实现原理", 三.1 打分:
// logits = x . Wg^T with an fp32 router weight and fp32 arithmetic. The bf16
// input x is exact in bf16; the fp32 weight is split exactly enough into three
// bf16 planes, Wg = hi + mid + lo (hi = bf16(Wg), mid = bf16(Wg - hi),
// lo = bf16(Wg - hi - mid): 24 significand bits), and the MMAs accumulate
// x.hi + x.mid + x.lo. Every product of two bf16 values is exact in fp32.
//
// Accumulating a whole 7168-wide row in one tensor-memory accumulator (1344
// MMAs) measured errors that grow with the number of MMAs and lean one way:
// the largest logits of the 896-expert layer came out up to 1.8e-4 low
// (4e-5 rms), enough to reorder experts whose scores differ by 1e-5. Here each
// 64-wide k-block is accumulated afresh (12 MMAs) in one of four tensor-memory
// accumulators, and the epilogue warps add the k-blocks' fp32 partial sums
// with Kahan's compensated summation (packed fp32x2 arithmetic, two token
// columns per instruction), so only 12 MMAs' accumulation error
// enters per k-block, with signs that vary across k-blocks, plus one rounding
// of the final value (measured: 2.1e-6 at most, as with fp64 sums, which cost
// the 896-expert router 0.5 ms in conversions; plain fp32 sums doubled the
// largest error).
//
// Layout: experts are the MMA M operand (128 per tile, the three planes of the
// same 128 experts are three A tiles of one stage), tokens are N (<= 128).
// Small batches split K across CTAs; partial sums go to part[split][T][E] and a
// reduction kernel adds them in split order in fp64 (deterministic).
#include "gemm_common.cuh"

namespace moe {
namespace {

using gemm::BK;
using gemm::BM;
using gemm::BMaps;

constexpr int RT_BN = 128;
constexpr int RT_STAGES = 3;
constexpr int RT_A_BYTES = BM * BK * 2;
constexpr int RT_B_BYTES = RT_BN * BK * 2;
constexpr int RT_STAGE_BYTES = 3 * RT_A_BYTES + RT_B_BYTES;
constexpr int RT_ACCS = 4;  // accumulator buffers (one k-block each)
constexpr int RT_TMEM_COLS = RT_ACCS * RT_BN;
constexpr int RT_SMEM_BYTES = 1024 + RT_STAGES * RT_STAGE_BYTES + 8 * (2 * RT_STAGES + 2 * RT_ACCS + 1) + 16;
constexpr int RT_EPI_WARPS = 8;  // two per TMEM lane quadrant, each 64 token columns
constexpr int RT_THREADS = 64 + 32 * RT_EPI_WARPS;

struct RouterParams {
    int T, E, Epad, H;
    int mtiles, ntiles, ksplit, kbps;  // k-blocks of 64 per split
    float* part;
    int32_t* status;
};

struct RUnit {
    int mt, ks, t0, n_valid, kb0, kb1;
};

__device__ __forceinline__ RUnit router_unit(const RouterParams& p, int u) {
    RUnit r;
    r.ks = u % p.ksplit;
    const int tile = u / p.ksplit;
    r.mt = tile % p.mtiles;
    const int nt = tile / p.mtiles;
    r.t0 = nt * RT_BN;
    r.n_valid = min(RT_BN, p.T - r.t0);
    r.kb0 = r.ks * p.kbps;
    r.kb1 = min(p.H / BK, r.kb0 + p.kbps);
    return r;
}

// One 3-D box: the same 128 x 64 tile of the three weight planes, planes outermost.
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const void* tmap, int32_t x, int32_t y,
                                            int32_t z, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

// hi / mid / lo bf16 planes of the fp32 router weight, rows padded to Epad with
// zeros. Eight consecutive weights per thread (H is a multiple of 64, so the eight
// share a row): two 16-byte loads and one 16-byte store per plane. Element i of
// [Epad][H] is a real weight exactly when i < E*H, so the padding needs no divide.
__device__ __forceinline__ uint32_t pack_bf16x2(__nv_bfloat16 a, __nv_bfloat16 b) {
    return (uint32_t)__bfloat16_as_ushort(a) | ((uint32_t)__bfloat16_as_ushort(b) << 16);
}

__global__ void __launch_bounds__(256) router_split_kernel(const float4* __restrict__ wg,
                                                           uint4* __restrict__ planes,
                                                           long n_valid8, long n8) {
    pdl_wait();
    pdl_trigger();
    for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n8;
         i += (long)gridDim.x * blockDim.x) {
        float w[8];
        if (i < n_valid8) {
            const float4 a = wg[2 * i], b = wg[2 * i + 1];
            w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
            w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) w[j] = 0.0f;
        }
        uint32_t hi[4], mid[4], lo[4];
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
            __nv_bfloat16 h[2], m[2], l[2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                h[q] = __float2bfloat16_rn(w[j + q]);
                const float r1 = w[j + q] - __bfloat162float(h[q]);
                m[q] = __float2bfloat16_rn(r1);
                l[q] = __float2bfloat16_rn(r1 - __bfloat162float(m[q]));
            }
            hi[j / 2] = pack_bf16x2(h[0], h[1]);
            mid[j / 2] = pack_bf16x2(m[0], m[1]);
            lo[j / 2] = pack_bf16x2(l[0], l[1]);
        }
        planes[i] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        planes[n8 + i] = make_uint4(mid[0], mid[1], mid[2], mid[3]);
        planes[2 * n8 + i] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
}

__global__ void __launch_bounds__(RT_THREADS, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ BMaps tmX,
                     const RouterParams p) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + RT_STAGES * RT_STAGE_BYTES);
    uint64_t* empty = full + RT_STAGES;
    uint64_t* tfull = empty + RT_STAGES;
    uint64_t* tempty = tfull + RT_ACCS;
    uint64_t* mma_done = tempty + RT_ACCS;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < RT_STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < RT_ACCS; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 32 * RT_EPI_WARPS);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmW);
        gemm::prefetch_bmaps(tmX);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, RT_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int total = p.mtiles * p.ntiles * p.ksplit;

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            for (int u = blockIdx.x; u < total && !*abort_flag; u += gridDim.x) {
                const RUnit r = router_unit(p, u);
                const int n16 = (r.n_valid + 15) & ~15;
                const uint32_t tx = 3 * RT_A_BYTES + n16 * BK * 2;
                bool ok = true;
                for (int kb = r.kb0; kb < r.kb1; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
                    uint8_t* st = smem + stage * RT_STAGE_BYTES;
                    mbar_arrive_expect_tx(&full[stage], tx);
                    tma_load_3d(st, &tmW, kb * BK, r.mt * BM, 0, &full[stage]);
                    gemm::load_b_rows(st + 3 * RT_A_BYTES, tmX, kb * BK, r.t0, n16, BK * 2,
                                      &full[stage]);
                    ++issued;
                    if (++stage == RT_STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
            }
            if (*abort_flag) {
                int s = stage;
                uint32_t ph = phase;
                for (int i = 0; i < min(issued, RT_STAGES); ++i) {
                    if (--s < 0) { s = RT_STAGES - 1; ph ^= 1; }
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
            bool ok = true;
            for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
                const RUnit r = router_unit(p, u);
                const uint32_t idesc = idesc_bf16(BM, (r.n_valid + 15) & ~15);
                for (int kb = r.kb0; kb < r.kb1; ++kb) {
                    // a fresh accumulator per k-block: the epilogue promotes it to fp64
                    if (!mbar_wait(&tempty[acc], acc_phase ^ 1, abort_flag)) { ok = false; break; }
                    if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t d = tmem_base + acc * RT_BN;
                    const uint32_t st = smem_u32(smem + stage * RT_STAGE_BYTES);
                    const uint32_t sb = st + 3 * RT_A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint64_t bd = sdesc_kmajor_sw128(sb + kk * 32);
#pragma unroll
                        for (int pl = 0; pl < 3; ++pl)
                            mma_bf16(d, sdesc_kmajor_sw128(st + pl * RT_A_BYTES + kk * 32), bd, idesc,
                                     (kk != 0 || pl != 0) ? 1u : 0u);
                    }
                    mma_commit(&empty[stage]);
                    mma_commit(&tfull[acc]);
                    if (++stage == RT_STAGES) { stage = 0; phase ^= 1; }
                    if (++acc == RT_ACCS) { acc = 0; acc_phase ^= 1; }
                }
            }
            mma_commit(mma_done);
            volatile int no_abort = 0;
            mbar_wait(mma_done, 0, &no_abort);
            if (*abort_flag) status_or(p.status, MOE_DEV_TIMEOUT);
        }
    } else {
        // epilogue: warp w reads TMEM lane quadrant w % 4 (experts 32*(w%4) ..) and
        // token columns 64*h .. 64*h+63 of each k-block's accumulator, adding them
        // into Kahan-compensated fp32 sums; the unit's sum is rounded once
        const int q = warp & 3;
        const int h = (warp - 2) >> 2;
        const int e = q * 32 + lane;  // expert within the M tile
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
            const RUnit r = router_unit(p, u);
            // Kahan sums of two token columns at a time (packed fp32x2 arithmetic)
            float2 sum[32], comp[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                sum[j] = make_float2(0.0f, 0.0f);
                comp[j] = make_float2(0.0f, 0.0f);
            }
            const float2 neg1 = make_float2(-1.0f, -1.0f);
            for (int kb = r.kb0; kb < r.kb1; ++kb) {
                if (!mbar_wait(&tfull[acc], acc_phase, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t taddr =
                    tmem_base + ((uint32_t)(q * 32) << 16) + acc * RT_BN + (uint32_t)(h * 64);
#pragma unroll
                for (int c0 = 0; c0 < 64; c0 += 16) {
                    if (h * 64 + c0 < r.n_valid) {  // warp-uniform
                        uint32_t v[16];
                        tmem_ld16(taddr + c0, v);
                        tmem_ld_wait(v);
#pragma unroll
                        for (int j = 0; j < 8; ++j) {  // Kahan: comp carries the lost low part
                            const int i = c0 / 2 + j;
                            const float2 x = make_float2(__uint_as_float(v[2 * j]),
                                                         __uint_as_float(v[2 * j + 1]));
                            const float2 y = __ffma2_rn(comp[i], neg1, x);     // x - comp
                            const float2 t = __fadd2_rn(sum[i], y);            // sum + y
                            comp[i] = __ffma2_rn(y, neg1, __ffma2_rn(sum[i], neg1, t));  // (t - sum) - y
                            sum[i] = t;
                        }
                    }
                }
                tc_fence_before();
                mbar_arrive(&tempty[acc]);
                if (++acc == RT_ACCS) { acc = 0; acc_phase ^= 1; }
            }
            if (!ok) break;
            const int eg = r.mt * BM + e;
            if (eg < p.E) {
                float* out = p.part + ((size_t)r.ks * p.T + r.t0) * p.E + eg;
#pragma unroll
                for (int j = 0; j < 64; ++j) {
                    const float hi = (j & 1) ? sum[j / 2].y : sum[j / 2].x;
                    const float lo = (j & 1) ? comp[j / 2].y : comp[j / 2].x;
                    if (h * 64 + j < r.n_valid) out[(size_t)(h * 64 + j) * p.E] = hi - lo;
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem_base, RT_TMEM_COLS);
    }
}

}  // namespace

// The three planes [3][Epad][H] as a 3-D tensor: box 64 columns x 128 rows x 3
// planes, 128-byte swizzle, so one copy fills the three A tiles of a stage.
static bool make_tmap_planes(CUtensorMap* tm, const void* planes, uint64_t Epad, uint64_t H) {
    auto enc = gemm::get_encode();
    if (!enc) return false;
    cuuint64_t dims[3] = {H, Epad, 3};
    cuuint64_t strides[2] = {H * 2, Epad * H * 2};
    cuuint32_t box[3] = {(cuuint32_t)BK, (cuuint32_t)BM, 3};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(planes), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// K splits: the count that minimises the estimated time, (waves of units) x
// (k-blocks per unit) plus the partial-sum slabs' round trip through memory
// (T x E x 8 bytes per split, costed at ~4 MB per k-block time: measured, two
// splits of the 16384-token, 896-expert router were 5% slower than one). Units of one split are equally long, so a grid a little above a
// multiple of the SM count pays a whole extra wave: splitting the 8192-token,
// 384-expert router into three gives four waves of a third as long instead of
// two full ones. At least 4 k-blocks per split; a plan depends on (T, E, H) and
// the SM count only.
RouterPlan router_plan(int T, int E, int H) {
    RouterPlan r;
    r.Epad = (E + BM - 1) / BM * BM;
    const int KB = H / BK;
    const long base = (long)(r.Epad / BM) * ((T + RT_BN - 1) / RT_BN);
    const long sms = num_sms();
    const double slab_kb = (double)T * E * 8.0 / 4.0e6;  // one split's slab round trip, in k-block times
    int best = 1;
    double best_cost = 1e300;
    for (int s = 1; s <= std::max(1, KB / 4); ++s) {
        const int kbps = (KB + s - 1) / s;
        const int splits = (KB + kbps - 1) / kbps;
        if (splits != s) continue;  // same plan as a smaller count
        const long waves = (base * s + sms - 1) / sms;
        const double cost = (double)waves * kbps + (s > 1 ? s * slab_kb : 0.0);
        if (cost < best_cost - 1e-9) { best_cost = cost; best = s; }
    }
    r.kbps = (KB + best - 1) / best;
    r.splits = (KB + r.kbps - 1) / r.kbps;  // no empty split
    return r;
}

cudaError_t launch_router_tc(const void* x, const float* gate_w, void* planes, float* part, int T,
                             int E, int H, int32_t* status, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const cudaError_t attr_err =
        ensure_smem_limit(reinterpret_cast<const void*>(router_tc_kernel), RT_SMEM_BYTES);
    if (attr_err != cudaSuccess) return attr_err;
    const RouterPlan plan = router_plan(T, E, H);
    const long n = (long)plan.Epad * H;
    const long n8 = n / 8;
    launch_pdl(router_split_kernel, (unsigned)std::min<long>((n8 + 255) / 256, 8L * num_sms()), 256,
        0, st, reinterpret_cast<const float4*>(gate_w), static_cast<uint4*>(planes),
        (long)E * H / 8, n8);
    CUtensorMap tmW;
    BMaps tmX;
    if (!make_tmap_planes(&tmW, planes, plan.Epad, H) ||
        !gemm::make_bmaps(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, (uint64_t)T, H, BK))
        return cudaErrorInvalidValue;
    RouterParams p;
    p.T = T;
    p.E = E;
    p.Epad = plan.Epad;
    p.H = H;
    p.mtiles = plan.Epad / BM;
    p.ntiles = (T + RT_BN - 1) / RT_BN;
    p.ksplit = plan.splits;
    p.kbps = plan.kbps;
    p.part = part;
    p.status = status;
    const int units = p.mtiles * p.ntiles * p.ksplit;
    launch_pdl(router_tc_kernel, std::min(units, num_sms()), RT_THREADS, RT_SMEM_BYTES, st, tmW, tmX,
        p);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess && plan.splits > 1) e = launch_router_reduce(part, (long)T * E, plan.splits, st);
    return e;
}

}  // namespace moe
