// permute.cu -- dispatch permutation ("DeepSeek V3架构拆解：Kimi-K2-Thinking-NVFP4的MLA注意力与
// MoE路由实现原理", 三.4 推理执行: count each expert's tokens, argsort the tokens by
// expert id into contiguous blocks).
//
// Deterministic stable counting sort of the N = T*k (token, slot) pairs by
// expert id, in three launches without atomics on the output order (one
// launch doing all three steps when the pairs fit one chunk):
//   1. count:   per chunk of PERM_CHUNK pairs, a per-expert histogram;
//   2. scan:    expert totals -> expert_offsets, and each chunk's starting row
//               per expert (exclusive prefix over chunks);
//   3. scatter: inside a chunk each warp owns a contiguous slice; warp bases
//               come from per-warp histograms, and inside a warp the rank of a
//               pair among equal experts is the count of lower lanes matching
//               it (__match_any_sync), so pairs keep ascending order.
#include <mutex>

#include "internal.h"
#include "sm100.cuh"

namespace moe {

namespace {

constexpr int PERM_WARPS = 8;
constexpr int PERM_PER_WARP = 512;
constexpr int PERM_CHUNK = PERM_WARPS * PERM_PER_WARP;
constexpr int PERM_MAX_E = 1024;

__global__ void __launch_bounds__(256) perm_count_kernel(const int32_t* __restrict__ idx, long N,
                                                         int E, int32_t* __restrict__ chunk,
                                                         int32_t* status) {
    pdl_wait();
    pdl_trigger();
    __shared__ int32_t cnt[PERM_MAX_E];
    for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    const long base = (long)blockIdx.x * PERM_CHUNK;
    bool bad = false;
    for (int i = threadIdx.x; i < PERM_CHUNK; i += blockDim.x) {
        const long p = base + i;
        if (p >= N) break;
        const int e = idx[p];
        if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
        else bad = true;
    }
    if (bad) status_or(status, MOE_DEV_BAD_EXPERT);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) chunk[(size_t)blockIdx.x * E + e] = cnt[e];
}

// Single CTA of 1024 threads; thread e owns expert e.
__global__ void __launch_bounds__(1024) perm_scan_kernel(int32_t* __restrict__ chunk, int n_chunks,
                                                         int E, int32_t* __restrict__ offsets) {
    pdl_wait();
    pdl_trigger();
    __shared__ int32_t warp_sums[32];
    const int e = threadIdx.x;
    int total = 0;
    if (e < E)
        for (int c = 0; c < n_chunks; ++c) total += chunk[(size_t)c * E + e];
    // block exclusive scan of totals over experts
    const int lane = e & 31, wid = e >> 5;
    int v = total;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += o;
    }
    if (lane == 31) warp_sums[wid] = v;
    __syncthreads();
    if (wid == 0) {
        int s = warp_sums[lane];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, s, off);
            if (lane >= off) s += o;
        }
        warp_sums[lane] = s;  // inclusive over warps
    }
    __syncthreads();
    const int excl = v - total + (wid > 0 ? warp_sums[wid - 1] : 0);
    if (e < E) {
        offsets[e] = excl;
        int run = excl;
        for (int c = 0; c < n_chunks; ++c) {
            const int n = chunk[(size_t)c * E + e];
            chunk[(size_t)c * E + e] = run;
            run += n;
        }
    }
    if (e == E - 1) offsets[E] = excl + total;
}

__global__ void __launch_bounds__(PERM_WARPS * 32) perm_scatter_kernel(
    const int32_t* __restrict__ idx, long N, int E, const int32_t* __restrict__ chunk,
    int32_t* __restrict__ sorted_pair, int32_t* __restrict__ row_of) {
    pdl_wait();
    pdl_trigger();
    __shared__ int32_t wbase[PERM_WARPS][PERM_MAX_E];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < PERM_WARPS * E; i += blockDim.x) wbase[i / E][i % E] = 0;
    __syncthreads();
    const long wstart = (long)blockIdx.x * PERM_CHUNK + (long)w * PERM_PER_WARP;
    // phase 1: per-warp histogram (leader of each equal-expert lane set adds its size)
    for (int it = 0; it < PERM_PER_WARP; it += 32) {
        const long p = wstart + it + lane;
        const bool valid = p < N;
        const int e = valid ? idx[p] : -1;
        const bool ok = valid && e >= 0 && e < E;
        const unsigned act = __ballot_sync(0xffffffffu, ok);
        if (ok) {
            const unsigned m = __match_any_sync(act, e);
            if ((__ffs(m) - 1) == lane) wbase[w][e] += __popc(m);
        }
        __syncwarp();
    }
    __syncthreads();
    // phase 2: warp bases = chunk base + counts of lower warps
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = chunk[(size_t)blockIdx.x * E + e];
        for (int ww = 0; ww < PERM_WARPS; ++ww) {
            const int n = wbase[ww][e];
            wbase[ww][e] = run;
            run += n;
        }
    }
    __syncthreads();
    // phase 3: stable placement
    const unsigned lt = (1u << lane) - 1u;
    for (int it = 0; it < PERM_PER_WARP; it += 32) {
        const long p = wstart + it + lane;
        const bool valid = p < N;
        const int e = valid ? idx[p] : -1;
        const bool ok = valid && e >= 0 && e < E;
        const unsigned act = __ballot_sync(0xffffffffu, ok);
        if (ok) {
            const unsigned m = __match_any_sync(act, e);
            const int pos = wbase[w][e] + __popc(m & lt);
            sorted_pair[pos] = (int32_t)p;
            row_of[p] = pos;
            __syncwarp(act);
            if ((__ffs(m) - 1) == lane) wbase[w][e] += __popc(m);
        } else if (valid) {
            row_of[p] = -1;
        }
        __syncwarp();
    }
}

// All pairs in one chunk (N <= PERM_CHUNK): count, scan and scatter in one CTA,
// with per-warp histograms and in-warp ranks as in the three launches. The pairs
// are split evenly over the warps (span pairs each, a multiple of 32, in pair
// order), so small batches keep every warp busy; any split into contiguous
// ranges in warp order gives the same stable order. Each lane loads its
// span / 32 expert ids once, up front (independent loads), and both passes run
// on the registers.
__global__ void __launch_bounds__(PERM_WARPS * 32) perm_single_kernel(
    const int32_t* __restrict__ idx, long N, int E, int32_t* __restrict__ offsets,
    int32_t* __restrict__ sorted_pair, int32_t* __restrict__ row_of, int32_t* status) {
    pdl_wait();
    pdl_trigger();
    constexpr int PER_LANE = PERM_PER_WARP / 32;
    __shared__ int32_t wbase[PERM_WARPS][PERM_MAX_E];
    __shared__ int32_t excl[PERM_MAX_E];
    __shared__ int32_t part[PERM_WARPS * 32];
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int span = (int)((N + PERM_WARPS * 32 - 1) / (PERM_WARPS * 32)) * 32;  // <= PERM_PER_WARP
    const int n_it = span / 32;
    const long wstart = (long)w * span;
    int ev[PER_LANE];  // expert id of pair wstart + 32*i + lane, or -1 past N
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i) {
        const long p = wstart + 32 * i + lane;
        ev[i] = (i < n_it && p < N) ? idx[p] : -1;
    }
    for (int i = tid; i < PERM_WARPS * E; i += blockDim.x) wbase[i / E][i % E] = 0;
    __syncthreads();
    bool bad = false;
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i) {
        if (i >= n_it) break;  // warp-uniform
        const long p = wstart + 32 * i + lane;
        const int e = ev[i];
        const bool ok = p < N && e >= 0 && e < E;
        bad |= p < N && !ok;
        const unsigned act = __ballot_sync(0xffffffffu, ok);
        if (ok) {
            const unsigned m = __match_any_sync(act, e);
            if ((__ffs(m) - 1) == lane) wbase[w][e] += __popc(m);
        }
        __syncwarp();
    }
    if (bad) status_or(status, MOE_DEV_BAD_EXPERT);
    __syncthreads();
    // exclusive scan of the expert totals: thread tid owns experts [tid*per, (tid+1)*per)
    const int per = (E + blockDim.x - 1) / blockDim.x;
    int mine = 0;
    for (int e = tid * per; e < min(E, (tid + 1) * per); ++e) {
        int tot = 0;
        for (int ww = 0; ww < PERM_WARPS; ++ww) tot += wbase[ww][e];
        excl[e] = tot;
        mine += tot;
    }
    int v = mine;  // inclusive scan over threads
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += o;
    }
    part[tid] = v;
    __syncthreads();
    int base = v - mine;
    for (int ww = 0; ww < w; ++ww) base += part[ww * 32 + 31];
    for (int e = tid * per; e < min(E, (tid + 1) * per); ++e) {
        const int tot = excl[e];
        offsets[e] = base;
        int run = base;
        for (int ww = 0; ww < PERM_WARPS; ++ww) {
            const int n = wbase[ww][e];
            wbase[ww][e] = run;
            run += n;
        }
        base += tot;
    }
    if (tid == blockDim.x - 1) offsets[E] = base;
    __syncthreads();
    const unsigned lt = (1u << lane) - 1u;
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i) {
        if (i >= n_it) break;  // warp-uniform
        const long p = wstart + 32 * i + lane;
        const int e = ev[i];
        const bool valid = p < N;
        const bool ok = valid && e >= 0 && e < E;
        const unsigned act = __ballot_sync(0xffffffffu, ok);
        if (ok) {
            const unsigned m = __match_any_sync(act, e);
            const int pos = wbase[w][e] + __popc(m & lt);
            sorted_pair[pos] = (int32_t)p;
            row_of[p] = pos;
            __syncwarp(act);
            if ((__ffs(m) - 1) == lane) wbase[w][e] += __popc(m);
        } else if (valid) {
            row_of[p] = -1;
        }
        __syncwarp();
    }
}

}  // namespace

int permute_chunks(long N) { return (int)((N + PERM_CHUNK - 1) / PERM_CHUNK); }

cudaError_t launch_permute(const int32_t* idx, int T, int k, int E, int n_chunks, int32_t* chunk,
                           int32_t* offsets, int32_t* sorted_pair, int32_t* row_of,
                           int32_t* status, cudaStream_t st) {
    const long N = (long)T * k;
    if (n_chunks <= 1) {
        launch_pdl(perm_single_kernel, 1, PERM_WARPS * 32, 0, st, idx, N, E, offsets, sorted_pair,
            row_of, status);
        return cudaGetLastError();
    }
    launch_pdl(perm_count_kernel, n_chunks, 256, 0, st, idx, N, E, chunk, status);
    launch_pdl(perm_scan_kernel, 1, 1024, 0, st, chunk, n_chunks, E, offsets);
    launch_pdl(perm_scatter_kernel, n_chunks, PERM_WARPS * 32, 0, st, idx, N, E, chunk, sorted_pair,
        row_of);
    return cudaGetLastError();
}

}  // namespace moe

// ------------------------------------------------------------------------
// moe_permute_noalloc: the same three launches, with the per-chunk counts in a
// file-scope device array instead of a caller workspace, for callers that may
// not allocate device memory (see include/moe.h). Host code must not pass the
// array's name to a kernel: on the host that name is only a stand-in, so the
// device address is looked up once per device with cudaGetSymbolAddress.
static __device__ __align__(256) int32_t g_permute_noalloc_counts[MOE_PERMUTE_NOALLOC_MAX_COUNTS];

// Device address of the array on the current device (looked up on first use).
static int32_t* permute_noalloc_scratch() {
    static std::mutex mu;
    static int32_t* addr[64] = {nullptr};
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_permute_noalloc_counts) != cudaSuccess) return nullptr;
        addr[dev] = static_cast<int32_t*>(p);
    }
    return addr[dev];
}

extern "C" moe_status moe_permute_noalloc(const moe_config* cfg, const int32_t* topk_idx,
                                          int32_t T, int32_t* expert_offsets,
                                          int32_t* sorted_pair, int32_t* row_of,
                                          int32_t* dev_status, void* stream) {
    using namespace moe;
    if (!config_valid(cfg) || T < 0) return MOE_ERR_INVALID_ARG;
    if (!expert_offsets) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!topk_idx || !sorted_pair || !row_of)) return MOE_ERR_INVALID_ARG;
    const long N = (long)T * cfg->num_experts_per_tok;
    if (N > 0x7fffffffL) return MOE_ERR_INVALID_ARG;
    const int n_chunks = permute_chunks(N);
    if ((long)n_chunks * cfg->n_routed_experts > MOE_PERMUTE_NOALLOC_MAX_COUNTS)
        return MOE_ERR_WORKSPACE;
    int32_t* counts = permute_noalloc_scratch();
    if (!counts) return MOE_ERR_CUDA;
    const cudaError_t e = launch_permute(topk_idx, T, cfg->num_experts_per_tok,
                                         cfg->n_routed_experts, n_chunks, counts, expert_offsets,
                                         sorted_pair, row_of, dev_status,
                                         static_cast<cudaStream_t>(stream));
    return cuda_status(e);
}
