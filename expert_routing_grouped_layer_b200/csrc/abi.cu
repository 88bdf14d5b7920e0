// abi.cu -- the extern "C" entry points declared in include/moe.h: argument
// checks, workspace carve-up and the launch order of the layer.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <map>
#include <mutex>
#include <utility>

#include "internal.h"

namespace moe {

int permute_chunks(long N);

// SM count of the current device, cached per device (host threads may race to
// fill an entry; they all store the same value).
int num_sms() {
    static std::atomic<int> cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cache[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

cudaError_t ensure_smem_limit(const void* kernel, int bytes) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    static std::mutex mu;
    static std::map<std::pair<const void*, int>, int> limit;  // largest size set per (kernel, device)
    std::lock_guard<std::mutex> lock(mu);
    const auto key = std::make_pair(kernel, dev);
    const auto it = limit.find(key);
    if (it != limit.end() && it->second >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) limit[key] = bytes;
    return e;
}

bool config_valid(const moe_config* c) {
    if (!c) return false;
    if (c->hidden <= 0 || c->hidden % 128) return false;
    if (c->n_routed_experts < 1 || c->n_routed_experts > 1024) return false;
    if (c->num_experts_per_tok < 1 || c->num_experts_per_tok > 32) return false;
    if (c->num_experts_per_tok > c->n_routed_experts) return false;
    if (c->n_group < 1 || c->n_group > 32 || c->n_routed_experts % c->n_group) return false;
    if (c->topk_group < 1 || c->topk_group > c->n_group) return false;
    if ((long)c->topk_group * (c->n_routed_experts / c->n_group) < c->num_experts_per_tok) return false;
    if (c->moe_intermediate_size <= 0 || c->moe_intermediate_size % 128) return false;
    if (c->n_shared_experts < 0 || c->n_shared_experts > 4) return false;
    if (c->n_shared_experts > 0 &&
        (c->shared_intermediate_size <= 0 || c->shared_intermediate_size % 128))
        return false;
    if (c->norm_topk_prob != 0 && c->norm_topk_prob != 1) return false;
    if (!(c->routed_scaling_factor > 0.0f)) return false;
    if (c->score_fn != MOE_SCORE_SIGMOID && c->score_fn != MOE_SCORE_SQRTSOFTPLUS &&
        c->score_fn != MOE_SCORE_SOFTMAX)
        return false;
    if (!(c->swiglu_limit >= 0.0f) || isinf(c->swiglu_limit)) return false;
    if (c->wfmt < MOE_W_BF16 || c->wfmt > MOE_W_NVFP4) return false;
    if (c->afmt < MOE_A_BF16 || c->afmt > MOE_A_NVFP4) return false;
    if (c->afmt == MOE_A_NVFP4 &&
        !(c->nvfp4_x_scale > 0.0f && c->nvfp4_h_scale > 0.0f && !isinf(c->nvfp4_x_scale) &&
          !isinf(c->nvfp4_h_scale)))
        return false;
    return true;
}

// Valid configurations the expert kernels do not implement (yet).
moe_status config_supported(const moe_config* c) {
    if (c->n_shared_experts > 0 && c->shared_intermediate_size != c->moe_intermediate_size)
        return MOE_ERR_UNSUPPORTED;
    if (c->afmt == MOE_A_BF16 && (c->wfmt == MOE_W_BF16 || c->wfmt == MOE_W_FP8_E4M3_B128x128))
        return MOE_OK;
    // NVFP4 routed experts: 256 packed E2M1 values per 128-byte row of a stage,
    // two 128-row weight tiles per unit
    if (c->wfmt == MOE_W_NVFP4 && c->afmt == MOE_A_NVFP4 && c->hidden % 256 == 0 &&
        c->moe_intermediate_size % 256 == 0)
        return MOE_OK;
    // block-scaled tensor cores: E2M1 weights x E4M3 activations; the scale tiles
    // move by TMA in rows of 16 scales, so H and I must be multiples of 512
    if ((c->wfmt == MOE_W_FP4_E2M1_UE8M0_B32 || c->wfmt == MOE_W_MXFP4) &&
        (c->afmt == MOE_A_FP8_E4M3_POW2_B128 || c->afmt == MOE_A_MXFP8) && c->hidden % 512 == 0 &&
        c->moe_intermediate_size % 512 == 0)
        return MOE_OK;
    return MOE_ERR_UNSUPPORTED;
}

static size_t align_up(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

WsLayout ws_layout(const moe_config* c, int T) {
    WsLayout L{};
    const size_t E = c->n_routed_experts, k = c->num_experts_per_tok, H = c->hidden;
    const size_t I = c->moe_intermediate_size, S = c->n_shared_experts;
    const size_t N = (size_t)T * k;
    const size_t act_bytes = (c->afmt == MOE_A_BF16) ? 2 : 1;
    const RouterPlan rp = router_plan(T > 0 ? T : 1, (int)E, (int)H);
    L.router_splits = rp.splits;
    L.n_chunks = permute_chunks((long)N);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align_up(off + bytes);
        return o;
    };
    L.router_planes = take((size_t)3 * rp.Epad * H * 2);
    L.router_part = take((size_t)L.router_splits * T * E * 4);
    L.topk_idx = take(N * 4);
    L.topk_w = take(N * 4);
    L.offsets = take((E + 1) * 4);
    L.sorted_pair = take(N * 4);
    L.row_of = take(N * 4);
    L.chunk_counts = take((size_t)L.n_chunks * E * 4);
    if (c->afmt == MOE_A_NVFP4) {
        // packed routed rows (+ the token rows they are gathered from), then the
        // bf16 token rows of the shared experts; h likewise with bf16 shared rows
        L.xa = take(nvfp4_tail_offset((N + T) * H / 2) + (size_t)T * H * 2);
        L.xa_scale = take((N + T) * (H / 16));
        L.hbuf = take(nvfp4_tail_offset(N * I / 2) + S * T * I * 2);
        L.h_scale = take(N * (I / 16));
    } else {
        L.xa = take((N + T) * H * act_bytes);
        L.xa_scale = take(act_bytes == 1 ? (N + T) * (H / 32) : (f16_gate_up(c) ? (N + T) : 0));
        L.hbuf = take((N + S * T) * I * act_bytes);
        L.h_scale = take(act_bytes == 1 ? (N + S * T) * (I / 32) : (f16_gate_up(c) ? (N + S * T) : 0));
    }
    L.y = take(N * H * 2);
    L.shared_y = take(S * T * H * 2);
    L.x_norm = take((size_t)T * H * 2);
    L.total = off;
    return L;
}

}  // namespace moe

using namespace moe;

static inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

static inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

extern "C" {

size_t moe_workspace_bytes(const moe_config* cfg, int32_t T) {
    if (!config_valid(cfg) || T < 0) return 0;
    return ws_layout(cfg, T).total;
}

size_t moe_workspace_offset(const moe_config* cfg, int32_t T, int32_t which) {
    if (!config_valid(cfg) || T < 0) return (size_t)-1;
    const WsLayout L = ws_layout(cfg, T);
    switch (which) {
    case 0: return L.topk_idx;
    case 1: return L.topk_w;
    case 2: return L.offsets;
    case 3: return L.sorted_pair;
    case 4: return L.row_of;
    case 5: return L.y;
    case 6: return L.shared_y;
    case 7: return L.xa;
    case 8: return L.xa_scale;
    case 9: return L.hbuf;
    case 10: return L.h_scale;
    case 11: return L.x_norm;
    }
    return (size_t)-1;
}

const char* moe_status_string(moe_status s) {
    switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA launch error";
    }
    return "unknown status";
}

moe_status moe_gate_topk(const moe_config* cfg, const void* x, int32_t T, const float* gate_w,
                         const float* gate_bias, int32_t* topk_idx, float* topk_w,
                         int32_t* dev_status, void* ws, size_t ws_bytes, void* stream) {
    if (!config_valid(cfg) || T < 0) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!x || !gate_w || !gate_bias || !topk_idx || !topk_w || !ws) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(gate_w)) return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(cfg, T);
    if (ws_bytes < L.router_part + (size_t)L.router_splits * T * cfg->n_routed_experts * 4)
        return MOE_ERR_WORKSPACE;
    char* base = static_cast<char*>(ws);
    float* part = reinterpret_cast<float*>(base + L.router_part);
    cudaStream_t st = as_stream(stream);
    cudaError_t e = launch_router_tc(x, gate_w, base + L.router_planes, part, T,
                                     cfg->n_routed_experts, cfg->hidden, dev_status, st);
    if (e == cudaSuccess) e = launch_topk(cfg, part, gate_bias, T, topk_idx, topk_w, st);
    return cuda_status(e);
}

moe_status moe_permute(const moe_config* cfg, const int32_t* topk_idx, int32_t T,
                       int32_t* expert_offsets, int32_t* sorted_pair, int32_t* row_of,
                       int32_t* dev_status, void* ws, size_t ws_bytes, void* stream) {
    if (!config_valid(cfg) || T < 0) return MOE_ERR_INVALID_ARG;
    if (!expert_offsets || !ws) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!topk_idx || !sorted_pair || !row_of)) return MOE_ERR_INVALID_ARG;
    if ((long)T * cfg->num_experts_per_tok > 0x7fffffffL) return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(cfg, T);
    if (ws_bytes < L.chunk_counts + (size_t)L.n_chunks * cfg->n_routed_experts * 4)
        return MOE_ERR_WORKSPACE;
    int32_t* chunk = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + L.chunk_counts);
    return cuda_status(launch_permute(topk_idx, T, cfg->num_experts_per_tok, cfg->n_routed_experts,
                                      L.n_chunks, chunk, expert_offsets, sorted_pair, row_of,
                                      dev_status, as_stream(stream)));
}

moe_status moe_quantize_activations(const moe_config* cfg, const void* x, int32_t T, void* xq,
                                    void* xq_scale, void* stream) {
    if (!config_valid(cfg) || T < 0 || cfg->afmt == MOE_A_BF16) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!x || !xq || !xq_scale || !aligned16(x) || !aligned16(xq)) return MOE_ERR_INVALID_ARG;
    if (cfg->afmt == MOE_A_NVFP4) {
        if (cfg->hidden % 256) return MOE_ERR_INVALID_ARG;
        return cuda_status(launch_pack_nvfp4(x, cfg->hidden, cfg->nvfp4_x_scale, T, xq,
                                             static_cast<uint8_t*>(xq_scale), nullptr,
                                             as_stream(stream)));
    }
    return cuda_status(launch_pack_rows(cfg->afmt, x, cfg->hidden, nullptr, 0,
                                        cfg->num_experts_per_tok, T, T, xq,
                                        static_cast<uint8_t*>(xq_scale), 0, as_stream(stream)));
}

static bool weights_ok(const moe_config* cfg, const moe_weights* w, bool gate_up) {
    const void* r = gate_up ? w->w13 : w->w2;
    const void* rs = gate_up ? w->w13_scale : w->w2_scale;
    const void* sh = gate_up ? w->sh_w13 : w->sh_w2;
    const void* shs = gate_up ? w->sh_w13_scale : w->sh_w2_scale;
    const bool scaled = cfg->wfmt != MOE_W_BF16;
    const bool nvfp4 = cfg->wfmt == MOE_W_NVFP4;  // bf16 shared experts, tensor scales
    if (!r || !aligned16(r) || (scaled && (!rs || !aligned16(rs)))) return false;
    if (nvfp4 && !(gate_up ? w->w13_gscale : w->w2_gscale)) return false;
    if (cfg->n_shared_experts > 0 && (!sh || !aligned16(sh) || (scaled && !nvfp4 && !shs)))
        return false;
    return true;
}

static GroupedGemmArgs gemm_args(const moe_config* cfg, int T, const int32_t* offsets,
                                 int32_t* dev_status) {
    GroupedGemmArgs a{};
    a.E = cfg->n_routed_experts;
    a.S = cfg->n_shared_experts;
    a.T = T;
    a.k = cfg->num_experts_per_tok;
    a.N = T * a.k;
    a.H = cfg->hidden;
    a.I = cfg->moe_intermediate_size;
    a.wfmt = cfg->wfmt;
    a.afmt = cfg->afmt;
    a.offsets = offsets;
    a.status = dev_status;
    a.swiglu_limit = cfg->swiglu_limit;
    return a;
}

moe_status moe_pack_expert_inputs(const moe_config* cfg, const void* x, int32_t T,
                                  const int32_t* sorted_pair, void* xa, void* xa_scale,
                                  void* stream) {
    if (!config_valid(cfg) || T < 0) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!x || !sorted_pair || !xa || !aligned16(x) || !aligned16(xa)) return MOE_ERR_INVALID_ARG;
    if ((cfg->afmt != MOE_A_BF16 || f16_gate_up(cfg)) && !xa_scale) return MOE_ERR_INVALID_ARG;
    const int k = cfg->num_experts_per_tok, N = T * k;
    if (cfg->afmt == MOE_A_NVFP4) {
        // the token rows once (rows N..N+T-1, with the bf16 copy for the shared
        // experts behind the packed rows), then the routed rows gathered from them
        if (cfg->hidden % 256) return MOE_ERR_INVALID_ARG;
        const int H = cfg->hidden;
        uint8_t* q = static_cast<uint8_t*>(xa);
        uint8_t* qs = static_cast<uint8_t*>(xa_scale);
        void* xb = q + nvfp4_tail_offset((size_t)(N + T) * H / 2);
        cudaError_t e = launch_pack_nvfp4(x, H, cfg->nvfp4_x_scale, T, q + (size_t)N * H / 2,
                                          qs + (size_t)N * (H / 16), xb, as_stream(stream));
        if (e == cudaSuccess)
            e = launch_gather_nvfp4_rows(q + (size_t)N * H / 2, qs + (size_t)N * (H / 16), H,
                                         sorted_pair, N, k, T, q, qs, as_stream(stream));
        return cuda_status(e);
    }
    if (f16_gate_up(cfg))
        return cuda_status(launch_pack_f16_rows(x, cfg->hidden, sorted_pair, N, k, T, N + T, xa,
                                                static_cast<int8_t*>(xa_scale), as_stream(stream)));
    return cuda_status(launch_pack_rows(cfg->afmt, x, cfg->hidden, sorted_pair, N, k, T, N + T, xa,
                                        static_cast<uint8_t*>(xa_scale), 1, as_stream(stream)));
}

moe_status moe_expert_gate_up(const moe_config* cfg, const void* xa, const void* xa_scale,
                              int32_t T, const int32_t* expert_offsets, const moe_weights* w,
                              void* h, void* h_scale, int32_t* dev_status, void* stream) {
    if (!config_valid(cfg) || T < 0 || !w) return MOE_ERR_INVALID_ARG;
    const moe_status sup = config_supported(cfg);
    if (sup != MOE_OK) return sup;
    if (T == 0) return MOE_OK;
    const bool q = cfg->afmt != MOE_A_BF16;
    if (!xa || !expert_offsets || !h || !aligned16(xa) || !aligned16(h)) return MOE_ERR_INVALID_ARG;
    if (q && (!xa_scale || !h_scale)) return MOE_ERR_INVALID_ARG;
    if (f16_gate_up(cfg) && (!xa_scale || !h_scale)) return MOE_ERR_INVALID_ARG;
    if (!weights_ok(cfg, w, true)) return MOE_ERR_INVALID_ARG;
    GroupedGemmArgs a = gemm_args(cfg, T, expert_offsets, dev_status);
    if (cfg->afmt == MOE_A_NVFP4) {
        const int H = a.H, I = a.I, N = a.N;
        a.gemm = 1;
        a.w_routed = w->w13;
        a.w_routed_scale = w->w13_scale;
        a.w_gscale = w->w13_gscale;
        a.a_gscale = cfg->nvfp4_x_scale;
        a.out_gscale = cfg->nvfp4_h_scale;
        a.b_rows = xa;
        a.b_scale = static_cast<const uint8_t*>(xa_scale);
        a.out_routed = h;
        a.out_routed_scale = static_cast<uint8_t*>(h_scale);
        cudaError_t e = launch_grouped_gemm(a, as_stream(stream));
        if (e == cudaSuccess && a.S > 0) {  // bf16 shared experts on the bf16 token rows
            GroupedGemmArgs b = gemm_args(cfg, T, expert_offsets, dev_status);
            b.E = 0;
            b.N = 0;
            b.wfmt = MOE_W_BF16;
            b.afmt = MOE_A_BF16;
            b.gemm = 1;
            b.w_routed = b.w_shared = w->sh_w13;
            b.b_rows = static_cast<const uint8_t*>(xa) + nvfp4_tail_offset((size_t)(N + T) * H / 2);
            b.out_shared = static_cast<uint8_t*>(h) + nvfp4_tail_offset((size_t)N * I / 2);
            e = launch_grouped_gemm(b, as_stream(stream));
        }
        return cuda_status(e);
    }
    const size_t hrow = (size_t)a.I * (q ? 1 : 2);
    a.gemm = 1;
    a.w_routed = w->w13;
    a.w_routed_scale = w->w13_scale;
    a.w_shared = w->sh_w13;
    a.w_shared_scale = w->sh_w13_scale;
    a.b_rows = xa;
    a.b_scale = static_cast<const uint8_t*>(xa_scale);
    a.out_routed = h;
    a.out_shared = static_cast<char*>(h) + (size_t)a.N * hrow;
    a.out_routed_scale = static_cast<uint8_t*>(h_scale);
    a.out_shared_scale = q ? static_cast<uint8_t*>(h_scale) + (size_t)a.N * (a.I / 32) : nullptr;
    cudaError_t e = launch_grouped_gemm(a, as_stream(stream));
    if (e == cudaSuccess && f16_gate_up(cfg))  // the down projection's f16 input rows
        e = launch_rows_to_f16(h, a.I, a.N + a.S * a.T, static_cast<int8_t*>(h_scale), as_stream(stream));
    return cuda_status(e);
}

moe_status moe_expert_down(const moe_config* cfg, const void* h, const void* h_scale, int32_t T,
                           const int32_t* expert_offsets, const moe_weights* w, void* y,
                           void* shared_y, int32_t* dev_status, void* stream) {
    if (!config_valid(cfg) || T < 0 || !w) return MOE_ERR_INVALID_ARG;
    const moe_status sup = config_supported(cfg);
    if (sup != MOE_OK) return sup;
    if (T == 0) return MOE_OK;
    const bool q = cfg->afmt != MOE_A_BF16;
    if (!h || !expert_offsets || !y || !aligned16(h) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
    if (cfg->n_shared_experts > 0 && (!shared_y || !aligned16(shared_y))) return MOE_ERR_INVALID_ARG;
    if ((q || f16_gate_up(cfg)) && !h_scale) return MOE_ERR_INVALID_ARG;
    if (!weights_ok(cfg, w, false)) return MOE_ERR_INVALID_ARG;
    GroupedGemmArgs a = gemm_args(cfg, T, expert_offsets, dev_status);
    if (cfg->afmt == MOE_A_NVFP4) {
        a.gemm = 2;
        a.w_routed = w->w2;
        a.w_routed_scale = w->w2_scale;
        a.w_gscale = w->w2_gscale;
        a.a_gscale = cfg->nvfp4_h_scale;
        a.b_rows = h;
        a.b_scale = static_cast<const uint8_t*>(h_scale);
        a.out_routed = y;
        cudaError_t e = launch_grouped_gemm(a, as_stream(stream));
        if (e == cudaSuccess && a.S > 0) {  // bf16 shared experts on their bf16 rows of h
            GroupedGemmArgs b = gemm_args(cfg, T, expert_offsets, dev_status);
            b.E = 0;
            b.N = 0;
            b.wfmt = MOE_W_BF16;
            b.afmt = MOE_A_BF16;
            b.gemm = 2;
            b.w_routed = b.w_shared = w->sh_w2;
            b.b_rows = static_cast<const uint8_t*>(h) + nvfp4_tail_offset((size_t)a.N * a.I / 2);
            b.out_shared = shared_y;
            e = launch_grouped_gemm(b, as_stream(stream));
        }
        return cuda_status(e);
    }
    a.gemm = 2;
    a.w_routed = w->w2;
    a.w_routed_scale = w->w2_scale;
    a.w_shared = w->sh_w2;
    a.w_shared_scale = w->sh_w2_scale;
    a.b_rows = h;
    a.b_scale = static_cast<const uint8_t*>(h_scale);
    a.out_routed = y;
    a.out_shared = shared_y;
    return cuda_status(launch_grouped_gemm(a, as_stream(stream)));
}

moe_status moe_grouped_swiglu(const moe_config* cfg, const void* x, int32_t T,
                              const int32_t* sorted_pair, const int32_t* expert_offsets,
                              const moe_weights* w, void* y, void* shared_y, void* ws,
                              size_t ws_bytes, int32_t* dev_status, void* stream) {
    if (!config_valid(cfg) || T < 0 || !w) return MOE_ERR_INVALID_ARG;
    const moe_status sup = config_supported(cfg);
    if (sup != MOE_OK) return sup;
    if (T == 0) return MOE_OK;
    // everything is checked before the first launch
    if (!ws || !x || !sorted_pair || !expert_offsets || !y || !aligned16(x) || !aligned16(y))
        return MOE_ERR_INVALID_ARG;
    if (cfg->n_shared_experts > 0 && (!shared_y || !aligned16(shared_y))) return MOE_ERR_INVALID_ARG;
    if (!weights_ok(cfg, w, true) || !weights_ok(cfg, w, false)) return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(cfg, T);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    char* base = static_cast<char*>(ws);
    moe_status s = moe_pack_expert_inputs(cfg, x, T, sorted_pair, base + L.xa, base + L.xa_scale,
                                          stream);
    if (s == MOE_OK)
        s = moe_expert_gate_up(cfg, base + L.xa, base + L.xa_scale, T, expert_offsets, w,
                               base + L.hbuf, base + L.h_scale, dev_status, stream);
    if (s == MOE_OK)
        s = moe_expert_down(cfg, base + L.hbuf, base + L.h_scale, T, expert_offsets, w, y, shared_y,
                            dev_status, stream);
    return s;
}

moe_status moe_combine(const moe_config* cfg, const void* y, const void* shared_y,
                       const int32_t* row_of, const float* topk_w, int32_t T, void* out,
                       void* stream) {
    if (!config_valid(cfg) || T < 0) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    const int S = cfg->n_shared_experts;
    if (!y || !row_of || !topk_w || !out || (S > 0 && !shared_y)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(y) || !aligned16(out) || (S > 0 && !aligned16(shared_y)))
        return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_combine(y, shared_y, S, row_of, topk_w, T, cfg->num_experts_per_tok,
                                      cfg->hidden, out, as_stream(stream)));
}

moe_status moe_layer_forward(const moe_config* cfg, const void* x, int32_t T, const moe_weights* w,
                             void* out, void* ws, size_t ws_bytes, int32_t* dev_status,
                             void* stream) {
    if (!config_valid(cfg) || T < 0 || !w) return MOE_ERR_INVALID_ARG;
    const moe_status sup = config_supported(cfg);
    if (sup != MOE_OK) return sup;
    if (T == 0) return MOE_OK;
    // everything is checked before the first launch
    if (!x || !out || !ws || !w->gate_w || !w->gate_bias) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(out) || !aligned16(w->gate_w)) return MOE_ERR_INVALID_ARG;
    if (!weights_ok(cfg, w, true) || !weights_ok(cfg, w, false)) return MOE_ERR_INVALID_ARG;
    if ((long)T * cfg->num_experts_per_tok > 0x7fffffffL) return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(cfg, T);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    char* base = static_cast<char*>(ws);
    int32_t* idx = reinterpret_cast<int32_t*>(base + L.topk_idx);
    float* tw = reinterpret_cast<float*>(base + L.topk_w);
    int32_t* off = reinterpret_cast<int32_t*>(base + L.offsets);
    int32_t* sp = reinterpret_cast<int32_t*>(base + L.sorted_pair);
    int32_t* ro = reinterpret_cast<int32_t*>(base + L.row_of);
    void* y = base + L.y;
    void* sy = base + L.shared_y;
    moe_status s = moe_gate_topk(cfg, x, T, w->gate_w, w->gate_bias, idx, tw, dev_status, ws,
                                 ws_bytes, stream);
    if (s == MOE_OK) s = moe_permute(cfg, idx, T, off, sp, ro, dev_status, ws, ws_bytes, stream);
    if (s == MOE_OK)
        s = moe_grouped_swiglu(cfg, x, T, sp, off, w, y, sy, ws, ws_bytes, dev_status, stream);
    if (s == MOE_OK) s = moe_combine(cfg, y, sy, ro, tw, T, out, stream);
    return s;
}

moe_status moe_rmsnorm_prologue(const moe_config* cfg, const void* x, int32_t T, const float* norm_w,
                                float eps, void* x_norm, void* xq, void* xq_scale, void* stream) {
    if (!config_valid(cfg) || T < 0) return MOE_ERR_INVALID_ARG;
    if (!(eps >= 0.0f) || isinf(eps)) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!x || !norm_w || !x_norm || !aligned16(x) || !aligned16(norm_w) || !aligned16(x_norm))
        return MOE_ERR_INVALID_ARG;
    // FP8 / MX activations: the quantised rows in the same pass (NVFP4 layers
    // quantise their routed inputs from x_norm in the expert-input step)
    const bool q = cfg->afmt == MOE_A_FP8_E4M3_POW2_B128 || cfg->afmt == MOE_A_MXFP8;
    if (q && (cfg->hidden % 512 || !xq || !xq_scale || !aligned16(xq) || !aligned16(xq_scale)))
        return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_rmsnorm_quant(cfg->afmt, x, cfg->hidden, norm_w, eps, T, x_norm,
                                            q ? xq : nullptr,
                                            static_cast<uint8_t*>(q ? xq_scale : nullptr),
                                            as_stream(stream)));
}

moe_status moe_layer_forward_prenorm(const moe_config* cfg, const void* x, int32_t T,
                                     const float* norm_w, float eps, const moe_weights* w,
                                     void* out, void* ws, size_t ws_bytes, int32_t* dev_status,
                                     void* stream) {
    if (!config_valid(cfg) || T < 0 || !w) return MOE_ERR_INVALID_ARG;
    const moe_status sup = config_supported(cfg);
    if (sup != MOE_OK) return sup;
    if (!(eps >= 0.0f) || isinf(eps)) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    // everything is checked before the first launch
    if (!x || !norm_w || !out || !ws || !w->gate_w || !w->gate_bias) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(norm_w) || !aligned16(out) || !aligned16(w->gate_w))
        return MOE_ERR_INVALID_ARG;
    if (!weights_ok(cfg, w, true) || !weights_ok(cfg, w, false)) return MOE_ERR_INVALID_ARG;
    if ((long)T * cfg->num_experts_per_tok > 0x7fffffffL) return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(cfg, T);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    char* base = static_cast<char*>(ws);
    int32_t* idx = reinterpret_cast<int32_t*>(base + L.topk_idx);
    float* tw = reinterpret_cast<float*>(base + L.topk_w);
    int32_t* off = reinterpret_cast<int32_t*>(base + L.offsets);
    int32_t* sp = reinterpret_cast<int32_t*>(base + L.sorted_pair);
    int32_t* ro = reinterpret_cast<int32_t*>(base + L.row_of);
    void* xn = base + L.x_norm;
    void* y = base + L.y;
    void* sy = base + L.shared_y;
    const int k = cfg->num_experts_per_tok, H = cfg->hidden, N = T * k;
    cudaStream_t st = as_stream(stream);
    if (cfg->afmt == MOE_A_BF16 || cfg->afmt == MOE_A_NVFP4) {
        // bf16 / NVFP4 expert inputs: the prologue's output feeds the unchanged layer
        moe_status s = cuda_status(launch_rmsnorm_quant(MOE_A_BF16, x, H, norm_w, eps, T, xn,
                                                        nullptr, nullptr, st));
        if (s == MOE_OK)
            s = moe_layer_forward(cfg, xn, T, w, out, ws, ws_bytes, dev_status, stream);
        return s;
    }
    // quantised expert inputs: the prologue writes the token rows (rows N..N+T-1
    // of the expert input, the shared experts' rows) once; the routed rows are
    // gathered from them after the permutation
    uint8_t* xa = reinterpret_cast<uint8_t*>(base + L.xa);
    uint8_t* xas = reinterpret_cast<uint8_t*>(base + L.xa_scale);
    uint8_t* qrows = xa + (size_t)N * H;
    uint8_t* qscales = xas + (size_t)N * (H / 32);
    moe_status s = cuda_status(launch_rmsnorm_quant(cfg->afmt, x, H, norm_w, eps, T, xn, qrows,
                                                    qscales, st));
    if (s == MOE_OK)
        s = moe_gate_topk(cfg, xn, T, w->gate_w, w->gate_bias, idx, tw, dev_status, ws, ws_bytes,
                          stream);
    if (s == MOE_OK) s = moe_permute(cfg, idx, T, off, sp, ro, dev_status, ws, ws_bytes, stream);
    if (s == MOE_OK)
        s = cuda_status(launch_gather_token_rows(qrows, qscales, H, sp, N, k, T, xa, xas, st));
    if (s == MOE_OK)
        s = moe_expert_gate_up(cfg, xa, xas, T, off, w, base + L.hbuf, base + L.h_scale, dev_status,
                               stream);
    if (s == MOE_OK)
        s = moe_expert_down(cfg, base + L.hbuf, base + L.h_scale, T, off, w, y, sy, dev_status,
                            stream);
    if (s == MOE_OK) s = moe_combine(cfg, y, sy, ro, tw, T, out, stream);
    return s;
}

moe_status moe_selftest_wait_limit(int32_t* dev_status, void* stream) {
    if (!dev_status) return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_wait_limit_selftest(dev_status, as_stream(stream)));
}

}  // extern "C"
