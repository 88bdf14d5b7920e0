// internal.h -- launchers shared between the library's translation units
// (C++ linkage, not part of the public ABI).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "moe.h"

namespace moe {

// Workspace carve-up shared by every entry point (offsets in bytes).
// Router GEMM plan: expert rows padded to 128, K split for small batches.
struct RouterPlan {
    int Epad;    // experts rounded up to 128
    int splits;  // K splits (partial-sum slabs)
    int kbps;    // 64-wide k-blocks per split
};

struct WsLayout {
    size_t router_planes; // bf16 [3][Epad][H] hi/mid/lo planes of the router weight
    size_t router_part;   // fp32 [splits][T][E] partial router sums
    size_t topk_idx;      // int32 [T][k]
    size_t topk_w;        // fp32 [T][k]
    size_t offsets;       // int32 [E+1]
    size_t sorted_pair;   // int32 [N]
    size_t row_of;        // int32 [N]
    size_t chunk_counts;  // int32 [n_chunks][E]
    size_t xa;            // gathered expert input rows [(N+T)][H] (bf16 or e4m3)
    size_t xa_scale;      // uint8 E8M0 [(N+T)][H/32]
    size_t hbuf;          // intermediate [(N+S*T)][I] (bf16 or e4m3)
    size_t h_scale;       // uint8 E8M0 [(N+S*T)][I/32]
    size_t y;             // bf16 [N][H]
    size_t shared_y;      // bf16 [S][T][H]
    size_t x_norm;        // bf16 [T][H] RMSNorm output (layer calls with the prologue)
    size_t total;
    int router_splits;
    int n_chunks;
};

bool config_valid(const moe_config* c);
// Raises a kernel's opt-in dynamic shared-memory limit on the current device to
// at least `bytes`; the size set per (kernel, device) pair is cached, so a call
// at or below it does nothing. A failed call leaves the cached size as it was.
cudaError_t ensure_smem_limit(const void* kernel, int bytes);
// Status of a launch error: MOE_ERR_UNSUPPORTED for an operation the device or
// driver does not support, MOE_ERR_CUDA for any other failure.
inline moe_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return MOE_OK;
    if (e == cudaErrorNotSupported) return MOE_ERR_UNSUPPORTED;
    return MOE_ERR_CUDA;
}
moe_status config_supported(const moe_config* c);
WsLayout ws_layout(const moe_config* c, int T);
int num_sms();

// Kernel launchers (return a cudaError_t of the launch).
RouterPlan router_plan(int T, int E, int H);
cudaError_t launch_router_tc(const void* x, const float* gate_w, void* planes, float* part, int T,
                             int E, int H, int32_t* status, cudaStream_t st);
cudaError_t launch_router_reduce(float* part, long n, int splits, cudaStream_t st);
cudaError_t launch_topk(const moe_config* c, const float* part, const float* bias, int T,
                        int32_t* idx, float* w, cudaStream_t st);
cudaError_t launch_permute(const int32_t* idx, int T, int k, int E, int n_chunks, int32_t* chunk,
                           int32_t* offsets, int32_t* sorted_pair, int32_t* row_of,
                           int32_t* status, cudaStream_t st);
cudaError_t launch_pack_rows(int afmt, const void* x, int H, const int32_t* sorted_pair, int N,
                             int k, int T, int n_rows, void* out, uint8_t* out_scale, int per32,
                             cudaStream_t st);
// f16 expert input rows with per-row power-of-two exponents (FP8-weight layers)
cudaError_t launch_pack_f16_rows(const void* x, int H, const int32_t* sorted_pair, int N, int k,
                                 int T, int n_rows, void* out, int8_t* xs, cudaStream_t st);
// bf16 rows [n_rows][C] -> f16 rows times 2^-e in place, e per row in xs (C % 8 == 0).
cudaError_t launch_rows_to_f16(void* rows, int C, int n_rows, int8_t* xs, cudaStream_t st);
// true when the expert GEMMs run on f16 operands (FP8 weights, bf16 activations):
// token rows and the SwiGLU output travel as f16 rows with per-row exponents
inline bool f16_gate_up(const moe_config* c) {
    return c->wfmt == MOE_W_FP8_E4M3_B128x128 && c->afmt == MOE_A_BF16;
}
// Post-attention RMSNorm (double arithmetic, one bf16 rounding) of x bf16
// [T][H] with weight w fp32 [H] into xn bf16 [T][H]; for a quantised afmt also
// E4M3 rows q [T][H] and E8M0 scales qs [T][H/32] of xn in one pass.
cudaError_t launch_rmsnorm_quant(int afmt, const void* x, int H, const float* w, float eps, int T,
                                 void* xn, void* q, uint8_t* qs, cudaStream_t st);
// 8-bit token rows [T][H] with their per-32 scale rows [T][H/32] gathered into
// expert order: out row r < N is token sorted_pair[r] / k (H % 512 == 0).
cudaError_t launch_gather_token_rows(const void* rows, const uint8_t* scales, int H,
                                     const int32_t* sorted_pair, int N, int k, int T, void* out,
                                     uint8_t* out_scale, cudaStream_t st);
// NVFP4 expert input rows of x bf16 [T][H] with tensor scale g: codes q
// [T][H/2] (two per byte), E4M3 scale codes qs [T][H/16]; xb (optional) gets a
// copy of the bf16 rows. H % 256 == 0.
cudaError_t launch_pack_nvfp4(const void* x, int H, float g, int T, void* q, uint8_t* qs, void* xb,
                              cudaStream_t st);
// NVFP4 token rows [T][H/2] with scale rows [T][H/16] gathered into expert order
// (out row r < N is token sorted_pair[r] / k).
cudaError_t launch_gather_nvfp4_rows(const void* rows, const uint8_t* scales, int H,
                                     const int32_t* sorted_pair, int N, int k, int T, void* out,
                                     uint8_t* out_scale, cudaStream_t st);
// NVFP4 layers: byte offset of the bf16 rows that follow the packed rows in the
// expert-input (xa) and intermediate (h) buffers
inline size_t nvfp4_tail_offset(size_t packed_bytes) { return (packed_bytes + 255) & ~size_t(255); }
cudaError_t launch_combine(const void* y, const void* shared_y, int S, const int32_t* row_of,
                           const float* w, int T, int k, int H, void* out, cudaStream_t st);
// one warp waits on a barrier nothing arrives on until the pipeline wait limit;
// sets MOE_DEV_TIMEOUT in *status
cudaError_t launch_wait_limit_selftest(int32_t* status, cudaStream_t st);

struct GroupedGemmArgs {
    // problem
    int gemm;           // 1: gate/up + SwiGLU, 2: down projection
    int E, S, T, N, k;  // experts, shared experts, tokens, pairs, top-k
    int H, I;
    int wfmt, afmt;
    const int32_t* offsets;  // [E+1]
    // operands
    const void* w_routed;  // w13 or w2
    const void* w_routed_scale;
    const void* w_shared;  // sh_w13 or sh_w2
    const void* w_shared_scale;
    const void* b_rows;  // gemm1: xa [(N+T)][H]; gemm2: hbuf [(N+S*T)][I]
    const uint8_t* b_scale;
    void* out_routed;  // gemm1: hbuf rows [0,N); gemm2: y
    void* out_shared;  // gemm1: hbuf rows [N, N+S*T); gemm2: shared_y
    uint8_t* out_routed_scale;
    uint8_t* out_shared_scale;
    int32_t* status;
    float swiglu_limit;  // gemm1: 0 = off, else SiLU(min(g, L)) * clamp(u, -L, L)
    // NVFP4 only: per routed expert fp32 tensor scale of the weight, the B
    // operand's tensor scale, and (gemm1) the quantised intermediate's
    const float* w_gscale;
    float a_gscale;
    float out_gscale;
};
cudaError_t launch_grouped_gemm(const GroupedGemmArgs& a, cudaStream_t st);

}  // namespace moe
