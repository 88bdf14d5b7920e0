// gemm_dispatch.cu -- picks the expert GEMM kernel for a weight/activation format.
#include "internal.h"

namespace moe {
namespace gemm {
cudaError_t launch_gemm_bf16(const GroupedGemmArgs& a, cudaStream_t st);
cudaError_t launch_gemm_fp8w(const GroupedGemmArgs& a, cudaStream_t st);
cudaError_t launch_gemm_mx(const GroupedGemmArgs& a, cudaStream_t st);
cudaError_t launch_gemm_nvfp4(const GroupedGemmArgs& a, cudaStream_t st);
}  // namespace gemm

cudaError_t launch_grouped_gemm(const GroupedGemmArgs& a, cudaStream_t st) {
    if (a.wfmt == MOE_W_NVFP4) {  // routed experts only; the caller runs the bf16 shared experts
        if (a.afmt == MOE_A_NVFP4) return gemm::launch_gemm_nvfp4(a, st);
        return cudaErrorNotSupported;
    }
    if (a.wfmt == MOE_W_FP4_E2M1_UE8M0_B32 || a.wfmt == MOE_W_MXFP4) {
        if (a.afmt == MOE_A_MXFP8 || a.afmt == MOE_A_FP8_E4M3_POW2_B128)
            return gemm::launch_gemm_mx(a, st);
        return cudaErrorNotSupported;
    }
    if (a.afmt != MOE_A_BF16) return cudaErrorNotSupported;
    if (a.wfmt == MOE_W_BF16) return gemm::launch_gemm_bf16(a, st);
    if (a.wfmt == MOE_W_FP8_E4M3_B128x128) return gemm::launch_gemm_fp8w(a, st);
    return cudaErrorNotSupported;
}

}  // namespace moe
