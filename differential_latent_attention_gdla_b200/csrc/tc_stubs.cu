// tc_stubs.cu -- tensor-core launchers not yet available in this build.
#include "kernels.h"
namespace gdla {
bool gemm_tc_supported(const GemmParams&) { return false; }
cudaError_t launch_gemm_tc(const GemmParams&, int*, cudaStream_t) { return cudaErrorNotSupported; }
bool attn_tc_supported(const AttnParams&, gdla_dtype) { return false; }
cudaError_t launch_attn_tc(const AttnParams&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace gdla
