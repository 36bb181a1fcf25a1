// gemv_bf16.cu -- instantiations of the streaming GEMV for bf16 weights.
#include "gemv_kernel.cuh"

namespace vc {
cudaError_t launch_gemv_bf16(const GemvLaunch& L, const GemvArgs& a, cudaStream_t s) { return launch_nt<FMT_BF16, 64>(L, a, s); }
}  // namespace vc
