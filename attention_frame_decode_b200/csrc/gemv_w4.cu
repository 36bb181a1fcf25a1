// gemv_w4.cu -- instantiations of the streaming GEMV for w4 weights.
#include "gemv_kernel.cuh"

namespace vc {
cudaError_t launch_gemv_w4(const GemvLaunch& L, const GemvArgs& a, cudaStream_t s) { return L.group == 128 ? launch_nt<FMT_W4, 128>(L, a, s) : launch_nt<FMT_W4, 64>(L, a, s); }
}  // namespace vc
