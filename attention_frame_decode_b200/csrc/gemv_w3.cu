// gemv_w3.cu -- instantiations of the streaming GEMV for w3 weights.
#include "gemv_kernel.cuh"

namespace vc {
cudaError_t launch_gemv_w3(const GemvLaunch& L, const GemvArgs& a, cudaStream_t s) { return L.group == 128 ? launch_nt<FMT_W3, 128>(L, a, s) : launch_nt<FMT_W3, 64>(L, a, s); }
}  // namespace vc
