// gemv_w8.cu -- instantiations of the streaming GEMV for w8 weights.
#include "gemv_kernel.cuh"

namespace vc {
cudaError_t launch_gemv_w8(const GemvLaunch& L, const GemvArgs& a, cudaStream_t s) { return L.group == 128 ? launch_nt<FMT_W8, 128>(L, a, s) : launch_nt<FMT_W8, 64>(L, a, s); }
}  // namespace vc
