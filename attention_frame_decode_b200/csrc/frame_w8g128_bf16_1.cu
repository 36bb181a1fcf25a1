// frame_w8g128_bf16_1.cu -- the frame kernel for one pair of weight formats (one translation unit
// per pair, so that they compile in parallel).
#include "frame_kernel.cuh"

namespace vc {
cudaError_t frame_launch_w8g128_bf16_1(const FrameParams& p, int num_sms, size_t smem, cudaStream_t s) {
    return frame_launch_t<FMT_W8, 128, FMT_BF16, 64, 1>(p, num_sms, smem, s);
}
}  // namespace vc
