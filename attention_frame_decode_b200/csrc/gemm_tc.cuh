// gemm_tc.cuh -- tcgen05 (5th-gen tensor core) GEMM for the prefill projections:
//   C[M][N] = A[M][K] . W[N][K]^T   (bf16 operands, fp32 accumulation in tensor memory)
// with fused epilogues.  A and W are row-major (K contiguous) and loaded by TMA.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace vc {

enum GemmEpi : int {
    GE_F32 = 0,        // out_f32[m][n] = acc
    GE_ROWSCALE = 1,   // out[m][n] = bf16(acc * row_scale[m])
    GE_RELU2 = 2,      // out[m][n] = bf16(relu(acc * row_scale[m])^2)
    GE_RESID = 3,      // out_f32[m][n] += acc   (residual stream)
    GE_QKV = 4,        // q rows -> out, k/v rows -> KV cache at frame t0 + m (bf16, scaled by row_scale)
};

struct GemmArgs {
    int f16;              // operands fp16 (1) or bf16 (0)
    int out_f16;          // GE_RELU2 outputs stored as fp16 bits of the bf16-rounded value (else bf16)
    const void* A;        // 16-bit [M][lda]
    int lda, M;
    const void* W;        // 16-bit [N][ldw]
    int ldw, N, K;
    const float* row_scale;   // [M] or null (1)
    uint16_t* out;            // bf16 [M][ldo]
    int ldo;
    float* out_f32;           // fp32 [M][ldo32]
    int ldo32;
    // GE_QKV
    int Hq, Hk, Dh, cap, t0;
    uint16_t *kcache, *vcache;   // this layer and slot: [Hk][cap][Dh]
    int* status;
};

cudaError_t launch_gemm_tc(int epi, const GemmArgs& a, cudaStream_t s);

}  // namespace vc
