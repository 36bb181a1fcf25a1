// prefill.cuh -- opening-context prefill of one session (chunked SSD + causal GQA + GEMMs).
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/vc.h"

namespace vc {

struct PrefillCtx {
    const vc_config* cfg;
    const vc_layer_weights* layers;
    const float* final_norm;
    int d, L, H, P, N, G, W, E, Cx, NG, Hq, Hk, Dh, F, cap, n_slots, num_sms;
    uint8_t* ws;
    size_t ws_bytes;
    float* ssm;
    uint16_t *conv, *k, *v;
    int32_t* ctx_len;
    int32_t* status;
    float* tap;   // test tap or null: residual stream [L+1][T][d] (entry 0 = input, l+1 after layer l)
    uint16_t* tap_zx;   // test tap or null: bf16 in_proj outputs [n_mamba][T][E+Cx+H]
    cudaStream_t side;   // weight unpacking, one GEMM ahead of the caller's stream
    cudaEvent_t ev[5];   // unpacked[2], gemm done[2], call start
};

// Mamba-2 mixer of one layer over T frames from zero state: conv (ring written), chunked SSD
// (final state written to ssm), y (before gating) and the gated-norm output act
struct PfMixer {
    int T, E, Cx, H, P, N, G, W, NG, f16;
    float eps;
    const vc_layer_weights* Lw;
    const uint16_t* zx;                              // bf16 [T][E+Cx+H]
    float *xc, *dt, *lam, *y, *schunk;               // scratch (carve_mixer); y fp32 [T][E]
    uint16_t* xc16;                                  // fp16 copy of xc [T][Cx] (tensor-core operands)
    uint16_t* sin16;                                 // bf16 state entering each chunk [nch][H][P][N]
    float* ssm;                                      // [H][P][N]
    uint16_t* ring;                                  // [W][Cx]
    uint16_t* act;                                   // [T][act_ld]
    int act_ld;
    int* status;                                     // device status word (bounded waits of the tcgen05 kernels)
};
size_t prefill_mixer_scratch_bytes(int T, int E, int Cx, int H, int P, int N);
void carve_mixer(PfMixer& m, uint8_t* base);
cudaError_t prefill_mixer(const PfMixer& m, cudaStream_t s);

// chunk outputs of the chunked SSD on tcgen05 (ssd_tc.cu); shapes: N in {64, 128}, P a multiple of
// 16 up to 128
bool ssd_out_tc_supported(int N, int P, int E, int Cx);
// chunk states (and the within-chunk cumulative log decay) on tcgen05; shapes: N = 128, P a
// multiple of 16 up to 128
bool ssd_state_tc_supported(int N, int P, int E, int Cx);
cudaError_t launch_ssd_state_tc(const float* xc, const float* dt, const float* A_log, int T, int H, int P, int N, int G,
                                int E, int Cx, float* lam, float* schunk, int* status, cudaStream_t s);
cudaError_t launch_ssd_out_tc(const uint16_t* xc16, const uint16_t* sin16, const float* dt, const float* lam,
                              const float* Dv, float* y, int T, int H, int P, int N, int G, int E, int Cx, int* status,
                              cudaStream_t s);

size_t prefill_workspace_bytes(int d, int L, int E, int Cx, int H, int P, int N, int G, int Hq, int Hk, int Dh, int F,
                               int cap);
cudaError_t run_prefill(const PrefillCtx& c, const uint16_t* x, int T, int slot, cudaStream_t s);

}  // namespace vc
