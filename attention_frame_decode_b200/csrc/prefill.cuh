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
};

size_t prefill_workspace_bytes(int d, int L, int E, int Cx, int H, int P, int N, int G, int Hq, int Hk, int Dh, int F,
                               int cap);
cudaError_t run_prefill(const PrefillCtx& c, const uint16_t* x, int T, int slot, cudaStream_t s);

}  // namespace vc
