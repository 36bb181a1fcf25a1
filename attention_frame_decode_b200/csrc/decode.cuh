// decode.cuh -- per-frame mixer kernels of the decode step (Mamba-2 step, GQA decode attention)
// and the step-input kernel.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace vc {

struct InputArgs {
    const uint16_t* x;      // [B][d] bf16 frame inputs (with emb_t/emb_f: the speech embeddings)
    // optional fusion of the previous frame's tokens: x + emb_t[tok_t[b]] + emb_f[tok_f[b]] (a token
    // outside [0, V) adds nothing), summed in fp32 and rounded once to bf16
    const uint16_t* emb_t;  // [Vt][d] bf16 or null
    const uint16_t* emb_f;  // [Vf][d] bf16 or null
    const int* tok_t;       // [B] previous text tokens (the step's own output buffer)
    const int* tok_f;       // [B] previous function tokens
    int Vt, Vf;
    int B, d, unit_rows, n_units;
    float* r;               // [B][d] residual stream (fp32)
    const float* gamma;     // first layer's pre-norm gamma
    uint16_t* act;          // [B][act_ld]
    int act_ld, act_f16;
    float* parts;           // [B][n_units] sum of squares of r per unit of rows
    float* tap;             // optional hidden tap [B][d]
    const int* ctx_len;
    const int* slots;
    int cap;
    int* ok;                // [B]
    int* status;
};

struct MambaStepArgs {
    const uint16_t* zx;     // [B][zx_ld] bf16: z(E) | x(E) B(G*N) C(G*N) | dt_raw(H)
    int zx_ld;
    float* ssm;             // this layer, [n_slots][H][P][N]
    uint16_t* conv;         // this layer, [n_slots][W][Cx] bf16, frame t's row in slot t mod W
    const float *conv_w, *conv_b, *A_log, *D, *dt_bias, *gnorm;
    uint16_t* act;          // [B][act_ld] out_proj input: v * gamma_n
    int act_ld, act_f16;
    float* parts;           // [B][2H] sum of v^2 per (head, half)
    const int* ctx_len;
    const int* slots;
    const int* ok;
    int B, H, P, N, G, W, E, Cx;
    int* status;
};

struct AttnArgs {
    const uint16_t* q;      // [B][q_ld] bf16
    int q_ld;
    const uint16_t *kcache, *vcache;   // this layer, [n_slots][Hk][cap][Dh]
    int Hq, Hk, Dh, cap, max_splits;
    const int* ctx_len;
    const int* slots;
    const int* ok;
    float* scratch;         // [B][Hk][max_splits][GQ][Dh + 2]
    int* counters;          // [B][Hk]
    uint16_t* act;          // [B][act_ld] o_proj input
    int act_ld, act_f16;
    int B;
    int* status;
};

static constexpr int kAttnSplit = 128;  // keys per split

cudaError_t launch_input(const InputArgs& a, cudaStream_t s);
cudaError_t launch_mamba_step(const MambaStepArgs& a, int pdl, cudaStream_t s);
cudaError_t launch_attn_decode(const AttnArgs& a, int pdl, cudaStream_t s);

// shapes the two mixer kernels cover (their launch functions refuse the others)
bool mamba_step_supported(int P, int N);
bool attn_decode_supported(int Hq, int Hk, int Dh);

}  // namespace vc
