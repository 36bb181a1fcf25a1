/*
 * oracle.h -- plain, slow CPU reference of the hybrid Mamba-2 / attention
 * backbone frame step (TEST INFRASTRUCTURE ONLY).
 *
 * Only the test-suite, the smoke check and the benchmark's CPU-baseline leg
 * may load this library.  It shares no code, header or table with the CUDA
 * library; its inputs come from the seeded generator package (synth/) or from
 * its own quantizer.
 *
 * Sources of the arithmetic (page titles and sections):
 *  - "NemotronLabs VoiceChat 11B: GPTQ 3-bit LLM, MLX", introduction: the
 *    backbone is Nemotron-Nano-9B-v2 (56 layers mixing Mamba-2 and attention)
 *    with GPTQ weights in groups of 64; its per-frame step is bandwidth bound.
 *  - "NemotronLabs VoiceChat" (SGLang-Omni cookbook), overview: each 80 ms
 *    frame, the thinker decodes a text token and a function token greedily;
 *    backbone and KV cache in bf16.
 *  - The pages name the layer kinds but print no equations.  The plainest
 *    reading is used: the Mamba-2 layer of Dao & Gu, "Transformers are SSMs"
 *    (arXiv:2405.21060): causal depthwise conv1d over a ring of past inputs,
 *    dt = softplus(dt_raw + dt_bias), decay a = exp(A*dt) with A = -exp(A_log),
 *    state update h = a*h + dt*(x outer B), readout y = C.h + D*x, output
 *    gate y*silu(z) followed by a grouped RMSNorm; GQA attention with no
 *    positional encoding; a squared-ReLU MLP; pre-RMSNorm residual blocks.
 *    The chunked prefill follows that paper's block decomposition of the
 *    semiseparable matrix (its "SSD algorithm": diagonal blocks, chunk
 *    states, state passing, off-diagonal outputs).
 *
 * Precision: all arithmetic in double.  Two modes:
 *   OR_EXACT  -- no rounding at all (used for the invariant self-checks);
 *   OR_MIRROR -- rounds to bf16 at the points where the GPU path stores a
 *                bf16 tensor (listed in oracle.c, "storage points").
 */
#ifndef VC_ORACLE_H
#define VC_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { OR_BF16 = 0, OR_W8 = 1, OR_W4 = 2, OR_W3 = 3 };
enum { OR_EXACT = 0, OR_MIRROR = 1 };

/* A linear weight W[N][K] (y = W u).
 *   OR_BF16: q = uint16 bf16 bits, row-major [N][K]; scales/zeros unused.
 *   OR_W8  : q = int8 two's complement, 4 per uint32 little-endian, row-major
 *            [N][ceil(K/4)]; scales fp16 bits [N][ceil(K/group)]; symmetric.
 *   OR_W4/OR_W3: q = b-bit unsigned codes as a little-endian bit stream along K,
 *            [N][ceil(K*b/32)] uint32; scales fp16 [N][ng]; zeros b-bit stream
 *            [N][ceil(ng*b/32)], ng = ceil(K/group); w = s*(q - z).          */
typedef struct {
    int fmt, group, N, K;
    const void* q;
    const uint16_t* scales;
    const uint32_t* zeros;
} or_mat;

typedef struct {
    int d_model;
    const char* pattern;  /* one char per layer: 'M' Mamba-2, '*' attention, '-' MLP */
    int ssm_heads, ssm_head_dim, ssm_state, ssm_groups, conv_width, norm_groups;
    int attn_q_heads, attn_kv_heads, attn_head_dim;
    int mlp_hidden, vocab_text, vocab_func;
    double eps;
} or_config;

typedef struct {
    const float* norm;                     /* [d] pre-RMSNorm gamma */
    or_mat in_proj, out_proj;              /* Mamba-2: [E+Cx+H][d], [d][E] */
    const float *conv_w, *conv_b;          /* [Cx][W] (k = W-1 multiplies the newest row), [Cx] */
    const float *A_log, *D, *dt_bias;      /* [H] */
    const float* gnorm;                    /* [E] gated-RMSNorm gamma */
    or_mat qkv, o;                         /* attention: [(Hq+2Hk)Dh][d], [d][Hq*Dh] */
    or_mat up, down;                       /* MLP: [F][d], [d][F] */
} or_layer;

typedef struct {
    const or_layer* layers;                /* indexed by layer */
    const float* final_norm;               /* [d] */
    or_mat head_text, head_func;
} or_weights;

/* Session state, oracle's own logical layout (all double):
 *   ssm  [n_mamba][n_slots][H][P][N]
 *   conv [n_mamba][n_slots][W-1][Cx]   last W-1 pre-conv xBC rows, oldest first
 *   k, v [n_attn][n_slots][Hk][cap][Dh]
 *   ctx_len [n_slots] frames cached so far                                   */
typedef struct {
    int n_slots, kv_capacity;
    double *ssm, *conv, *k, *v;
    int32_t* ctx_len;
} or_state;

/* RTN group quantizer into the canonical packed format above; decisions in
 * fp32 exactly as documented in oracle.c.  w is fp32 [N][K]. */
void or_quantize(int fmt, int group, int N, int K, const float* w, uint32_t* q, uint16_t* scales,
                 uint32_t* zeros);
/* unpacked integer codes [N][K] (int32), zeros [N][ng] (0 for W8) and scales as
 * double [N][ng] */
void or_codes(const or_mat* W, int32_t* codes, int32_t* zeros, double* scales);
/* dequantized W as double [N][K] (exact: s*(q-z) with s an fp16 value) */
void or_dequant(const or_mat* W, double* out);
/* y[N] = W u, u[K] (double) */
void or_matvec(const or_mat* W, const double* u, double* y);

/* One decode step for B sessions.  x: bf16 bits [B][d]; slots: [B] or NULL (=0..B-1).
 * Outputs: tok_text/tok_func [B]; optional taps: hidden [n_layers+1][B][d]
 * (residual stream after each layer, entry 0 = input), logits [2][B][V]
 * (text then function).
 * Returns 0, or 1 if a session's cache is full (that session is skipped).
 * Pinned by: T steps == the brute-force full-sequence evaluation (every weight
 * format, one and two norm groups), ctx = 0 attention == v, the closed forms of
 * the test suite, and the mirror-mode storage points holding bf16 values. */
int or_step(const or_config* cfg, const or_weights* w, or_state* st, int B, const uint16_t* x,
            const int32_t* slots, int mode, int32_t* tok_text, int32_t* tok_func, double* hidden,
            double* logits);

/* One layer of the decode step, teacher-forced: the residual stream entering layer `layer` is
 * given (r_in [B][d], double) instead of being computed from the frame input.  Runs that layer
 * exactly as or_step does (same storage points), updating the layer's own state in st (its SSM
 * state and conv history, or its K/V row at position ctx_len), and writes the residual leaving the
 * layer to r_out [B][d].  ctx_len is not advanced.  slots as in or_step.
 * Returns 0; 1 if an attention layer meets a full cache; 2 for a bad layer index.
 * Pinned by: chaining it over every layer, then or_heads, equals or_step bit for bit, and by an
 * independent numpy restatement of one layer of each kind with the mirror-mode roundings. */
int or_layer_step(const or_config* cfg, const or_weights* w, or_state* st, int layer, int B,
                  const double* r_in, const int32_t* slots, int mode, double* r_out);

/* The final norm, both vocabulary heads and the greedy tokens of B rows, teacher-forced from the
 * residual stream r [B][d] leaving the last layer.  logits (optional) [2][B][max(Vt, Vf)]. */
void or_heads(const or_config* cfg, const or_weights* w, int B, const double* r, int mode, int32_t* tok_text,
              int32_t* tok_func, double* logits);

/* Prefill of T frames into one zero-initialised slot, layer by layer.
 * ssd_chunk = 0: Mamba-2 layers use the sequential recurrence;
 * ssd_chunk = Q > 0: they use the chunked SSD algorithm with chunk length Q.
 * hidden (optional): [n_layers+1][T][d].  Sets ctx_len[slot] = T.
 * Pinned by: the final SSM state, conv history and K/V equal T decode steps from
 * an empty slot. */
int or_prefill(const or_config* cfg, const or_weights* w, or_state* st, int slot, int T,
               const uint16_t* x, int mode, int ssd_chunk, double* hidden);

/* One layer of or_prefill, teacher-forced: r_in [T][d] is the residual stream of the T frames
 * entering layer `layer`; runs that layer as or_prefill does (frames ctx_len[slot] ..
 * ctx_len[slot]+T-1 of the slot), updates the layer's state in st and writes the residual leaving
 * the layer to r_out [T][d].  ctx_len is not advanced.  Returns 0, 1 if the frames do not fit the
 * cache, 2 for a bad layer index.  Pinned by: chaining it over every layer equals or_prefill. */
int or_prefill_layer(const or_config* cfg, const or_weights* w, or_state* st, int slot, int layer, int T,
                     const double* r_in, int mode, int ssd_chunk, double* r_out);

/* Isolated Mamba-2 mixer over T frames for one session (used by the kernel-level
 * checks): input zxbcdt [T][E+Cx+H] (double), state in/out ssm [H][P][N] and
 * conv history [W-1][Cx]; outputs the gated-norm input v [T][E] (= y*silu(z))
 * and y [T][E] (= y before gating).  ssd_chunk as in or_prefill.
 * Pinned by: chunked == sequential (Q in 1, 3, 16, 64, 70, 256; ragged T; a
 * non-zero initial state), the memoryless limit, pure decay at x = 0, and the
 * hand-worked scalar recurrence (tests/golden/ssm_scalar.txt). */
void or_mamba_mixer(const or_config* cfg, const or_layer* L, int T, const double* zxbcdt, double* ssm,
                    double* conv, int ssd_chunk, double* y_out, double* v_out);

/* Fused per-frame input of a session ("NVIDIA NemotronLabs VoiceChat 11B" blog, "Key design
 * decisions" 3: the user's channel and the agent's channels are summed into one input per frame):
 * out[b] = bf16( speech[b] + emb_text[tok_text[b]] + emb_func[tok_func[b]] ), the sum exact (in
 * double) and rounded once to nearest-even bf16; a token outside [0, V) adds nothing.
 * speech/out: bf16 bits [B][d]; emb_text [Vt][d], emb_func [Vf][d] bf16 bits.
 * Pinned by: no token gives the speech row itself, a zero speech row gives the
 * token's row, and a worked sum whose one rounding differs from two. */
void or_fuse_inputs(int B, int d, const uint16_t* speech, const uint16_t* emb_text, int Vt,
                    const uint16_t* emb_func, int Vf, const int32_t* tok_text, const int32_t* tok_func,
                    uint16_t* out);

/* Rounding helpers exposed for tests: RNE to bf16 / fp16 value, in double. */
double or_round_bf16(double v);
double or_round_fp16(double v);

/* threads the oracle's parallel loops use (1 without OpenMP) */
int or_threads(void);

#ifdef __cplusplus
}
#endif
#endif
