/*
 * vc.h -- C ABI of libvc: the per-frame decode step and the opening-context prefill of the
 * hybrid Mamba-2 / attention LLM backbone of a full-duplex speech model, on one B200.
 *
 * What it computes (sources: the pages' titles and sections):
 *   - "NemotronLabs VoiceChat" (SGLang-Omni cookbook), intro and "Request parameters": every
 *     80 ms frame advances the thinker, which yields a text token and a function token
 *     per frame and always decodes greedily; backbone and KV cache run in bf16
 *     ("Known limitations").
 *   - "NemotronLabs VoiceChat 11B: GPTQ 3-bit LLM, MLX", intro and "Measurements": the LLM is
 *     Nemotron-Nano-9B-v2, a 56-layer hybrid of Mamba-2 and attention, GPTQ-quantized at group
 *     size 64 (3 or 4 bits); the LLM step is memory-bandwidth bound; the speech side's fused
 *     per-frame input embedding is the LLM's input ("Recipe").
 *   - "Nemotron Voicechat on DGX Spark" intro: GPTQ W8 weights for the same backbone.
 *   - "NVIDIA NemotronLabs VoiceChat 11B" (blog), "Key design decisions" 2-3: the backbone
 *     interleaves Mamba layers with attention layers; user and agent channels are summed into
 *     one input per frame.
 * The pages print no layer equations.  The plainest reading is used: a pre-RMSNorm residual
 * stack of Mamba-2 blocks (Dao & Gu, "Transformers are SSMs"), GQA attention without
 * positional encoding and squared-ReLU MLPs; two vocabulary heads after a final RMSNorm.
 *
 * Conventions for every call:
 *   - Device pointers are allocated and owned by the caller (e.g. PyTorch).  The library owns
 *     only host objects and CUDA graphs; it never allocates device memory.
 *   - All work is asynchronous on the caller's stream.  A call returns a host-detected error
 *     synchronously and launches nothing in that case.  Conditions only the device can see
 *     (a session whose KV cache is full, a non-finite logit) are OR-ed into the caller's
 *     device status word (VC_DEV_* bits); the affected session's step writes nothing and its
 *     tokens are -1.  No kernel traps or spins without a bound.
 *   - 16-byte alignment is required for every device pointer.
 *   - One backbone handle must not be used from two host threads at once.
 */
#ifndef VC_H
#define VC_H
#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* vc_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
    VC_OK = 0,
    VC_ERR_INVALID_ARG = 1,  /* bad pointer, size, alignment or shape */
    VC_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. a head group count > 16) */
    VC_ERR_CUDA = 3,         /* a CUDA runtime call failed; see vc_last_cuda_error() */
    VC_ERR_CAPACITY = 4,     /* host-visible capacity violation (e.g. prefill past kv_capacity) */
    VC_ERR_STATE = 5         /* the call is not valid in the current state */
} vc_status;

/* device status bits (OR-ed into vc_state.status) */
#define VC_DEV_CAPACITY 1   /* a session's KV cache was full; its step was skipped */
#define VC_DEV_NONFINITE 2  /* a non-finite logit was produced */
#define VC_DEV_TIMEOUT 4    /* an internal bounded wait ran out */

/* weight storage formats (weight-only, per-group along K) */
typedef enum {
    VC_W_BF16 = 0,       /* dense bf16 */
    VC_W_INT8_SYM = 1,   /* 8-bit symmetric codes, fp16 scale per group: w = s*q, q in [-127,127] */
    VC_W_INT4_ASYM = 2,  /* 4-bit codes + 4-bit zero + fp16 scale per group: w = s*(q - z) */
    VC_W_INT3_ASYM = 3   /* 3-bit codes + 3-bit zero + fp16 scale per group */
} vc_wfmt;

typedef struct {
    int d_model;
    const char* pattern;   /* one char per layer: 'M' Mamba-2, '*' attention, '-' MLP */
    int ssm_heads, ssm_head_dim, ssm_state, ssm_groups, conv_width, norm_groups;
    int attn_q_heads, attn_kv_heads, attn_head_dim;
    int mlp_hidden, vocab_text, vocab_func;
    float eps;             /* RMSNorm epsilon (pre-norm, gated norm, final norm) */
    int wfmt, group_size;  /* format of every linear weight of the layers */
    int head_fmt;          /* format of the two vocabulary heads (same group_size) */
    int max_batch;         /* sessions per vc_step call, 1..16 */
    int kv_capacity;       /* frames per session the KV cache holds */
    int n_slots;           /* session slots in the state buffers */
} vc_config;

/* A linear weight y = W u, W[N][K], in the device layout written by vc_quantize_weight /
 * vc_pack_bf16_weight / vc_pack_weight (size vc_weight_bytes).  data: device pointer. */
typedef struct {
    const void* data;
    int fmt, group, N, K;
} vc_qmat;

/* Per-layer weights (device pointers, fp32 vectors); unused members of other layer kinds may
 * be NULL.  Mamba-2: in_proj [E+Cx+H][d] with rows [z(E) | x(E) B(G*N) C(G*N) | dt(H)],
 * out_proj [d][E], conv_w [Cx][W] (column W-1 multiplies the newest frame), conv_b [Cx],
 * A_log, D, dt_bias [H], gnorm [E].  Attention: qkv [(Hq+2Hk)*Dh][d] rows [q | k | v],
 * o [d][Hq*Dh].  MLP: up [F][d], down [d][F].  norm [d]: the layer's pre-RMSNorm gamma. */
typedef struct {
    const float* norm;
    vc_qmat in_proj, out_proj;
    const float *conv_w, *conv_b, *A_log, *D, *dt_bias, *gnorm;
    vc_qmat qkv, o;
    vc_qmat up, down;
} vc_layer_weights;

typedef struct {
    const vc_layer_weights* layers;  /* host array of n_layers entries (copied at create) */
    const float* final_norm;         /* [d] */
    vc_qmat head_text, head_func;
} vc_weights;

/* Session state (device, caller-owned), n_slots sessions:
 *   ssm  fp32 [n_mamba][n_slots][H][P][N]
 *   conv bf16 [n_mamba][n_slots][W][Cx]: ring of the last W pre-conv rows [x|B|C]; the row of
 *        frame t (0-based, counted per session) is kept in ring slot t mod W
 *   k, v bf16 [n_attn][n_slots][Hk][kv_capacity][Dh]
 *   ctx_len int32 [n_slots]: frames processed so far per session
 *   status int32 [1]: device status word (VC_DEV_* bits), never cleared by the library */
typedef struct {
    float* ssm;
    void* conv;
    void* k;
    void* v;
    int32_t* ctx_len;
    int32_t* status;
} vc_state;

typedef struct vc_backbone vc_backbone;

/* ---- weight preparation (not on the per-frame path) ---------------------------------- */

/* bytes of the device layout of an [N][K] weight in format fmt with group size group
 * (64 or 128; ignored for VC_W_BF16); 0 for an unsupported combination */
size_t vc_weight_bytes(int fmt, int group, int N, int K);

/* Round-to-nearest group quantization of fp32 w[N][K] (device) into the device layout out
 * (device, vc_weight_bytes).  Decisions in IEEE fp32: W8 s = fp16(amax/127),
 * q = clamp(rne(w/s), +-127); W4/W3 s = fp16((max-min)/Q), z = clamp(rne(-min/s), 0, Q),
 * q = clamp(rne(w/s) + z, 0, Q); s := 1 when it would round to 0.  VC_W_BF16 rounds to bf16.
 * Source: GPTQ-style weight-only groups of "NemotronLabs VoiceChat 11B: GPTQ 3-bit LLM, MLX",
 * "Recipe"; GPTQ's calibration itself is not part of this call. */
vc_status vc_quantize_weight(int fmt, int group, int N, int K, const float* w, void* out, vc_stream_t stream);

/* bf16 w[N][K] (device) -> VC_W_BF16 device layout */
vc_status vc_pack_bf16_weight(int N, int K, const uint16_t* w, void* out, vc_stream_t stream);

/* Already-quantized GPTQ-style weights (device) -> device layout.  q: codes as a little-endian
 * bit stream along K per row, [N][ceil(K*b/32)] uint32 (W8: int8 two's complement);
 * scales fp16 [N][ceil(K/group)]; zeros (W4/W3) b-bit stream [N][ceil(ngroups*b/32)]. */
vc_status vc_pack_weight(int fmt, int group, int N, int K, const uint32_t* q, const uint16_t* scales,
                         const uint32_t* zeros, void* out, vc_stream_t stream);

/* test/debug: dequantized weight as fp32 [N][K] (device); exact s*(q - z) */
vc_status vc_debug_dequant(const vc_qmat* w, float* out, vc_stream_t stream);

/* ---- backbone ----------------------------------------------------------------------- */

/* bytes of device workspace a backbone with this config needs (caller allocates) */
size_t vc_workspace_bytes(const vc_config* cfg);

/* Creates the backbone of the frame step: the 56-layer hybrid of Mamba-2 and attention layers
 * (in the order of cfg->pattern) with its two vocabulary heads ("NemotronLabs VoiceChat 11B: GPTQ
 * 3-bit LLM, MLX", introduction: Nemotron-Nano-9B-v2, 56 layers; "NVIDIA NemotronLabs VoiceChat
 * 11B" blog, "Key design decisions" 2: Mamba layers interleaved with attention layers;
 * "NemotronLabs VoiceChat" (SGLang-Omni cookbook), overview: a text head and a function head).
 * Validates cfg and weights, carves the workspace (device, vc_workspace_bytes, zeroed here on
 * `stream`) and returns a handle.  Weight and workspace memory must stay valid until
 * vc_destroy.  Nothing is launched except the workspace clear.  VC_ERR_UNSUPPORTED (before any
 * CUDA call) for shapes the decode kernels do not cover: an attention head dim that does not
 * divide 256, or a Mamba-2 head with P/2 + 2N > 512.  VC_ERR_INVALID_ARG for a bad config,
 * missing or misaligned pointers or a workspace that is too small; *out is NULL then. */
vc_status vc_backbone_create(const vc_config* cfg, const vc_weights* weights, void* workspace,
                             size_t workspace_bytes, vc_stream_t stream, vc_backbone** out);

/* options: VC_OPT_FRAME (1 = run each decode frame as one launch of the persistent frame kernel
 * where it covers the backbone's formats and shapes; 0 = one kernel per operation, default),
 * VC_OPT_GRAPH (per-kernel path: 1 = capture and replay one CUDA graph per call signature,
 * default; 0 = launch the kernels directly), VC_OPT_PDL (per-kernel path: 1 = programmatic
 * dependent launch, default), VC_OPT_GEMV_SHAPE (per-kernel path, projections of up to 8 rows:
 * how the streaming GEMV occupies an SM; 0 = two 8-warp CTAs per SM, each with half of the ring
 * budget (default); 1 = one 8-warp CTA per SM with half of the ring budget, so that a CTA of the
 * next projection fits beside it and, under programmatic dependent launch, issues its first
 * weight copies while this one runs; 2 = one 8-warp CTA per SM with the whole ring budget
 * (deeper rings, no room beside it).  On a B200, 0 gives the fastest step (fewer resident warps
 * per SM cost more than the prefetch or the deeper rings gain).  The results agree up to the order
 * of fp32 sums; other values give VC_ERR_INVALID_ARG) */
#define VC_OPT_GRAPH 1
#define VC_OPT_PDL 2
#define VC_OPT_FRAME 3
#define VC_OPT_GEMV_SHAPE 4
vc_status vc_set_option(vc_backbone* h, int option, int value);

/* 1 if a vc_step of B rows on this backbone runs as one launch of the frame kernel (the option is
 * on and the kernel covers the backbone's weight formats and shapes at this B), else 0 */
int vc_uses_frame_kernel(const vc_backbone* h, int B);

/* One decode frame for B sessions (1 <= B <= max_batch): each session's fused frame input
 * goes through every layer and both heads and yields one greedy text token and one greedy
 * function token ("NemotronLabs VoiceChat" (SGLang-Omni cookbook), overview: the thinker advances
 * once per 80 ms frame and emits a text and a function token, decoded greedily; "NemotronLabs
 * VoiceChat 11B: GPTQ 3-bit LLM, MLX", measurement bullets: this per-frame LLM step).
 * x: bf16 [B][d_model] (device) fused frame inputs.  slots: int32 [B] (device) session slot of
 * each row, or NULL for 0..B-1 (slots must be distinct).  tok_text, tok_func: int32 [B]
 * (device) greedy tokens (lowest index on ties).  Advances ctx_len[slot] by 1 for every
 * session whose cache had room.  Runs as one launch of the frame kernel where it covers the
 * backbone (vc_uses_frame_kernel), else one kernel per operation; a device-side VC_DEV_TIMEOUT
 * (a bounded wait gave up) leaves the workspace's internal counters undefined, and the backbone
 * must then be destroyed and created again. */
vc_status vc_step(vc_backbone* h, const void* x, int B, const int32_t* slots, const vc_state* state,
                  int32_t* tok_text, int32_t* tok_func, vc_stream_t stream);

/* Token embeddings for the fused-input step (device, caller-owned): bf16 [vocab_text][d_model]
 * and [vocab_func][d_model]. */
typedef struct {
    const void* emb_text;
    const void* emb_func;
} vc_token_embeddings;

/* One frame whose input is fused on the device from this frame's speech embedding and the
 * tokens the previous frame emitted -- the user and agent channels summed into one input per
 * frame ("NVIDIA NemotronLabs VoiceChat 11B" blog, "Key design decisions" 3; the fused per-frame
 * embedding of "NemotronLabs VoiceChat 11B: GPTQ 3-bit LLM, MLX", Recipe) -- so that a session
 * runs frame after frame without a host round trip.  For each row b:
 *   x[b] = bf16( speech[b] + emb_text[tok_text[b]] + emb_func[tok_func[b]] )
 * summed in fp32 in that order and rounded once; a token outside [0, vocab) (e.g. -1 before the
 * first frame, or from a skipped session) adds nothing.  tok_text / tok_func (device, int32 [B])
 * hold the previous tokens on entry and this frame's tokens on return (the same buffers feed the
 * next call).  speech: bf16 [B][d_model] (device).  Otherwise as vc_step. */
vc_status vc_step_fused(vc_backbone* h, const void* speech, const vc_token_embeddings* emb, int B,
                        const int32_t* slots, const vc_state* state, int32_t* tok_text, int32_t* tok_func,
                        vc_stream_t stream);

/* The same frame with host buffers: copies x (host, ideally pinned) to the device, runs the
 * step and copies the tokens back into tok_text/tok_func (host), all on `stream`; the caller
 * synchronizes the stream before reading the tokens. */
vc_status vc_step_host(vc_backbone* h, const void* x_host, int B, const int32_t* slots, const vc_state* state,
                       int32_t* tok_text_host, int32_t* tok_func_host, vc_stream_t stream);

/* Prefill of T frames x bf16 [T][d_model] (device) into session `slot` -- the opening context a
 * streaming session consumes before its frames ("NemotronLabs VoiceChat 11B: GPTQ 3-bit LLM,
 * MLX", Recipe: the prompt is taken in as one block before the caller's speech).  The slot
 * starts empty: whatever it held is overwritten -- a used slot is not refused with VC_ERR_STATE,
 * since telling a used slot from an empty one would need a read of the device's ctx_len.  Mamba-2 layers run the chunked SSD (Dao & Gu, "Transformers are SSMs",
 * chunk 256) over the frames, attention layers causal GQA; the call writes the final SSM state,
 * the conv ring (the last W-1 frames' rows, frame t in slot t mod W, the other slot zero) and
 * KV rows 0..T-1 of the slot and sets ctx_len[slot] = T.  No tokens are produced.
 * 1 <= T <= kv_capacity (else VC_ERR_CAPACITY / VC_ERR_INVALID_ARG, nothing launched).  Uses the
 * backbone's workspace (prefill scratch sized for kv_capacity frames); asynchronous on stream.
 * It may run concurrently with vc_step calls of other slots on other streams (they use disjoint
 * parts of the workspace); two vc_prefill calls on one backbone must not overlap in time. */
vc_status vc_prefill(vc_backbone* h, const void* x, int T, int slot, const vc_state* state, vc_stream_t stream);

/* test/debug taps for the next vc_step calls (device fp32 buffers or NULL):
 * hidden [n_layers+1][B][d] residual stream after each layer (entry 0 = input),
 * logits [2][B][max(vocab_text, vocab_func)] (text, function). */
vc_status vc_debug_set_taps(vc_backbone* h, float* hidden, float* logits);

/* test/debug tap for the next vc_step calls (device fp32 buffer or NULL): zx
 * [n_mamba][B][E+Cx+H], the in_proj output of each Mamba-2 layer before its bf16 storage rounding
 * (the mixer consumes the bf16 rounding, to nearest even, of these values). */
vc_status vc_debug_set_zx_taps(vc_backbone* h, float* zx);

/* test/debug taps for the next vc_prefill calls (device buffers or NULL), for the T of that call;
 * the caller sizes them: hidden fp32 [n_layers+1][T][d], the residual stream of every prefilled
 * frame after each layer (entry 0 = input); zx bf16 [n_mamba][T][E+Cx+H], each Mamba-2 layer's
 * in_proj output as its mixer consumes it. */
vc_status vc_debug_set_prefill_taps(vc_backbone* h, float* hidden, void* zx);

/* test/debug: one Mamba-2 mixer step (the kernel vc_step runs for a Mamba-2 layer) on given
 * inputs.  zx: bf16 [B][E+Cx+H] in_proj outputs; ssm/conv: this layer's state slices
 * ([n_slots][H][P][N] fp32, [n_slots][W][Cx] bf16); slots [B] or NULL; ctx_len [n_slots] is read,
 * not advanced.  Outputs act bf16 [B][E] = bf16(y*silu(z)*gnorm) and parts fp32 [B][2H], the sum of
 * (y*silu(z))^2 over each half of each head. */
vc_status vc_debug_mamba_step(const vc_config* cfg, const vc_layer_weights* layer, const void* zx, int B,
                              const int32_t* slots, float* ssm, void* conv, const int32_t* ctx_len, void* act,
                              float* parts, int32_t* status, vc_stream_t stream);

/* test/measurement: y = W u with the decode step's streaming GEMV kernel.
 * act: 16-bit [B][act_ld] (device; bf16 bits for VC_W_BF16 weights, fp16 bits for quantized
 * ones), act_ld a multiple of 128 and >= K rounded up to 128, columns K..act_ld-1 zero;
 * 1 <= B <= 16.  out: fp32 [B][N] (device).  scratch: device buffer of vc_gemv_scratch_bytes()
 * bytes, zero on first use; every call returns the counters and accumulators it uses to zero.
 * Split row units are summed as in vc_step (fp32 reductions into accumulators, order varying
 * from run to run) when their accumulators fit the scratch, else in worker order. */
size_t vc_gemv_scratch_bytes(void);
vc_status vc_debug_gemv(const vc_qmat* w, const void* act, int act_ld, int B, float* out, void* scratch,
                        vc_stream_t stream);

/* test: the prefill's Mamba-2 mixer of one layer over T frames of one session that starts empty
 * (the kernels vc_prefill runs between a Mamba-2 layer's two projections): causal conv + SiLU,
 * chunked SSD with chunks of 256 frames, gated RMSNorm.
 * zx: bf16 [T][E+Cx+H] in_proj outputs (device).  Outputs (device): ssm fp32 [H][P][N] final state,
 * conv bf16 [W][Cx] ring (frame t in slot t mod W, the other slots zero), y fp32 [T][E] the SSM
 * output before gating, act bf16 [T][E] = bf16(y*silu(z) * rsqrt(mean over the norm group + eps)
 * * gnorm).  scratch: device, vc_debug_mamba_prefill_scratch_bytes(cfg, T) bytes, 16-byte aligned. */
size_t vc_debug_mamba_prefill_scratch_bytes(const vc_config* cfg, int T);
vc_status vc_debug_mamba_prefill(const vc_config* cfg, const vc_layer_weights* layer, const void* zx, int T, float* ssm,
                                 void* conv, float* y, void* act, void* scratch, vc_stream_t stream);

/* test/measurement: out = A . W^T with the prefill's tensor-core GEMM (tcgen05, fp32 accumulation
 * in tensor memory), the contraction of the prefill projections over the frames.
 * A: [M][lda] and W: [N][ldw] 16-bit row-major (device, 16-byte aligned; bf16 bits, or fp16 bits
 * when f16 != 0), K a multiple of 8, lda and ldw multiples of 8 and >= K.  out: fp32 [M][ldo]
 * (device).  status: device word; VC_DEV_TIMEOUT is or-ed in if an internal wait ran out. */
vc_status vc_debug_gemm(const void* A, int lda, int M, const void* W, int ldw, int N, int K, int f16, float* out,
                        int ldo, int32_t* status, vc_stream_t stream);

/* The GEMV of vc_debug_gemv for callers that cannot allocate device memory (a per-frame
 * real-time loop, where cudaMalloc/cudaFree can synchronize the device and stall the frame; a
 * host whose device memory belongs to another allocator).  No counterpart in the method's
 * sources: an operational variant of the decode GEMV, nothing the model computes differs.
 * Same arguments and argument checks as vc_debug_gemv, without the scratch argument: the scratch
 * is a static device array of vc_gemv_noalloc_scratch_bytes() = 4.25 MiB + 256 B in the library
 * (4 MiB of partial sums, 65536 arrival counters and a status word, the counters and status zero
 * at load), and the launch uses at most 32 SMs' worth of CTAs.  Results equal vc_debug_gemv's
 * up to the order of the fp32 sums (a different grid splits the rows differently), not bit for
 * bit.  A weight with more than 65536 row units (16*R rows each) returns VC_ERR_CAPACITY.  Every
 * call looks up the array's device address on the current device (a runtime query; nothing is
 * allocated).  All calls on a device share the array: calls that overlap in time race and give
 * wrong results, so callers order them.  A completed call leaves the counters zero; a call whose
 * bounded wait for a weight copy gave up ORs VC_DEV_TIMEOUT into the status word and may leave
 * counters non-zero, after which results are not valid until vc_gemv_noalloc_reset. */
size_t vc_gemv_noalloc_scratch_bytes(void);
vc_status vc_debug_gemv_noalloc(const vc_qmat* w, const void* act, int act_ld, int B, float* out,
                                vc_stream_t stream);
/* the status word of the no-allocation GEMV (VC_DEV_* bits of every call since load or the last
 * reset) into *status (host); synchronizes `stream` */
vc_status vc_gemv_noalloc_status(int32_t* status, vc_stream_t stream);
/* zeroes the no-allocation GEMV's counters and status word on `stream` (a device memset) */
vc_status vc_gemv_noalloc_reset(vc_stream_t stream);

/* Releases the handle and what the library owns for it (host objects, CUDA graphs, its streams
 * and events); the caller's device memory (weights, state, workspace) is left to the caller.
 * Work the handle queued must be complete (or its stream synchronized) before the call.  The
 * handle's lifetime spans the sessions of one served model ("NemotronLabs VoiceChat"
 * (SGLang-Omni cookbook), overview: one thinker serves the frames of its sessions). */
void vc_destroy(vc_backbone* h);

const char* vc_status_string(vc_status s);
const char* vc_last_cuda_error(void);

#ifdef __cplusplus
}
#endif
#endif
