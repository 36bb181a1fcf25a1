// api.cu -- the C ABI of libvc (include/vc.h): weight preparation, backbone handle, the
// per-frame step as one CUDA graph of ~145 kernels chained with programmatic dependent launch.
#include <cuda_runtime.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <map>
#include <memory>
#include <string>
#include <tuple>
#include <vector>

#include "../../include/vc.h"
#include "common.cuh"
#include "decode.cuh"
#include "frame.cuh"
#include "gemm_tc.cuh"
#include "gemv.cuh"
#include "gemv_core.cuh"
#include "layout.cuh"
#include "prefill.cuh"

using namespace vc;

static thread_local char g_cuda_err[256] = "";

static vc_status cuda_fail(cudaError_t e, const char* where) {
    snprintf(g_cuda_err, sizeof(g_cuda_err), "%s: %s", where, cudaGetErrorString(e));
    return VC_ERR_CUDA;
}
namespace vc {
// error recording for the C ABI functions defined in other translation units
vc_status record_cuda_failure(cudaError_t e, const char* where) { return cuda_fail(e, where); }
}  // namespace vc

#define CK(call)                                         \
    do {                                                 \
        cudaError_t e_ = (call);                         \
        if (e_ != cudaSuccess) return cuda_fail(e_, #call); \
    } while (0)

static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

static bool fmt_ok(int fmt, int group) {
    if (fmt == VC_W_BF16) return true;
    if (fmt < 0 || fmt > 3) return false;
    return group == 64 || group == 128;
}

// ------------------------------------------------------------------------------------------
// weight preparation
// ------------------------------------------------------------------------------------------
extern "C" size_t vc_weight_bytes(int fmt, int group, int N, int K) {
    if (!fmt_ok(fmt, group) || N <= 0 || K <= 0) return 0;
    return (size_t)mat_geom(fmt, fmt == VC_W_BF16 ? 64 : group, N, K).bytes;
}

extern "C" vc_status vc_quantize_weight(int fmt, int group, int N, int K, const float* w, void* out,
                                        vc_stream_t stream) {
    if (!fmt_ok(fmt, group) || N <= 0 || K <= 0 || !w || !out || !aligned16(out)) return VC_ERR_INVALID_ARG;
    CK(launch_quantize(fmt, fmt == VC_W_BF16 ? 64 : group, N, K, w, (uint8_t*)out, (cudaStream_t)stream));
    return VC_OK;
}

extern "C" vc_status vc_pack_bf16_weight(int N, int K, const uint16_t* w, void* out, vc_stream_t stream) {
    if (N <= 0 || K <= 0 || !w || !out || !aligned16(out)) return VC_ERR_INVALID_ARG;
    CK(launch_pack_bf16(N, K, w, (uint8_t*)out, (cudaStream_t)stream));
    return VC_OK;
}

extern "C" vc_status vc_pack_weight(int fmt, int group, int N, int K, const uint32_t* q, const uint16_t* scales,
                                    const uint32_t* zeros, void* out, vc_stream_t stream) {
    if (fmt == VC_W_BF16 || !fmt_ok(fmt, group) || N <= 0 || K <= 0 || !q || !scales || !out || !aligned16(out))
        return VC_ERR_INVALID_ARG;
    if (fmt != VC_W_INT8_SYM && !zeros) return VC_ERR_INVALID_ARG;
    CK(launch_pack_canonical(fmt, group, N, K, q, scales, zeros, (uint8_t*)out, (cudaStream_t)stream));
    return VC_OK;
}

extern "C" vc_status vc_debug_dequant(const vc_qmat* w, float* out, vc_stream_t stream) {
    if (!w || !w->data || !out || !fmt_ok(w->fmt, w->group) || w->N <= 0 || w->K <= 0) return VC_ERR_INVALID_ARG;
    CK(launch_dequant(w->fmt, w->fmt == VC_W_BF16 ? 64 : w->group, w->N, w->K, (const uint8_t*)w->data, out,
                      (cudaStream_t)stream));
    return VC_OK;
}

// ------------------------------------------------------------------------------------------
// backbone
// ------------------------------------------------------------------------------------------
struct Dims {
    int d, L, H, P, N, G, W, E, Cx, NG, Hq, Hk, Dh, F, Vt, Vf, nm, na, B, cap, slots;
    int zx_rows, qkv_rows, attn_splits;
};

struct Workspace {
    float* r;
    uint16_t *act_a, *act_m, *act_o, *act_h;
    int lda, ldm, ldo, ldh;
    uint16_t *zx, *q;
    float *parts_r, *parts_g;
    int n_units_d;
    int* ok;
    float* partials;
    int* counters;
    float* accum;
    float* attn_scratch;
    int* attn_counters;
    unsigned long long* keys;
    int* done;
    uint16_t* x_stage;
    int32_t* tok_stage;
    uint8_t* prefill;   // prefill scratch (see prefill.cuh)
    size_t prefill_bytes;
    FrameProgram* prog;  // the frame kernel's program (device copy)
    int* fk_sync;        // [0] barrier arrivals, [1] abort flag of the frame kernel
};

struct GraphKey {
    int B;
    const void* slots;
    vc_state st;
    const void* tt;
    const void* tf;
    const float* th;
    const float* tl;
    const float* tz;
    const void* et;   // token embeddings of the fused-input variant (null: plain inputs)
    const void* ef;
    bool operator<(const GraphKey& o) const {
        return memcmp(this, &o, sizeof(GraphKey)) < 0;
    }
};

struct vc_backbone {
    vc_config cfg;
    std::string pattern;
    Dims D;
    std::vector<vc_layer_weights> layers;
    vc_weights w;
    Workspace ws;
    int num_sms = 148;
    int use_graph = 1, use_pdl = 1, use_frame = 0;
    int gemv_shape = 0;   // VC_OPT_GEMV_SHAPE
    // the frame kernel's program as last uploaded, and the call signature it was built for
    std::unique_ptr<FrameProgram> host_prog;
    GraphKey prog_key;
    bool prog_valid = false;
    float* tap_hidden = nullptr;
    float* tap_logits = nullptr;
    float* tap_prefill = nullptr;
    float* tap_zx = nullptr;
    uint16_t* tap_prefill_zx = nullptr;
    struct Graph {
        cudaGraph_t graph;
        cudaGraphExec_t exec;
        cudaGraphNode_t input_node;   // the step-input kernel (the graph's only root)
        const void* x;                // frame input the input node currently reads
    };
    std::map<GraphKey, Graph> graphs;
    cudaStream_t capture_stream = nullptr;
    cudaStream_t prefill_side = nullptr;   // unpacks the next layer weight while a GEMM runs
    cudaEvent_t pf_ev[5] = {};              // unpacked[2], gemm done[2], call start
};

static size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

static bool dims_from_cfg(const vc_config* c, Dims& D) {
    if (!c || !c->pattern) return false;
    D.d = c->d_model;
    D.L = (int)strlen(c->pattern);
    D.H = c->ssm_heads; D.P = c->ssm_head_dim; D.N = c->ssm_state; D.G = c->ssm_groups; D.W = c->conv_width;
    D.E = D.H * D.P; D.Cx = D.E + 2 * D.G * D.N; D.NG = c->norm_groups;
    D.Hq = c->attn_q_heads; D.Hk = c->attn_kv_heads; D.Dh = c->attn_head_dim;
    D.F = c->mlp_hidden; D.Vt = c->vocab_text; D.Vf = c->vocab_func;
    D.nm = D.na = 0;
    for (int l = 0; l < D.L; ++l) {
        char k = c->pattern[l];
        if (k == 'M') D.nm++;
        else if (k == '*') D.na++;
        else if (k != '-') return false;
    }
    D.B = c->max_batch; D.cap = c->kv_capacity; D.slots = c->n_slots;
    D.zx_rows = D.E + D.Cx + D.H;
    D.qkv_rows = (D.Hq + 2 * D.Hk) * D.Dh;
    // attention split scratch, sized for the smaller splits of the two decode paths
    D.attn_splits = (D.cap + kFkAttnSplit - 1) / kFkAttnSplit;
    if (D.L < 1 || D.d <= 0 || D.d % 64 || D.B < 1 || D.B > 16 || D.slots < D.B || D.cap < 1) return false;
    if (D.nm) {
        if (D.H <= 0 || D.P <= 0 || D.P % 2 || D.N <= 0 || D.N % 4 || D.G <= 0 || D.H % D.G || D.W < 2 || D.W > 8)
            return false;
        if (D.NG <= 0 || D.NG > 16 || D.E % D.NG || (2 * D.H) % D.NG) return false;
        if ((D.E / D.NG) % 128) return false;   // norm groups align with GEMV k-steps
        if (D.E % 64) return false;
    }
    if (D.na) {
        if (D.Hk <= 0 || D.Hq % D.Hk || D.Hq / D.Hk > 8 || D.Dh % 16 || D.Dh > 256 || D.Dh < 32) return false;
    }
    if (D.Vt <= 0 || D.Vf <= 0) return false;
    return true;
}

// fp32 accumulators of the step's split GEMV units: the largest launch's units x R x NT x 128
static size_t accum_floats(const vc_config* c, const Dims& D) {
    const int NT = D.B > 8 ? 2 : 1;
    auto units = [&](int fmt, int N) {
        const int grp = fmt == VC_W_BF16 ? 64 : c->group_size;
        const LayoutInfo L = layout_info(fmt, grp);
        return (size_t)((N + 16 * L.R - 1) / (16 * L.R)) * L.R * NT * 128;
    };
    size_t m = 0;
    for (int N : {D.zx_rows, D.qkv_rows, D.F, D.d}) m = std::max(m, units(c->wfmt, N));
    m = std::max(m, units(c->head_fmt, D.Vt) + units(c->head_fmt, D.Vf));
    return m;
}

extern "C" size_t vc_workspace_bytes(const vc_config* cfg) {
    Dims D;
    if (!dims_from_cfg(cfg, D)) return 0;
    const int B = D.B;
    size_t total = 0;
    auto add = [&](size_t bytes) { total = align_up(total, 256) + bytes; };
    const int lda = round_up(D.d, 128), ldm = round_up(D.E > 0 ? D.E : 64, 128),
              ldo = round_up(D.Hq * D.Dh > 0 ? D.Hq * D.Dh : 64, 128), ldh = round_up(D.F > 0 ? D.F : 64, 128);
    add((size_t)B * D.d * 4);                 // r
    add((size_t)B * lda * 2);                 // act_a
    add((size_t)B * ldm * 2);                 // act_m
    add((size_t)B * ldo * 2);                 // act_o
    add((size_t)B * ldh * 2);                 // act_h
    add((size_t)B * D.zx_rows * 2);           // zx
    add((size_t)B * D.Hq * D.Dh * 2);         // q
    add((size_t)B * ((D.d + 15) / 16) * 4);   // parts_r (one per 16-row unit)
    add((size_t)B * 2 * D.H * 4 + 16);        // parts_g
    add((size_t)16 * 4);                      // ok
    add(gemv_partials_bytes(256));            // partials (any SM count up to 256)
    add(gemv_counter_ints() * 4);             // counters
    add((size_t)B * D.Hk * D.attn_splits * (D.Hq / (D.Hk ? D.Hk : 1)) * (D.Dh + 2) * 4 + 16);  // attention splits
    add((size_t)B * D.Hk * 4 + 16);           // attention counters
    add(2 * 16 * 8);                          // keys
    add(16);                                  // done
    add((size_t)B * D.d * 2);                 // x staging
    add(2 * 16 * 4);                          // token staging
    add(prefill_workspace_bytes(D.d, D.L, D.E, D.Cx, D.H, D.P, D.N, D.G, D.Hq, D.Hk, D.Dh, D.F, D.cap));
    add(accum_floats(cfg, D) * 4);            // split-unit accumulators
    add(sizeof(FrameProgram));                // the frame kernel's program
    add(256);                                 // its barrier and abort words
    return align_up(total, 256);
}

static void carve(vc_backbone* h, uint8_t* base) {
    Dims& D = h->D;
    Workspace& W = h->ws;
    const int B = D.B;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        off = align_up(off, 256);
        uint8_t* p = base + off;
        off += bytes;
        return p;
    };
    W.lda = round_up(D.d, 128);
    W.ldm = round_up(D.E > 0 ? D.E : 64, 128);
    W.ldo = round_up(D.Hq * D.Dh > 0 ? D.Hq * D.Dh : 64, 128);
    W.ldh = round_up(D.F > 0 ? D.F : 64, 128);
    W.r = (float*)take((size_t)B * D.d * 4);
    W.act_a = (uint16_t*)take((size_t)B * W.lda * 2);
    W.act_m = (uint16_t*)take((size_t)B * W.ldm * 2);
    W.act_o = (uint16_t*)take((size_t)B * W.ldo * 2);
    W.act_h = (uint16_t*)take((size_t)B * W.ldh * 2);
    W.zx = (uint16_t*)take((size_t)B * D.zx_rows * 2);
    W.q = (uint16_t*)take((size_t)B * D.Hq * D.Dh * 2);
    W.parts_r = (float*)take((size_t)B * ((D.d + 15) / 16) * 4);
    W.parts_g = (float*)take((size_t)B * 2 * D.H * 4 + 16);
    W.ok = (int*)take(16 * 4);
    W.partials = (float*)take(gemv_partials_bytes(256));
    W.counters = (int*)take(gemv_counter_ints() * 4);
    W.attn_scratch = (float*)take((size_t)B * D.Hk * D.attn_splits * (D.Hq / (D.Hk ? D.Hk : 1)) * (D.Dh + 2) * 4 + 16);
    W.attn_counters = (int*)take((size_t)B * D.Hk * 4 + 16);
    W.keys = (unsigned long long*)take(2 * 16 * 8);
    W.done = (int*)take(16);
    W.x_stage = (uint16_t*)take((size_t)B * D.d * 2);
    W.tok_stage = (int32_t*)take(2 * 16 * 4);
    W.prefill_bytes = prefill_workspace_bytes(D.d, D.L, D.E, D.Cx, D.H, D.P, D.N, D.G, D.Hq, D.Hk, D.Dh, D.F, D.cap);
    W.prefill = take(W.prefill_bytes);
    W.accum = (float*)take(accum_floats(&h->cfg, D) * 4);
    W.prog = (FrameProgram*)take(sizeof(FrameProgram));
    W.fk_sync = (int*)take(256);
}

static bool qmat_ok(const vc_qmat& m, int fmt, int group, int N, int K) {
    return m.data && aligned16(m.data) && m.fmt == fmt && (fmt == VC_W_BF16 || m.group == group) && m.N == N &&
           m.K == K;
}

extern "C" vc_status vc_backbone_create(const vc_config* cfg, const vc_weights* weights, void* workspace,
                                        size_t workspace_bytes, vc_stream_t stream, vc_backbone** out) {
    if (!out) return VC_ERR_INVALID_ARG;
    *out = nullptr;
    Dims D;
    if (!dims_from_cfg(cfg, D)) return VC_ERR_INVALID_ARG;
    if (!fmt_ok(cfg->wfmt, cfg->group_size) || !fmt_ok(cfg->head_fmt, cfg->group_size)) return VC_ERR_INVALID_ARG;
    // shapes the decode kernels do not cover are refused here rather than at the first step
    if ((D.na && !attn_decode_supported(D.Hq, D.Hk, D.Dh)) || (D.nm && !mamba_step_supported(D.P, D.N)))
        return VC_ERR_UNSUPPORTED;
    if (!weights || !weights->layers || !weights->final_norm || !workspace || !aligned16(workspace))
        return VC_ERR_INVALID_ARG;
    if (workspace_bytes < vc_workspace_bytes(cfg)) return VC_ERR_INVALID_ARG;
    const int fmt = cfg->wfmt, grp = cfg->group_size;
    for (int l = 0; l < D.L; ++l) {
        const vc_layer_weights& L = weights->layers[l];
        if (!L.norm) return VC_ERR_INVALID_ARG;
        char k = cfg->pattern[l];
        if (k == 'M') {
            if (!qmat_ok(L.in_proj, fmt, grp, D.zx_rows, D.d) || !qmat_ok(L.out_proj, fmt, grp, D.d, D.E))
                return VC_ERR_INVALID_ARG;
            if (!L.conv_w || !L.conv_b || !L.A_log || !L.D || !L.dt_bias || !L.gnorm) return VC_ERR_INVALID_ARG;
        } else if (k == '*') {
            if (!qmat_ok(L.qkv, fmt, grp, D.qkv_rows, D.d) || !qmat_ok(L.o, fmt, grp, D.d, D.Hq * D.Dh))
                return VC_ERR_INVALID_ARG;
        } else {
            if (!qmat_ok(L.up, fmt, grp, D.F, D.d) || !qmat_ok(L.down, fmt, grp, D.d, D.F)) return VC_ERR_INVALID_ARG;
        }
    }
    if (!qmat_ok(weights->head_text, cfg->head_fmt, grp, D.Vt, D.d) ||
        !qmat_ok(weights->head_func, cfg->head_fmt, grp, D.Vf, D.d))
        return VC_ERR_INVALID_ARG;

    vc_backbone* h = new vc_backbone();
    h->cfg = *cfg;
    h->pattern = cfg->pattern;
    h->cfg.pattern = h->pattern.c_str();
    h->D = D;
    h->layers.assign(weights->layers, weights->layers + D.L);
    h->w = *weights;
    h->w.layers = h->layers.data();
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (h->num_sms > 256) h->num_sms = 256;
    carve(h, (uint8_t*)workspace);
    cudaError_t e = cudaMemsetAsync(workspace, 0, vc_workspace_bytes(cfg), (cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&h->capture_stream, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&h->prefill_side, cudaStreamNonBlocking);
    for (int i = 0; i < 5 && e == cudaSuccess; ++i) e = cudaEventCreateWithFlags(&h->pf_ev[i], cudaEventDisableTiming);
    if (e != cudaSuccess) {
        const vc_status st = cuda_fail(e, "vc_backbone_create");
        vc_destroy(h);   // releases whichever streams and events were created
        return st;
    }
    *out = h;
    return VC_OK;
}

static void clear_graphs(vc_backbone* h) {
    for (auto& kv : h->graphs) {
        cudaGraphExecDestroy(kv.second.exec);
        cudaGraphDestroy(kv.second.graph);
    }
    h->graphs.clear();
}

extern "C" vc_status vc_set_option(vc_backbone* h, int option, int value) {
    if (!h) return VC_ERR_INVALID_ARG;
    if (option == VC_OPT_GRAPH) h->use_graph = value != 0;
    else if (option == VC_OPT_PDL) h->use_pdl = value != 0;
    else if (option == VC_OPT_FRAME) h->use_frame = value != 0;
    else if (option == VC_OPT_GEMV_SHAPE && value >= 0 && value <= 2) h->gemv_shape = value;
    else return VC_ERR_INVALID_ARG;
    clear_graphs(h);
    h->prog_valid = false;
    return VC_OK;
}

extern "C" vc_status vc_debug_set_prefill_taps(vc_backbone* h, float* hidden, void* zx) {
    if (!h) return VC_ERR_INVALID_ARG;
    h->tap_prefill = hidden;
    h->tap_prefill_zx = (uint16_t*)zx;
    return VC_OK;
}

extern "C" vc_status vc_debug_set_zx_taps(vc_backbone* h, float* zx) {
    if (!h) return VC_ERR_INVALID_ARG;
    h->tap_zx = zx;
    clear_graphs(h);
    h->prog_valid = false;
    return VC_OK;
}

extern "C" vc_status vc_debug_set_taps(vc_backbone* h, float* hidden, float* logits) {
    if (!h) return VC_ERR_INVALID_ARG;
    h->tap_hidden = hidden;
    h->tap_logits = logits;
    clear_graphs(h);
    h->prog_valid = false;
    return VC_OK;
}

static GemvMat gm(const vc_qmat& q) {
    MatGeom G = mat_geom(q.fmt, q.fmt == VC_W_BF16 ? 64 : q.group, q.N, q.K);
    return GemvMat{(const uint8_t*)q.data, q.N, q.K, G.NU, G.KT};
}

// Receives the step's sequence of operations: launched as kernels one by one (recorded into a
// graph, or launched directly), or collected into the frame kernel's program.
struct StepSink {
    virtual cudaError_t input(const InputArgs& a) = 0;
    virtual cudaError_t gemv(const GemvLaunch& l, const GemvArgs& a) = 0;
    virtual cudaError_t mamba(const MambaStepArgs& a) = 0;
    virtual cudaError_t attn(const AttnArgs& a) = 0;
    virtual ~StepSink() = default;
};

struct LaunchSink : StepSink {
    cudaStream_t s;
    int pdl;
    LaunchSink(cudaStream_t s_, int pdl_) : s(s_), pdl(pdl_) {}
    cudaError_t input(const InputArgs& a) override { return launch_input(a, s); }
    cudaError_t gemv(const GemvLaunch& l, const GemvArgs& a) override { return launch_gemv(l, a, s); }
    cudaError_t mamba(const MambaStepArgs& a) override { return launch_mamba_step(a, pdl, s); }
    cudaError_t attn(const AttnArgs& a) override { return launch_attn_decode(a, pdl, s); }
};

struct ProgramSink : StepSink {
    FrameProgram& P;
    int cap;
    explicit ProgramSink(FrameProgram& p, int cap_) : P(p), cap(cap_) { P.n_ops = P.n_gemv = P.n_mamba = P.n_attn = 0; }
    cudaError_t op(int kind, int idx) {
        if (P.n_ops >= kFkMaxOps) return cudaErrorInvalidValue;
        P.ops[P.n_ops++] = FkOp{kind, idx};
        return cudaSuccess;
    }
    cudaError_t input(const InputArgs& a) override {
        P.input = a;
        return op(FK_INPUT, 0);
    }
    cudaError_t gemv(const GemvLaunch& l, const GemvArgs& a) override {
        if (P.n_gemv >= kFkMaxGemv) return cudaErrorInvalidValue;
        FkGemv& G = P.gemv[P.n_gemv];
        memset(&G, 0, sizeof(G));
        G.a = a;
        G.epi = l.epi;
        G.head = l.epi == EPI_ARGMAX;
        return op(FK_GEMV, P.n_gemv++);
    }
    cudaError_t mamba(const MambaStepArgs& a) override {
        if (P.n_mamba >= kFkMaxMix || P.n_gemv < 1) return cudaErrorInvalidValue;
        // the frame kernel accumulates the gated norm's sums; the in_proj op before clears them
        FkGemv& prev = P.gemv[P.n_gemv - 1];
        prev.zero_buf = a.parts;
        prev.zero_n = a.B * 2 * a.H;
        P.mamba[P.n_mamba] = a;
        return op(FK_MAMBA, P.n_mamba++);
    }
    cudaError_t attn(const AttnArgs& a) override {
        if (P.n_attn >= kFkMaxMix) return cudaErrorInvalidValue;
        AttnArgs f = a;
        f.max_splits = (cap + kFkAttnSplit - 1) / kFkAttnSplit;
        P.attn[P.n_attn] = f;
        cudaError_t e = op(FK_ATTN, P.n_attn);
        if (e == cudaSuccess) e = op(FK_ATTN_MERGE, P.n_attn);
        P.n_attn++;
        return e;
    }
};

// the step's sequence of operations
static cudaError_t record_step(vc_backbone* h, const void* x, int B, const int32_t* slots, const vc_state* st,
                               int32_t* tt, int32_t* tf, const vc_token_embeddings* emb, StepSink& sink) {
    const Dims& D = h->D;
    const Workspace& W = h->ws;
    const int fmt = h->cfg.wfmt, grp = h->cfg.group_size;
    const int act_f16 = act_f16_for(fmt);
    const LayoutInfo LI = layout_info(fmt, fmt == VC_W_BF16 ? 64 : grp);
    const int unit_rows = 16 * LI.R;
    const int n_units_d = (D.d + unit_rows - 1) / unit_rows;
    cudaError_t e;

    InputArgs ia{};
    ia.x = (const uint16_t*)x; ia.B = B; ia.d = D.d; ia.unit_rows = unit_rows; ia.n_units = n_units_d;
    ia.r = W.r; ia.gamma = h->layers[0].norm; ia.act = W.act_a; ia.act_ld = W.lda; ia.act_f16 = act_f16;
    ia.parts = W.parts_r; ia.tap = h->tap_hidden; ia.ctx_len = st->ctx_len; ia.slots = slots; ia.cap = D.cap;
    ia.ok = W.ok; ia.status = st->status;
    if (emb) {
        ia.emb_t = (const uint16_t*)emb->emb_text; ia.emb_f = (const uint16_t*)emb->emb_func;
        ia.tok_t = tt; ia.tok_f = tf; ia.Vt = D.Vt; ia.Vf = D.Vf;
    }
    if ((e = sink.input(ia)) != cudaSuccess) return e;

    InScale pre{};
    pre.parts = W.parts_r; pre.n_groups = 1; pre.per_group = n_units_d; pre.group_cols = W.lda;
    pre.inv_width = 1.0f / D.d; pre.eps = h->cfg.eps;

    GemvArgs base{};
    base.nmat = 1; base.B = B; base.partials = W.partials; base.counters = W.counters; base.accum = W.accum;
    base.status = st->status;
    base.slots = slots; base.ok = W.ok; base.ctx_len = st->ctx_len;
    GemvLaunch gl{};
    gl.fmt = fmt; gl.group = grp; gl.num_sms = h->num_sms; gl.pdl = h->use_pdl; gl.shape = h->gemv_shape;

    auto resid_epi = [&](GemvArgs& a, int l) {
        a.resid = W.r; a.resid_ld = D.d;
        const bool last = l == D.L - 1;
        a.gamma_next = last ? h->w.final_norm : h->layers[l + 1].norm;
        a.act_next = W.act_a; a.act_next_ld = W.lda;
        a.act_next_f16 = last ? act_f16_for(h->cfg.head_fmt) : act_f16;
        a.parts_next = W.parts_r; a.parts_ld = n_units_d;
        a.tap = h->tap_hidden ? h->tap_hidden + (size_t)(l + 1) * B * D.d : nullptr;
        a.tap_ld = D.d;
    };

    int mi = 0, ai = 0;
    for (int l = 0; l < D.L; ++l) {
        const vc_layer_weights& Lw = h->layers[l];
        const char kind = h->cfg.pattern[l];
        if (kind == 'M') {
            GemvArgs a = base;
            a.mat[0] = gm(Lw.in_proj); a.act = W.act_a; a.act_ld = W.lda; a.insc = pre;
            a.out = W.zx; a.out_ld = D.zx_rows; a.out_f16 = 0;
            if (h->tap_zx) { a.tap = h->tap_zx + (size_t)mi * B * D.zx_rows; a.tap_ld = D.zx_rows; }
            gl.epi = EPI_STORE;
            if ((e = sink.gemv(gl, a)) != cudaSuccess) return e;

            MambaStepArgs ma{};
            ma.zx = W.zx; ma.zx_ld = D.zx_rows;
            ma.ssm = st->ssm + (size_t)mi * D.slots * D.H * D.P * D.N;
            ma.conv = (uint16_t*)st->conv + (size_t)mi * D.slots * D.W * D.Cx;
            ma.conv_w = Lw.conv_w; ma.conv_b = Lw.conv_b; ma.A_log = Lw.A_log; ma.D = Lw.D; ma.dt_bias = Lw.dt_bias;
            ma.gnorm = Lw.gnorm; ma.act = W.act_m; ma.act_ld = W.ldm; ma.act_f16 = act_f16; ma.parts = W.parts_g;
            ma.ctx_len = st->ctx_len; ma.slots = slots; ma.ok = W.ok; ma.B = B; ma.H = D.H; ma.P = D.P; ma.N = D.N;
            ma.G = D.G; ma.W = D.W; ma.E = D.E; ma.Cx = D.Cx; ma.status = st->status;
            if ((e = sink.mamba(ma)) != cudaSuccess) return e;

            a = base;
            a.mat[0] = gm(Lw.out_proj); a.act = W.act_m; a.act_ld = W.ldm;
            a.insc.parts = W.parts_g; a.insc.n_groups = D.NG; a.insc.per_group = 2 * D.H / D.NG;
            a.insc.group_cols = D.E / D.NG; a.insc.inv_width = (float)D.NG / D.E; a.insc.eps = h->cfg.eps;
            resid_epi(a, l);
            gl.epi = EPI_RESID;
            if ((e = sink.gemv(gl, a)) != cudaSuccess) return e;
            mi++;
        } else if (kind == '*') {
            GemvArgs a = base;
            a.mat[0] = gm(Lw.qkv); a.act = W.act_a; a.act_ld = W.lda; a.insc = pre;
            a.q_out = W.q; a.q_ld = D.Hq * D.Dh;
            const size_t kvl = (size_t)ai * D.slots * D.Hk * D.cap * D.Dh;
            a.kcache = (uint16_t*)st->k + kvl; a.vcache = (uint16_t*)st->v + kvl;
            a.Hq = D.Hq; a.Hk = D.Hk; a.Dh = D.Dh; a.cap = D.cap;
            gl.epi = EPI_QKV;
            if ((e = sink.gemv(gl, a)) != cudaSuccess) return e;

            AttnArgs aa{};
            aa.q = W.q; aa.q_ld = D.Hq * D.Dh; aa.kcache = a.kcache; aa.vcache = a.vcache;
            aa.Hq = D.Hq; aa.Hk = D.Hk; aa.Dh = D.Dh; aa.cap = D.cap; aa.max_splits = (D.cap + kAttnSplit - 1) / kAttnSplit;
            aa.ctx_len = st->ctx_len; aa.slots = slots; aa.ok = W.ok; aa.scratch = W.attn_scratch;
            aa.counters = W.attn_counters; aa.act = W.act_o; aa.act_ld = W.ldo; aa.act_f16 = act_f16; aa.B = B;
            aa.status = st->status;
            if ((e = sink.attn(aa)) != cudaSuccess) return e;

            a = base;
            a.mat[0] = gm(Lw.o); a.act = W.act_o; a.act_ld = W.ldo;
            resid_epi(a, l);
            gl.epi = EPI_RESID;
            if ((e = sink.gemv(gl, a)) != cudaSuccess) return e;
            ai++;
        } else {
            GemvArgs a = base;
            a.mat[0] = gm(Lw.up); a.act = W.act_a; a.act_ld = W.lda; a.insc = pre;
            a.out = W.act_h; a.out_ld = W.ldh; a.out_f16 = act_f16;
            gl.epi = EPI_RELU2;
            if ((e = sink.gemv(gl, a)) != cudaSuccess) return e;
            a = base;
            a.mat[0] = gm(Lw.down); a.act = W.act_h; a.act_ld = W.ldh;
            resid_epi(a, l);
            gl.epi = EPI_RESID;
            if ((e = sink.gemv(gl, a)) != cudaSuccess) return e;
        }
    }
    // final norm is folded into the last residual epilogue (gamma_final) + the input scale here
    GemvArgs a = base;
    a.nmat = 2;
    a.mat[0] = gm(h->w.head_text);
    a.mat[1] = gm(h->w.head_func);
    a.act = W.act_a; a.act_ld = W.lda; a.insc = pre;
    a.keys = W.keys; a.tok[0] = tt; a.tok[1] = tf; a.ctx_len_mut = st->ctx_len; a.done = W.done;
    a.tap = h->tap_logits; a.tap_ld = D.Vt > D.Vf ? D.Vt : D.Vf;
    GemvLaunch hl = gl;
    hl.fmt = h->cfg.head_fmt;
    hl.epi = EPI_ARGMAX;
    return sink.gemv(hl, a);
}

static vc_status check_step_args(vc_backbone* h, const void* x, int B, const vc_state* st, const void* tt,
                                 const void* tf) {
    if (!h || !x || !st || !tt || !tf) return VC_ERR_INVALID_ARG;
    if (B < 1 || B > h->D.B) return VC_ERR_INVALID_ARG;
    if (!st->ctx_len || !st->status) return VC_ERR_INVALID_ARG;
    if (h->D.nm && (!st->ssm || !st->conv || !aligned16(st->ssm) || !aligned16(st->conv))) return VC_ERR_INVALID_ARG;
    if (h->D.na && (!st->k || !st->v || !aligned16(st->k) || !aligned16(st->v))) return VC_ERR_INVALID_ARG;
    return VC_OK;
}

static FrameGeom frame_geom(const vc_backbone* h, int B) {
    FrameGeom g{};
    g.lfmt = h->cfg.wfmt;
    g.lgrp = g.lfmt == VC_W_BF16 ? 64 : h->cfg.group_size;
    g.hfmt = h->cfg.head_fmt;
    g.hgrp = g.hfmt == VC_W_BF16 ? 64 : h->cfg.group_size;
    g.nt = B > 8 ? 2 : 1;
    return g;
}

// the whole frame as one launch of the frame kernel; cudaErrorNotSupported where it has no
// instantiation for the backbone's formats and shapes (the caller then launches per kernel)
static cudaError_t run_frame(vc_backbone* h, const void* x, int B, const int32_t* slots, const vc_state* st,
                             int32_t* tt, int32_t* tf, cudaStream_t s, const vc_token_embeddings* emb) {
    const FrameGeom g = frame_geom(h, B);
    if (!frame_supported(g, h->D.na ? h->D.Hq / h->D.Hk : 1, h->D.na ? h->D.Dh : 64, h->D.nm ? h->D.N : 4))
        return cudaErrorNotSupported;
    int slots_per_warp = 0, slot_bytes = 0;
    size_t smem = 0;
    frame_ring(g, &slots_per_warp, &slot_bytes, &smem);
    GraphKey key;
    memset(&key, 0, sizeof(key));
    key.B = B; key.slots = slots; key.st = *st;
    key.th = h->tap_hidden; key.tl = h->tap_logits; key.tz = h->tap_zx;
    if (emb) { key.et = emb->emb_text; key.ef = emb->emb_func; }
    cudaError_t e;
    if (!h->prog_valid || memcmp(&key, &h->prog_key, sizeof(key)) != 0) {
        if (!h->host_prog) h->host_prog.reset(new FrameProgram());
        ProgramSink ps(*h->host_prog, h->D.cap);
        // the frame input and the token buffers are the launch's (FrameParams), not the program's
        if ((e = record_step(h, x, B, slots, st, tt, tf, emb, ps)) != cudaSuccess) return e;
        if ((e = cudaMemcpyAsync(h->ws.prog, h->host_prog.get(), sizeof(FrameProgram), cudaMemcpyHostToDevice, s)))
            return e;
        h->prog_key = key;
        h->prog_valid = true;
    }
    FrameParams fp{};
    fp.prog = h->ws.prog;
    fp.x = (const uint16_t*)x;
    fp.tok_t = tt;
    fp.tok_f = tf;
    fp.barrier = (unsigned*)h->ws.fk_sync;   // words 0 and 2; zero since create (workspace clear)
    fp.abort = h->ws.fk_sync + 1;
    fp.status = st->status;
    fp.slots = slots_per_warp;
    fp.slot_bytes = slot_bytes;
    return launch_frame(g, fp, h->num_sms, s);
}

static vc_status run_step(vc_backbone* h, const void* x, int B, const int32_t* slots, const vc_state* st, int32_t* tt,
                          int32_t* tf, cudaStream_t s, const vc_token_embeddings* emb = nullptr) {
    if (h->use_frame) {
        const cudaError_t e = run_frame(h, x, B, slots, st, tt, tf, s, emb);
        if (e == cudaSuccess) return VC_OK;
        if (e != cudaErrorNotSupported) return cuda_fail(e, "vc_step frame kernel");
    }
    if (!h->use_graph) {
        LaunchSink ls(s, h->use_pdl);
        cudaError_t e = record_step(h, x, B, slots, st, tt, tf, emb, ls);
        return e == cudaSuccess ? VC_OK : cuda_fail(e, "vc_step launch");
    }
    GraphKey key;
    memset(&key, 0, sizeof(key));
    key.B = B; key.slots = slots; key.st = *st; key.tt = tt; key.tf = tf;
    key.th = h->tap_hidden; key.tl = h->tap_logits; key.tz = h->tap_zx;
    if (emb) { key.et = emb->emb_text; key.ef = emb->emb_func; }
    auto it = h->graphs.find(key);
    if (it == h->graphs.end()) {
        if (h->graphs.size() > 64) clear_graphs(h);
        cudaStream_t cs = h->capture_stream;
        CK(cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal));
        LaunchSink ls(cs, h->use_pdl);
        cudaError_t e = record_step(h, x, B, slots, st, tt, tf, emb, ls);
        cudaGraph_t g = nullptr;
        cudaError_t e2 = cudaStreamEndCapture(cs, &g);
        if (e != cudaSuccess) {
            if (g) cudaGraphDestroy(g);
            return cuda_fail(e, "vc_step capture");
        }
        if (e2 != cudaSuccess) return cuda_fail(e2, "cudaStreamEndCapture");
        // the input kernel is the only root node
        size_t nroots = 0;
        CK(cudaGraphGetRootNodes(g, nullptr, &nroots));
        if (nroots != 1) {
            cudaGraphDestroy(g);
            return cuda_fail(cudaErrorUnknown, "vc_step graph shape");
        }
        cudaGraphNode_t root;
        CK(cudaGraphGetRootNodes(g, &root, &nroots));
        cudaGraphExec_t ex = nullptr;
        e = cudaGraphInstantiate(&ex, g, 0);
        if (e != cudaSuccess) {
            cudaGraphDestroy(g);
            return cuda_fail(e, "cudaGraphInstantiate");
        }
        it = h->graphs.emplace(key, vc_backbone::Graph{g, ex, root, x}).first;
    }
    vc_backbone::Graph& G = it->second;
    if (G.x != x) {
        // same call signature, new frame input: patch the input kernel's argument in place
        cudaKernelNodeParams kp;
        CK(cudaGraphKernelNodeGetParams(G.input_node, &kp));
        InputArgs ia = *reinterpret_cast<InputArgs*>(kp.kernelParams[0]);
        ia.x = (const uint16_t*)x;
        void* args[1] = {&ia};
        kp.kernelParams = args;
        CK(cudaGraphExecKernelNodeSetParams(G.exec, G.input_node, &kp));
        G.x = x;
    }
    CK(cudaGraphLaunch(G.exec, s));
    return VC_OK;
}

extern "C" int vc_uses_frame_kernel(const vc_backbone* h, int B) {
    if (!h || B < 1 || B > h->D.B || !h->use_frame) return 0;
    return frame_supported(frame_geom(h, B), h->D.na ? h->D.Hq / h->D.Hk : 1, h->D.na ? h->D.Dh : 64,
                           h->D.nm ? h->D.N : 4) ? 1 : 0;
}

extern "C" vc_status vc_step(vc_backbone* h, const void* x, int B, const int32_t* slots, const vc_state* state,
                             int32_t* tok_text, int32_t* tok_func, vc_stream_t stream) {
    vc_status st = check_step_args(h, x, B, state, tok_text, tok_func);
    if (st != VC_OK) return st;
    if (!aligned16(x)) return VC_ERR_INVALID_ARG;
    return run_step(h, x, B, slots, state, tok_text, tok_func, (cudaStream_t)stream);
}

extern "C" vc_status vc_step_fused(vc_backbone* h, const void* speech, const vc_token_embeddings* emb, int B,
                                   const int32_t* slots, const vc_state* state, int32_t* tok_text, int32_t* tok_func,
                                   vc_stream_t stream) {
    vc_status st = check_step_args(h, speech, B, state, tok_text, tok_func);
    if (st != VC_OK) return st;
    if (!emb || !emb->emb_text || !emb->emb_func || !aligned16(speech)) return VC_ERR_INVALID_ARG;
    return run_step(h, speech, B, slots, state, tok_text, tok_func, (cudaStream_t)stream, emb);
}

extern "C" vc_status vc_step_host(vc_backbone* h, const void* x_host, int B, const int32_t* slots,
                                  const vc_state* state, int32_t* tok_text_host, int32_t* tok_func_host,
                                  vc_stream_t stream) {
    vc_status st = check_step_args(h, x_host, B, state, tok_text_host, tok_func_host);
    if (st != VC_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    CK(cudaMemcpyAsync(h->ws.x_stage, x_host, (size_t)B * h->D.d * 2, cudaMemcpyHostToDevice, s));
    st = run_step(h, h->ws.x_stage, B, slots, state, h->ws.tok_stage, h->ws.tok_stage + 16, s);
    if (st != VC_OK) return st;
    CK(cudaMemcpyAsync(tok_text_host, h->ws.tok_stage, (size_t)B * 4, cudaMemcpyDeviceToHost, s));
    CK(cudaMemcpyAsync(tok_func_host, h->ws.tok_stage + 16, (size_t)B * 4, cudaMemcpyDeviceToHost, s));
    return VC_OK;
}

extern "C" vc_status vc_prefill(vc_backbone* h, const void* x, int T, int slot, const vc_state* state,
                                vc_stream_t stream) {
    if (!h || !x || !state || !aligned16(x)) return VC_ERR_INVALID_ARG;
    if (T < 1 || slot < 0 || slot >= h->D.slots) return VC_ERR_INVALID_ARG;
    if (T > h->D.cap) return VC_ERR_CAPACITY;
    if (!state->ctx_len || !state->status) return VC_ERR_INVALID_ARG;
    PrefillCtx c{};
    c.cfg = &h->cfg;
    c.layers = h->layers.data();
    c.final_norm = h->w.final_norm;
    c.d = h->D.d; c.L = h->D.L; c.H = h->D.H; c.P = h->D.P; c.N = h->D.N; c.G = h->D.G; c.W = h->D.W;
    c.E = h->D.E; c.Cx = h->D.Cx; c.NG = h->D.NG; c.Hq = h->D.Hq; c.Hk = h->D.Hk; c.Dh = h->D.Dh; c.F = h->D.F;
    c.cap = h->D.cap; c.n_slots = h->D.slots; c.num_sms = h->num_sms;
    c.ws = h->ws.prefill; c.ws_bytes = h->ws.prefill_bytes;
    c.ssm = state->ssm; c.conv = (uint16_t*)state->conv; c.k = (uint16_t*)state->k; c.v = (uint16_t*)state->v;
    c.ctx_len = state->ctx_len; c.status = state->status;
    c.tap = h->tap_prefill;
    c.tap_zx = h->tap_prefill_zx;
    c.side = h->prefill_side;
    for (int i = 0; i < 5; ++i) c.ev[i] = h->pf_ev[i];
    cudaError_t e = run_prefill(c, (const uint16_t*)x, T, slot, (cudaStream_t)stream);
    if (e == cudaErrorNotSupported) return VC_ERR_UNSUPPORTED;
    if (e == cudaErrorInvalidValue) return VC_ERR_INVALID_ARG;
    return e == cudaSuccess ? VC_OK : cuda_fail(e, "vc_prefill");
}

extern "C" vc_status vc_debug_mamba_step(const vc_config* cfg, const vc_layer_weights* layer, const void* zx, int B,
                                         const int32_t* slots, float* ssm, void* conv, const int32_t* ctx_len,
                                         void* act, float* parts, int32_t* status, vc_stream_t stream) {
    Dims D;
    if (!dims_from_cfg(cfg, D) || !D.nm || !layer || !zx || !ssm || !conv || !ctx_len || !act || !parts || !status)
        return VC_ERR_INVALID_ARG;
    if (B < 1 || B > D.slots || !aligned16(ssm)) return VC_ERR_INVALID_ARG;
    MambaStepArgs ma{};
    ma.zx = (const uint16_t*)zx; ma.zx_ld = D.zx_rows; ma.ssm = ssm; ma.conv = (uint16_t*)conv;
    ma.conv_w = layer->conv_w; ma.conv_b = layer->conv_b; ma.A_log = layer->A_log; ma.D = layer->D;
    ma.dt_bias = layer->dt_bias; ma.gnorm = layer->gnorm; ma.act = (uint16_t*)act; ma.act_ld = D.E; ma.act_f16 = 0;
    ma.parts = parts; ma.ctx_len = ctx_len; ma.slots = slots; ma.ok = nullptr; ma.B = B; ma.H = D.H; ma.P = D.P;
    ma.N = D.N; ma.G = D.G; ma.W = D.W; ma.E = D.E; ma.Cx = D.Cx; ma.status = status;
    CK(launch_mamba_step(ma, 0, (cudaStream_t)stream));
    return VC_OK;
}

extern "C" size_t vc_gemv_scratch_bytes(void) {
    return align_up(gemv_partials_bytes(256), 256) + gemv_counter_ints() * 4;
}

extern "C" vc_status vc_debug_gemv(const vc_qmat* w, const void* act, int act_ld, int B, float* out, void* scratch,
                                   vc_stream_t stream) {
    if (!w || !w->data || !act || !out || !scratch || !aligned16(act) || !aligned16(scratch)) return VC_ERR_INVALID_ARG;
    if (!fmt_ok(w->fmt, w->group) || w->N <= 0 || w->K <= 0 || B < 1 || B > 16) return VC_ERR_INVALID_ARG;
    if (act_ld % 128 || act_ld < round_up(w->K, 128)) return VC_ERR_INVALID_ARG;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    GemvArgs a{};
    a.nmat = 1;
    a.mat[0] = gm(*w);
    a.act = (const uint16_t*)act;
    a.act_ld = act_ld;
    a.B = B;
    a.tap = out;
    a.tap_ld = w->N;
    a.partials = (float*)scratch;
    a.counters = (int*)((uint8_t*)scratch + align_up(gemv_partials_bytes(256), 256));
    // split units are summed as in the step (fp32 accumulators in the zeroed partial area, left
    // zeroed) when they fit there; otherwise contributors' partials are summed in worker order
    {
        const int grp = w->fmt == VC_W_BF16 ? 64 : w->group;
        const LayoutInfo Lw = layout_info(w->fmt, grp);
        const size_t need = (size_t)a.mat[0].NU * Lw.R * (B > 8 ? 2 : 1) * 128 * 4;
        if (need <= gemv_partials_bytes(256)) a.accum = a.partials;
    }
    GemvLaunch L{};
    L.fmt = w->fmt;
    L.group = w->fmt == VC_W_BF16 ? 64 : w->group;
    L.epi = EPI_STORE;
    L.num_sms = sms > 256 ? 256 : sms;
    L.pdl = 0;
    CK(launch_gemv(L, a, (cudaStream_t)stream));
    return VC_OK;
}

extern "C" size_t vc_debug_mamba_prefill_scratch_bytes(const vc_config* cfg, int T) {
    Dims D;
    if (!dims_from_cfg(cfg, D) || !D.nm || T < 1) return 0;
    return prefill_mixer_scratch_bytes(T, D.E, D.Cx, D.H, D.P, D.N);
}

extern "C" vc_status vc_debug_mamba_prefill(const vc_config* cfg, const vc_layer_weights* layer, const void* zx, int T,
                                            float* ssm, void* conv, float* y, void* act, void* scratch,
                                            vc_stream_t stream) {
    Dims D;
    if (!dims_from_cfg(cfg, D) || !D.nm || !layer || !zx || !ssm || !conv || !y || !act || !scratch || T < 1)
        return VC_ERR_INVALID_ARG;
    if (!aligned16(scratch) || !aligned16(zx)) return VC_ERR_INVALID_ARG;
    PfMixer m{};
    m.T = T; m.E = D.E; m.Cx = D.Cx; m.H = D.H; m.P = D.P; m.N = D.N; m.G = D.G; m.W = D.W; m.NG = D.NG;
    m.eps = cfg->eps;
    m.f16 = 0;
    m.Lw = layer;
    m.zx = (const uint16_t*)zx;
    carve_mixer(m, (uint8_t*)scratch);
    m.ssm = ssm; m.ring = (uint16_t*)conv; m.act = (uint16_t*)act; m.act_ld = D.E;
    cudaStream_t s = (cudaStream_t)stream;
    CK(cudaMemsetAsync(m.status, 0, 4, s));
    CK(prefill_mixer(m, s));
    CK(cudaMemcpyAsync(y, m.y, (size_t)T * D.E * 4, cudaMemcpyDeviceToDevice, s));
    return VC_OK;
}

extern "C" vc_status vc_debug_gemm(const void* A, int lda, int M, const void* W, int ldw, int N, int K, int f16,
                                   float* out, int ldo, int32_t* status, vc_stream_t stream) {
    if (!A || !W || !out || !status || !aligned16(A) || !aligned16(W)) return VC_ERR_INVALID_ARG;
    if (M < 1 || N < 1 || K < 1 || K % 8 || lda % 8 || ldw % 8 || lda < K || ldw < K || ldo < N)
        return VC_ERR_INVALID_ARG;
    GemmArgs a{};
    a.f16 = f16 != 0;
    a.A = A; a.lda = lda; a.M = M;
    a.W = W; a.ldw = ldw; a.N = N; a.K = K;
    a.out_f32 = out; a.ldo32 = ldo;
    a.status = status;
    cudaError_t e = launch_gemm_tc(GE_F32, a, (cudaStream_t)stream);
    if (e == cudaErrorInvalidValue) return VC_ERR_INVALID_ARG;
    CK(e);
    return VC_OK;
}

extern "C" void vc_destroy(vc_backbone* h) {
    if (!h) return;
    clear_graphs(h);
    if (h->capture_stream) cudaStreamDestroy(h->capture_stream);
    if (h->prefill_side) cudaStreamDestroy(h->prefill_side);
    for (int i = 0; i < 5; ++i)
        if (h->pf_ev[i]) cudaEventDestroy(h->pf_ev[i]);
    delete h;
}

extern "C" const char* vc_status_string(vc_status s) {
    switch (s) {
        case VC_OK: return "ok";
        case VC_ERR_INVALID_ARG: return "invalid argument";
        case VC_ERR_UNSUPPORTED: return "unsupported";
        case VC_ERR_CUDA: return "CUDA error";
        case VC_ERR_CAPACITY: return "capacity exceeded";
        case VC_ERR_STATE: return "invalid state";
    }
    return "unknown status";
}

extern "C" const char* vc_last_cuda_error(void) { return g_cuda_err; }
