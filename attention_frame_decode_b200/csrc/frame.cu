// frame.cu -- ring geometry and dispatch of the persistent frame kernel (frame_kernel.cuh); the
// kernel is instantiated once per pair of weight formats in frame_<pair>.cu.
#include <algorithm>

#include "frame_kernel.cuh"

namespace vc {

// dynamic shared memory of one CTA for the rings (the activation area comes on top)
static constexpr int kFrameSmemBudget = 224 * 1024 - kFkActBytes;

// the instantiated (layer format, group, head format, group, column tiles) tuples
#define VC_FRAME_FORMATS(X) \
    X(bf16_bf16_1, FMT_BF16, 64, FMT_BF16, 64, 1) \
    X(bf16_bf16_2, FMT_BF16, 64, FMT_BF16, 64, 2) \
    X(w4_bf16_1, FMT_W4, 64, FMT_BF16, 64, 1) \
    X(w4_bf16_2, FMT_W4, 64, FMT_BF16, 64, 2) \
    X(w4_w4_1, FMT_W4, 64, FMT_W4, 64, 1) \
    X(w4_w4_2, FMT_W4, 64, FMT_W4, 64, 2) \
    X(w3_bf16_1, FMT_W3, 64, FMT_BF16, 64, 1) \
    X(w3_bf16_2, FMT_W3, 64, FMT_BF16, 64, 2) \
    X(w8g128_bf16_1, FMT_W8, 128, FMT_BF16, 64, 1) \
    X(w8g128_bf16_2, FMT_W8, 128, FMT_BF16, 64, 2) \
    X(w8_w8_1, FMT_W8, 64, FMT_W8, 64, 1)

#define VC_FRAME_DECL(TAG, LF, LG, HF, HG, NT) \
    cudaError_t frame_launch_##TAG(const FrameParams& p, int num_sms, size_t smem, cudaStream_t s);
VC_FRAME_FORMATS(VC_FRAME_DECL)
#undef VC_FRAME_DECL

void frame_ring(const FrameGeom& g, int* slots, int* slot_bytes, size_t* smem) {
    const int warps = fk_warps(g.nt);
    const int bbL = layout_info(g.lfmt, g.lgrp).block_bytes, bbH = layout_info(g.hfmt, g.hgrp).block_bytes;
    // a slot holds one chunk of whole blocks of either format; choose the slot size that keeps the
    // most layer-weight bytes in flight per warp (the layers are most of a frame's bytes)
    int best_slot = 0, best_ns = 0;
    long long best_eff = -1;
    for (int k = 1; k <= 8; ++k) {
        const int slot = std::max(k * bbL, bbH);
        int ns = kFrameSmemBudget / (warps * slot);
        if (ns > kMaxSlots) ns = kMaxSlots;
        if (ns < 2) continue;
        const long long eff = (long long)ns * (slot / bbL) * bbL;
        if (eff > best_eff) { best_eff = eff; best_slot = slot; best_ns = ns; }
    }
    *slots = best_ns;
    *slot_bytes = best_slot;
    *smem = (size_t)warps * best_ns * best_slot + kFkActBytes;
}

bool frame_supported(const FrameGeom& g, int GQ, int Dh, int N) {
    bool attn = false;
#define VC_FK_ATTN_OK(G, D) attn = attn || (GQ == G && Dh == 32 * D);
    VC_FK_ATTN_SHAPES(VC_FK_ATTN_OK)
#undef VC_FK_ATTN_OK
    if (!attn || N < 4 || N > 128 || N % 4) return false;
    bool fmt = false;
#define VC_FK_FMT_OK(TAG, LF, LG, HF, HG, NT) \
    fmt = fmt || (g.lfmt == LF && g.lgrp == LG && g.hfmt == HF && g.hgrp == HG && g.nt == NT);
    VC_FRAME_FORMATS(VC_FK_FMT_OK)
#undef VC_FK_FMT_OK
    return fmt;
}

cudaError_t launch_frame(const FrameGeom& g, const FrameParams& p, int num_sms, cudaStream_t s) {
    int slots = 0, slot_bytes = 0;
    size_t smem = 0;
    frame_ring(g, &slots, &slot_bytes, &smem);
    if (slots < 2 || slots != p.slots || slot_bytes != p.slot_bytes) return cudaErrorInvalidValue;
#define VC_FRAME_CASE(TAG, LF, LG, HF, HG, NT) \
    if (g.lfmt == LF && g.lgrp == LG && g.hfmt == HF && g.hgrp == HG && g.nt == NT) \
        return frame_launch_##TAG(p, num_sms, smem, s);
    VC_FRAME_FORMATS(VC_FRAME_CASE)
#undef VC_FRAME_CASE
    return cudaErrorNotSupported;
}

}  // namespace vc
