// frame.cuh -- host-visible declarations of the persistent frame kernel: one cooperative launch
// runs a whole decode frame (input, every layer's projections and mixers, both heads).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "decode.cuh"
#include "gemv.cuh"

namespace vc {

enum FkKind : int {
    FK_INPUT = 0,       // step input: residual, normalized activation, capacity check
    FK_GEMV = 1,        // one projection (or both heads) with its fused epilogue
    FK_MAMBA = 2,       // Mamba-2 single step (conv ring, SSM update and readout, gate)
    FK_ATTN = 3,        // GQA decode attention over 32-key splits (partial softmax sums)
    FK_ATTN_MERGE = 4,  // merge of the splits, o_proj input
};

struct alignas(16) FkGemv {
    GemvArgs a;        // the projection's arguments (tokens of the heads come from FrameParams)
    int epi;           // Epi
    int head;          // 1: a vocabulary head matrix (head format), 0: a layer matrix
    float* zero_buf;   // zeroed by CTA 0 while this op runs (sums the next mixer accumulates)
    int zero_n;
    int pad;
};

static_assert(sizeof(FkGemv) % 16 == 0, "FkGemv is copied to shared memory in 16-byte pieces");

struct FkOp {
    int kind, idx;
};

static constexpr int kFkMaxOps = 512;
static constexpr int kFkMaxGemv = 256;
static constexpr int kFkMaxMix = 128;
static constexpr int kFkAttnSplit = 32;   // keys per attention split of the frame kernel

struct FrameProgram {
    int n_ops, n_gemv, n_mamba, n_attn;
    InputArgs input;
    FkOp ops[kFkMaxOps];
    FkGemv gemv[kFkMaxGemv];
    MambaStepArgs mamba[kFkMaxMix];
    AttnArgs attn[kFkMaxMix];
};

struct FrameParams {
    const FrameProgram* prog;   // device copy (workspace)
    const uint16_t* x;          // this frame's input rows (the input op's x)
    int* tok_t;                 // greedy tokens out (and, for fused inputs, the previous tokens in)
    int* tok_f;
    unsigned* barrier;          // [0] grid barrier arrivals, [2] CTAs finished; zero at launch, and
                                // returned to zero by the last CTA of every launch
    int* abort;                 // set when a bounded wait gives up; zero at launch (likewise)
    int* status;
    int slots;                  // ring slots per warp
    int slot_bytes;             // bytes per ring slot
};

struct FrameGeom {
    int lfmt, lgrp, hfmt, hgrp, nt;
};

// ring geometry of a launch for this format pair (0 slots: not supported)
void frame_ring(const FrameGeom& g, int* slots, int* slot_bytes, size_t* smem);
// whether the frame kernel has an instantiation for these weight formats, this attention shape
// (GQ query heads per KV head, head dim Dh) and Mamba-2 state size N
bool frame_supported(const FrameGeom& g, int GQ, int Dh, int N);
// one frame: a cooperative launch of one CTA per SM; cudaErrorNotSupported for a format pair
// without an instantiation
cudaError_t launch_frame(const FrameGeom& g, const FrameParams& p, int num_sms, cudaStream_t s);

}  // namespace vc
