// gemv.cuh -- host-visible declarations of the streaming weight GEMV (y = W u for B <= 16 rows).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace vc {

enum Epi : int {
    EPI_STORE = 0,   // out[b][n] = act(y)
    EPI_RELU2 = 1,   // out[b][n] = act(relu(y)^2)
    EPI_RESID = 2,   // r[b][n] += y; act_next[b][n] = act(r * gamma_next); ssq parts of r
    EPI_QKV = 3,     // q rows -> q buffer; k/v rows -> KV cache at position ctx_len[slot]
    EPI_ARGMAX = 4,  // greedy token per row b (lowest index on ties), per matrix
};

struct GemvMat {
    const uint8_t* w;
    int N, K, NU, KT;
};

// input scales: the dot product of k-group q and batch row b is multiplied by
//   rsqrt(sum_i parts[b][q][i] * inv_width + eps)
// (pre-RMSNorm: one group of width d; gated RMSNorm: norm_groups groups).  parts == null: 1.
struct InScale {
    const float* parts;
    int n_groups, per_group, group_cols;
    float inv_width, eps;
};

struct GemvArgs {
    GemvMat mat[2];
    int nmat;
    const uint16_t* act;   // [B][act_ld], bf16 bits (BF16 weights) or fp16 bits (quantized)
    int act_ld, B;
    InScale insc;
    // epilogue
    uint16_t* out;
    int out_ld, out_f16;
    float* resid;
    int resid_ld;
    const float* gamma_next;
    uint16_t* act_next;
    int act_next_ld, act_next_f16;
    float* parts_next;
    int parts_ld;
    float* tap;           // optional fp32 copy of the epilogue values ([nmat][B][tap_ld])
    int tap_ld;
    // attention q/k/v split
    uint16_t* q_out;
    int q_ld;
    uint16_t *kcache, *vcache;   // this layer's [n_slots][Hk][cap][Dh]
    int Hq, Hk, Dh, cap;
    const int* ctx_len;
    const int* slots;
    const int* ok;
    // greedy heads
    unsigned long long* keys;    // [2][16]
    int* tok[2];
    int* ctx_len_mut;
    int* done;
    // scratch + status
    float* partials;
    int* counters;
    // optional: per-unit fp32 accumulators (zero on entry, left zero), R*NT*128 floats per unit
    // of every matrix of the launch.  When set, contributors to a split unit add their fragment
    // sums atomically and the last one reads the total once (shorter tail; the summation order
    // then varies from run to run); when null, partials are summed in worker order.
    float* accum;
    int* status;
};

struct GemvLaunch {
    int fmt, group, epi;
    int num_sms;
    int pdl;
    // up to 8 rows: 0 = two CTAs per SM, each with half the ring budget; 1 = one CTA per SM with
    // half the budget (the next launch's CTA fits beside it); 2 = one CTA per SM, whole budget
    int shape;
};

// size in bytes of the scratch partial buffer and counters needed by any launch on num_sms SMs
size_t gemv_partials_bytes(int num_sms);
size_t gemv_counter_ints();

cudaError_t launch_gemv(const GemvLaunch& L, const GemvArgs& a, cudaStream_t s);

// weight preparation (not on the step path)
cudaError_t launch_quantize(int fmt, int group, int N, int K, const float* w, uint8_t* out, cudaStream_t s);
cudaError_t launch_pack_bf16(int N, int K, const uint16_t* w, uint8_t* out, cudaStream_t s);
cudaError_t launch_pack_canonical(int fmt, int group, int N, int K, const uint32_t* q, const uint16_t* scales,
                                  const uint32_t* zeros, uint8_t* out, cudaStream_t s);
cudaError_t launch_dequant(int fmt, int group, int N, int K, const uint8_t* w, float* out, cudaStream_t s);
// dense 16-bit row-major copy [N][ldo] (bf16, or fp16 of the dequantized value when f16 = 1)
cudaError_t launch_unpack16(int fmt, int group, int N, int K, const uint8_t* w, uint16_t* out, int ldo, int f16,
                            cudaStream_t s);

}  // namespace vc
