// attn_decode.cu -- GQA decode attention for one frame, split over the key axis.
//
// Layer kind: the attention layers of the hybrid backbone ("Hybrid Mamba/Transformer backbone",
// NVIDIA NemotronLabs VoiceChat 11B blog, "Key design decisions" 2); no positional encoding.
// For session b and KV head j, the Hq/Hk query heads i share keys/values j:
//     s_t = q_i . K_t / sqrt(Dh),  o_i = sum_t softmax(s)_t V_t,  t = 0..ctx (the new frame's key
//     is the last one, appended by the qkv projection's epilogue).
// Each CTA takes 128 keys: K and V rows are bulk-copied to shared memory (rows of earlier
// frames before griddepcontrol.wait), scores/softmax/P.V are fp32 on CUDA cores, and the CTA
// writes (max, sum, unnormalised output).  The last CTA of a (session, KV head) rescales and
// merges all splits (log-sum-exp) and writes bf16(o), the o_proj input.
#include "common.cuh"
#include "decode.cuh"

namespace vc {

static constexpr int kAttnThreads = 256;
static constexpr int kMaxGQ = 8;

static size_t attn_smem_bytes(int GQ, int Dh, int max_splits) {
    const int nparts = kAttnThreads / Dh;
    return (size_t)2 * kAttnSplit * Dh * 2          // K, V tiles (bf16)
           + (size_t)GQ * Dh * 4                     // q (fp32, pre-scaled)
           + (size_t)GQ * kAttnSplit * 4             // scores / probabilities
           + (size_t)nparts * GQ * Dh * 4            // P.V partials over key subsets
           + (size_t)max_splits * GQ * 4 + 64;       // merge weights
}

__global__ void __launch_bounds__(kAttnThreads) attn_decode_kernel(const AttnArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ uint64_t bar;
    __shared__ int last_flag;
    __shared__ float Ls[kMaxGQ];
    pdl_trigger();

    const int split = blockIdx.x, j = blockIdx.y, b = blockIdx.z;
    const int GQ = a.Hq / a.Hk, Dh = a.Dh;
    const int slot = a.slots ? a.slots[b] : b;
    const int t = a.ctx_len[slot];          // frames cached before this one; key t is the new frame
    const int nkeys = t + 1;
    const int nsplit = (nkeys + kAttnSplit - 1) / kAttnSplit;
    if (split >= nsplit || t >= a.cap) return;
    const int k0 = split * kAttnSplit, k1 = min(nkeys, k0 + kAttnSplit), nk = k1 - k0;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nparts = kAttnThreads / Dh;

    uint16_t* Ks = reinterpret_cast<uint16_t*>(smem);                  // [128][Dh]
    uint16_t* Vs = Ks + kAttnSplit * Dh;                                // [128][Dh]
    float* qs = reinterpret_cast<float*>(Vs + kAttnSplit * Dh);         // [GQ][Dh]
    float* ps = qs + GQ * Dh;                                           // [GQ][128]
    float* red = ps + GQ * kAttnSplit;                                  // [nparts][GQ][Dh]
    float* wts = red + nparts * GQ * Dh;                                // [max_splits][GQ]

    const size_t head_off = ((size_t)slot * a.Hk + j) * a.cap;
    const uint16_t* Kg = a.kcache + head_off * Dh;
    const uint16_t* Vg = a.vcache + head_off * Dh;
    const int nold = min(k1, t) - k0;      // rows written by earlier frames
    if (tid == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        if (nold > 0) {
            const uint32_t bytes = (uint32_t)(nold * Dh * 2);
            mbar_arrive_expect_tx(&bar, 2 * bytes);
            bulk_g2s(Ks, Kg + (size_t)k0 * Dh, bytes, &bar);
            bulk_g2s(Vs, Vg + (size_t)k0 * Dh, bytes, &bar);
        }
    }
    __syncthreads();
    pdl_wait();
    if (!a.ok[b]) {
        if (nold > 0) mbar_wait(&bar, 0, a.status);   // never leave with copies in flight
        return;
    }
    if (k1 > t) {   // the new frame's key/value, written by this frame's qkv projection
        for (int i = tid; i < Dh; i += kAttnThreads) {
            Ks[(t - k0) * Dh + i] = Kg[(size_t)t * Dh + i];
            Vs[(t - k0) * Dh + i] = Vg[(size_t)t * Dh + i];
        }
    }
    const float scale = rsqrtf((float)Dh);
    for (int i = tid; i < GQ * Dh; i += kAttnThreads)
        qs[i] = bf16_bits_to_f(a.q[(size_t)b * a.q_ld + (size_t)(j * GQ) * Dh + i]) * scale;
    if (nold > 0 && !mbar_wait(&bar, 0, a.status)) return;
    __syncthreads();

    // scores: two threads per key, each half of the head dimension
    {
        const int key = tid >> 1, hf = tid & 1;
        const int hd = Dh / 2;
        float s[kMaxGQ];
#pragma unroll
        for (int i = 0; i < kMaxGQ; ++i) s[i] = 0.0f;
        if (key < nk) {
            const uint16_t* kr = Ks + key * Dh + hf * hd;
            const int nch = hd / 8;
            for (int cc = 0; cc < nch; ++cc) {
                const int c = (cc + key * 2 + hf) % nch;   // rotated chunk order: no bank conflicts
                const uint4 kv = *reinterpret_cast<const uint4*>(kr + c * 8);
                const uint32_t w[4] = {kv.x, kv.y, kv.z, kv.w};
                float kf[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    kf[2 * e] = __uint_as_float(w[e] << 16);
                    kf[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
                }
#pragma unroll
                for (int i = 0; i < kMaxGQ; ++i) {
                    if (i < GQ) {
                        const float4* qr = reinterpret_cast<const float4*>(qs + i * Dh + hf * hd + c * 8);
                        const float4 q0 = qr[0], q1 = qr[1];
                        s[i] = fmaf(q0.x, kf[0], s[i]); s[i] = fmaf(q0.y, kf[1], s[i]);
                        s[i] = fmaf(q0.z, kf[2], s[i]); s[i] = fmaf(q0.w, kf[3], s[i]);
                        s[i] = fmaf(q1.x, kf[4], s[i]); s[i] = fmaf(q1.y, kf[5], s[i]);
                        s[i] = fmaf(q1.z, kf[6], s[i]); s[i] = fmaf(q1.w, kf[7], s[i]);
                    }
                }
            }
        }
#pragma unroll
        for (int i = 0; i < kMaxGQ; ++i) {
            const float o = __shfl_xor_sync(0xffffffffu, s[i], 1);
            if (i < GQ && hf == 0 && key < nk) ps[i * kAttnSplit + key] = s[i] + o;
        }
    }
    __syncthreads();

    // per-head max / exp / sum over this split's keys
    float* part = a.scratch + ((((size_t)b * a.Hk + j) * a.max_splits + split) * GQ) * (Dh + 2);
    for (int i = warp; i < GQ; i += kAttnThreads / 32) {
        float mx = -INFINITY;
        for (int k = lane; k < nk; k += 32) mx = fmaxf(mx, ps[i * kAttnSplit + k]);
        mx = warp_max(mx);
        float sum = 0.0f;
        for (int k = lane; k < nk; k += 32) {
            const float e = expf(ps[i * kAttnSplit + k] - mx);
            ps[i * kAttnSplit + k] = e;
            sum += e;
        }
        sum = warp_sum(sum);
        if (lane == 0) {
            part[i * (Dh + 2) + Dh] = mx;
            part[i * (Dh + 2) + Dh + 1] = sum;
        }
    }
    __syncthreads();
    // unnormalised p . V: thread (d, key subset kp), then a reduction over the subsets
    {
        const int d = tid % Dh, kp = tid / Dh;
        float o[kMaxGQ];
#pragma unroll
        for (int i = 0; i < kMaxGQ; ++i) o[i] = 0.0f;
        for (int k = kp; k < nk; k += nparts) {
            const float v = bf16_bits_to_f(Vs[k * Dh + d]);
#pragma unroll
            for (int i = 0; i < kMaxGQ; ++i)
                if (i < GQ) o[i] = fmaf(ps[i * kAttnSplit + k], v, o[i]);
        }
#pragma unroll
        for (int i = 0; i < kMaxGQ; ++i)
            if (i < GQ) red[(kp * GQ + i) * Dh + d] = o[i];
    }
    __syncthreads();
    for (int idx = tid; idx < GQ * Dh; idx += kAttnThreads) {
        float o = 0.0f;
        for (int kp = 0; kp < nparts; ++kp) o += red[kp * GQ * Dh + idx];
        part[(idx / Dh) * (Dh + 2) + idx % Dh] = o;
    }

    // the last split of this (session, KV head) merges all splits
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        int* cnt = a.counters + b * a.Hk + j;
        last_flag = atomicAdd(cnt, 1) == nsplit - 1;
        if (last_flag) *cnt = 0;
    }
    __syncthreads();
    if (!last_flag) return;
    __threadfence();
    const float* base = a.scratch + (((size_t)b * a.Hk + j) * a.max_splits) * GQ * (Dh + 2);
    for (int idx = tid; idx < nsplit * GQ; idx += kAttnThreads)
        wts[idx] = __ldcg(base + (size_t)idx * (Dh + 2) + Dh);        // m of (split, head)
    __syncthreads();
    if (tid < GQ) {
        float M = -INFINITY;
        for (int sp = 0; sp < nsplit; ++sp) M = fmaxf(M, wts[sp * GQ + tid]);
        float L = 0.0f;
#pragma unroll 8
        for (int sp = 0; sp < nsplit; ++sp) {
            const float w = expf(wts[sp * GQ + tid] - M);
            L = fmaf(__ldcg(base + ((size_t)sp * GQ + tid) * (Dh + 2) + Dh + 1), w, L);
            wts[sp * GQ + tid] = w;
        }
        Ls[tid] = L;
    }
    __syncthreads();
    for (int idx = tid; idx < GQ * Dh; idx += kAttnThreads) {
        const int i = idx / Dh, d = idx % Dh;
        float O = 0.0f;
#pragma unroll 8
        for (int sp = 0; sp < nsplit; ++sp) O = fmaf(__ldcg(base + ((size_t)sp * GQ + i) * (Dh + 2) + d), wts[sp * GQ + i], O);
        const float o = O / Ls[i];
        const size_t col = (size_t)(j * GQ + i) * Dh + d;
        a.act[(size_t)b * a.act_ld + col] = a.act_f16 ? act_bits<true>(o) : act_bits<false>(o);
    }
}

bool attn_decode_supported(int Hq, int Hk, int Dh) {
    return Hk > 0 && Hq % Hk == 0 && Hq / Hk <= kMaxGQ && Dh > 0 && Dh <= kAttnThreads && kAttnThreads % Dh == 0;
}

cudaError_t launch_attn_decode(const AttnArgs& a, int pdl, cudaStream_t s) {
    const int GQ = a.Hq / a.Hk;
    if (GQ > kMaxGQ || a.Dh > kAttnThreads || kAttnThreads % a.Dh) return cudaErrorInvalidValue;
    const size_t smem = attn_smem_bytes(GQ, a.Dh, a.max_splits);
    cudaError_t e = cudaFuncSetAttribute(attn_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(a.max_splits, a.Hk, a.B);
    cfg.blockDim = dim3(kAttnThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, attn_decode_kernel, a);
}

}  // namespace vc
