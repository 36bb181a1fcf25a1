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

// ------------------------------------------------------------------------------------------
// The same split on warp-level tensor-core MMA (mma.sync m16n8k16, bf16 operands, fp32
// accumulation) for head dims 64 and 128 and up to 16 query heads per KV head: the K and V rows
// arrive by the same bulk copies; the threads then permute each row's 16-byte chunks in place
// (chunk c of key row r to c ^ (r & 7)) so that the 8x8 matrix loads of eight consecutive keys
// hit eight different bank groups.  Scores: the GQ query heads are the 16 rows of the A operand,
// warp w takes keys 16w..16w+15 (two n8 tiles); the softmax over the split's keys goes through
// shared memory; P (bf16, as in the prefill's flash attention) is staged in shared memory and
// warp w forms the unnormalised output for head dims 16w..16w+15 over all the split's keys.  The
// split records and the merge are the scalar kernel's.
// ------------------------------------------------------------------------------------------
VC_DEV uint32_t ld_u32(const uint16_t* p) { return *reinterpret_cast<const uint32_t*>(p); }
VC_DEV uint32_t bf16x2_bits(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

VC_DEV void ldsm_x4(uint32_t (&r)[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}
VC_DEV void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}

static constexpr int kPsStride = kAttnSplit + 8;   // bf16 elements per row of the staged P

template <int DH>
static size_t attn_mma_smem_bytes(int max_splits) {
    return (size_t)2 * kAttnSplit * DH * 2          // K, V tiles (bf16, chunk-swizzled rows)
           + (size_t)16 * kPsStride * 2              // P (bf16) [16 heads][128 keys + pad]
           + (size_t)2 * (kAttnThreads / 32) * 16 * 4   // per-warp row max and sum
           + (size_t)max_splits * 16 * 4 + 64;       // merge weights
}

template <int DH>
__global__ void __launch_bounds__(kAttnThreads) attn_decode_mma_kernel(const AttnArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ uint64_t bar;
    __shared__ int last_flag;
    __shared__ float Ls[16];
    pdl_trigger();

    constexpr int CH = DH / 8;   // 16-byte chunks per row
    const int split = blockIdx.x, j = blockIdx.y, b = blockIdx.z;
    const int GQ = a.Hq / a.Hk, Dh = DH;
    const int slot = a.slots ? a.slots[b] : b;
    const int t = a.ctx_len[slot];
    const int nkeys = t + 1;
    const int nsplit = (nkeys + kAttnSplit - 1) / kAttnSplit;
    if (split >= nsplit || t >= a.cap) return;
    const int k0 = split * kAttnSplit, k1 = min(nkeys, k0 + kAttnSplit), nk = k1 - k0;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, tq = lane & 3;

    uint16_t* Ks = reinterpret_cast<uint16_t*>(smem);                  // [128][DH]
    uint16_t* Vs = Ks + kAttnSplit * DH;                                // [128][DH]
    uint16_t* Ps = Vs + kAttnSplit * DH;                                // [16][kPsStride]
    float* wmax = reinterpret_cast<float*>(Ps + 16 * kPsStride);        // [8][16]
    float* wsum = wmax + (kAttnThreads / 32) * 16;                      // [8][16]
    float* wts = wsum + (kAttnThreads / 32) * 16;                       // [max_splits][GQ]

    const size_t head_off = ((size_t)slot * a.Hk + j) * a.cap;
    const uint16_t* Kg = a.kcache + head_off * DH;
    const uint16_t* Vg = a.vcache + head_off * DH;
    const int nold = min(k1, t) - k0;      // rows written by earlier frames
    if (tid == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        if (nold > 0) {
            const uint32_t bytes = (uint32_t)(nold * DH * 2);
            mbar_arrive_expect_tx(&bar, 2 * bytes);
            bulk_g2s(Ks, Kg + (size_t)k0 * DH, bytes, &bar);
            bulk_g2s(Vs, Vg + (size_t)k0 * DH, bytes, &bar);
        }
    }
    // rows past the split's keys: zero (their scores are masked; V must not carry stale values)
    for (int idx = tid; idx < (kAttnSplit - nk) * CH; idx += kAttnThreads) {
        const int r = nk + idx / CH, c = idx % CH;
        reinterpret_cast<uint4*>(Ks + r * DH)[c] = make_uint4(0u, 0u, 0u, 0u);
        reinterpret_cast<uint4*>(Vs + r * DH)[c] = make_uint4(0u, 0u, 0u, 0u);
    }
    __syncthreads();
    pdl_wait();
    if (!a.ok[b]) {
        if (nold > 0) mbar_wait(&bar, 0, a.status);   // never leave with copies in flight
        return;
    }
    if (k1 > t) {   // the new frame's key/value, written by this frame's qkv projection
        for (int i = tid; i < DH; i += kAttnThreads) {
            Ks[(t - k0) * DH + i] = Kg[(size_t)t * DH + i];
            Vs[(t - k0) * DH + i] = Vg[(size_t)t * DH + i];
        }
    }
    // the query heads' A fragments (rows >= GQ zero), straight from global
    uint32_t qa[DH / 16][4];
    {
        const uint16_t* q0 = a.q + (size_t)b * a.q_ld + (size_t)(j * GQ) * DH;
#pragma unroll
        for (int ks = 0; ks < DH / 16; ++ks) {
            const int c = ks * 16 + 2 * tq;
            qa[ks][0] = g < GQ ? ld_u32(q0 + (size_t)g * DH + c) : 0u;
            qa[ks][1] = g + 8 < GQ ? ld_u32(q0 + (size_t)(g + 8) * DH + c) : 0u;
            qa[ks][2] = g < GQ ? ld_u32(q0 + (size_t)g * DH + c + 8) : 0u;
            qa[ks][3] = g + 8 < GQ ? ld_u32(q0 + (size_t)(g + 8) * DH + c + 8) : 0u;
        }
    }
    bool okc = true;
    if (nold > 0) okc = mbar_wait(&bar, 0, a.status);
    if (!__syncthreads_and(okc)) return;
    // permute each row's chunks in place: chunk c <-> c ^ (r & 7) (pairs swap)
    for (int idx = tid; idx < 2 * kAttnSplit * (CH / 2); idx += kAttnThreads) {
        const int tile = idx / (kAttnSplit * (CH / 2)), rem = idx % (kAttnSplit * (CH / 2));
        const int r = rem / (CH / 2), pidx = rem % (CH / 2), m = r & 7;
        if (m == 0) continue;
        // the pidx-th chunk c of the row with c < (c ^ m): pidx with a 0 inserted at m's top bit
        const int hb = 31 - __clz(m);
        const int c = ((pidx >> hb) << (hb + 1)) | (pidx & ((1 << hb) - 1));
        uint4* row = reinterpret_cast<uint4*>((tile ? Vs : Ks) + r * DH);
        const uint4 x = row[c], y = row[c ^ m];
        row[c] = y;
        row[c ^ m] = x;
    }
    __syncthreads();

    // scores of keys 16 warp .. 16 warp + 15: two n8 tiles
    constexpr float kLog2e = 1.4426950408889634f;
    const float scale = rsqrtf((float)DH);
    float s[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.0f;
    {
        const int m = lane >> 3, lr = lane & 7;
        const int key = 16 * warp + 8 * (m >> 1) + lr;
#pragma unroll
        for (int ks = 0; ks < DH / 16; ++ks) {
            const int ch = (2 * ks + (m & 1)) ^ (key & 7);
            uint32_t kb[4];
            ldsm_x4(kb, Ks + key * DH + ch * 8);
            mma_bf16(s[0], qa[ks], kb[0], kb[1]);
            mma_bf16(s[1], qa[ks], kb[2], kb[3]);
        }
    }
    // scale and mask; per-row max over the warp's keys, then over the warps
    float rmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int key = 16 * warp + 8 * nt + 2 * tq + (e & 1);
            s[nt][e] = key < nk ? s[nt][e] * scale : -INFINITY;
            rmax[e >> 1] = fmaxf(rmax[e >> 1], s[nt][e]);
        }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        rmax[h] = fmaxf(rmax[h], __shfl_xor_sync(0xffffffffu, rmax[h], 1));
        rmax[h] = fmaxf(rmax[h], __shfl_xor_sync(0xffffffffu, rmax[h], 2));
    }
    if (tq == 0) {
        wmax[warp * 16 + g] = rmax[0];
        wmax[warp * 16 + g + 8] = rmax[1];
    }
    __syncthreads();
    float M[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float mx = -INFINITY;
        for (int w = 0; w < kAttnThreads / 32; ++w) mx = fmaxf(mx, wmax[w * 16 + g + 8 * h]);
        M[h] = mx;   // finite: key 0 of the split is always present
    }
    float rsum[2] = {0.0f, 0.0f};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        float p[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            p[e] = s[nt][e] == -INFINITY ? 0.0f : exp2f((s[nt][e] - M[e >> 1]) * kLog2e);
            rsum[e >> 1] += p[e];
        }
        const int key = 16 * warp + 8 * nt + 2 * tq;
        *reinterpret_cast<uint32_t*>(Ps + g * kPsStride + key) = bf16x2_bits(p[0], p[1]);
        *reinterpret_cast<uint32_t*>(Ps + (g + 8) * kPsStride + key) = bf16x2_bits(p[2], p[3]);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        rsum[h] += __shfl_xor_sync(0xffffffffu, rsum[h], 1);
        rsum[h] += __shfl_xor_sync(0xffffffffu, rsum[h], 2);
    }
    if (tq == 0) {
        wsum[warp * 16 + g] = rsum[0];
        wsum[warp * 16 + g + 8] = rsum[1];
    }
    __syncthreads();
    float* part = a.scratch + ((((size_t)b * a.Hk + j) * a.max_splits + split) * GQ) * (Dh + 2);
    if (warp == 0 && lane < GQ) {
        float l = 0.0f, mx = -INFINITY;
        for (int w = 0; w < kAttnThreads / 32; ++w) {
            l += wsum[w * 16 + lane];
            mx = fmaxf(mx, wmax[w * 16 + lane]);
        }
        part[lane * (Dh + 2) + Dh] = mx;
        part[lane * (Dh + 2) + Dh + 1] = l;
    }
    // unnormalised P . V for head dims 16 warp .. 16 warp + 15 (warps beyond DH / 16 idle)
    if (warp < DH / 16) {
        float o[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.0f;
        const int m = lane >> 3, lr = lane & 7;
#pragma unroll
        for (int ks = 0; ks < kAttnSplit / 16; ++ks) {
            uint32_t pa[4];
            const uint16_t* pr = Ps + g * kPsStride + ks * 16 + 2 * tq;
            pa[0] = ld_u32(pr);
            pa[1] = ld_u32(pr + 8 * kPsStride);
            pa[2] = ld_u32(pr + 8);
            pa[3] = ld_u32(pr + 8 * kPsStride + 8);
            const int key = ks * 16 + 8 * (m & 1) + lr;
            const int ch = (2 * warp + (m >> 1)) ^ (key & 7);
            uint32_t vb[4];
            ldsm_x4_t(vb, Vs + key * DH + ch * 8);
            mma_bf16(o[0], pa, vb[0], vb[1]);
            mma_bf16(o[1], pa, vb[2], vb[3]);
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int d = 16 * warp + 8 * nt + 2 * tq;
            if (g < GQ) *reinterpret_cast<float2*>(part + g * (Dh + 2) + d) = make_float2(o[nt][0], o[nt][1]);
            if (g + 8 < GQ) *reinterpret_cast<float2*>(part + (g + 8) * (Dh + 2) + d) = make_float2(o[nt][2], o[nt][3]);
        }
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
        float Mx = -INFINITY;
        for (int sp = 0; sp < nsplit; ++sp) Mx = fmaxf(Mx, wts[sp * GQ + tid]);
        float L = 0.0f;
#pragma unroll 8
        for (int sp = 0; sp < nsplit; ++sp) {
            const float w = expf(wts[sp * GQ + tid] - Mx);
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
    // tensor-core form for head dims 64 and 128 (the scalar kernel for the others)
    const bool mma = (a.Dh == 128 || a.Dh == 64) && GQ <= 16;
    auto kern = !mma ? attn_decode_kernel : a.Dh == 128 ? attn_decode_mma_kernel<128> : attn_decode_mma_kernel<64>;
    const size_t smem = !mma ? attn_smem_bytes(GQ, a.Dh, a.max_splits)
                             : a.Dh == 128 ? attn_mma_smem_bytes<128>(a.max_splits) : attn_mma_smem_bytes<64>(a.max_splits);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
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
    return cudaLaunchKernelEx(&cfg, kern, a);
}

}  // namespace vc
