// decode.cu -- mixer kernels of the per-frame decode step.
//
// Mamba-2 single step (layer kind named on "NemotronLabs VoiceChat 11B: GPTQ 3-bit LLM, MLX";
// equations: Dao & Gu, "Transformers are SSMs", the Mamba-2 block), per (session, head, half of
// the head's P channels):
//   xc = silu(conv_b + sum_k conv_w[k] * window[k])  over a ring of the last W pre-conv rows,
//   dt = softplus(dt_raw + dt_bias), a = exp(A dt) with A = -exp(A_log),
//   S[p][n] <- a S[p][n] + dt x[p] B[n],  y[p] = sum_n C[n] S[p][n] + D x[p],
//   v = y * silu(z); the out_proj input is bf16(v * gamma_n) and the group RMS of v is
//   applied inside the out_proj GEMV from the per-(head, half) sums of squares written here.
// The fp32 state slice is prefetched with a bulk copy before griddepcontrol.wait (it was written
// by the previous frame) and written back once.
//
// GQA decode attention (no positional encoding), split over the key axis: each CTA scores the
// Hq/Hk query heads of one KV head against up to 64 cached keys (bulk-copied to shared memory),
// keeps (max, sum, unnormalised output) and the last CTA of the (session, KV head) merges the
// splits with the usual log-sum-exp rescaling.
#include "common.cuh"
#include "decode.cuh"

namespace vc {

// ------------------------------------------------------------------------------------------
// step input: r = fp32(x), act = bf16(r * gamma_0), row-unit sums of squares, capacity check
// ------------------------------------------------------------------------------------------
__global__ void input_kernel(const InputArgs a) {
    pdl_trigger();
    const int b = blockIdx.x;
    const int slot = a.slots ? a.slots[b] : b;
    if (threadIdx.x == 0) {
        const int okb = a.ctx_len[slot] < a.cap;
        a.ok[b] = okb;
        if (!okb) atomicOr(a.status, VC_DEV_CAPACITY);
    }
    for (int k = threadIdx.x; k < a.d; k += blockDim.x) {
        const float v = bf16_bits_to_f(a.x[(size_t)b * a.d + k]);
        a.r[(size_t)b * a.d + k] = v;
        const float an = v * a.gamma[k];
        a.act[(size_t)b * a.act_ld + k] = a.act_f16 ? act_bits<true>(an) : act_bits<false>(an);
        if (a.tap) a.tap[(size_t)b * a.d + k] = v;
    }
    for (int u = threadIdx.x; u < a.n_units; u += blockDim.x) {
        float ss = 0.0f;
        const int k1 = min(a.d, (u + 1) * a.unit_rows);
        for (int k = u * a.unit_rows; k < k1; ++k) {
            const float v = bf16_bits_to_f(a.x[(size_t)b * a.d + k]);
            ss += v * v;
        }
        a.parts[(size_t)b * a.n_units + u] = ss;
    }
}

cudaError_t launch_input(const InputArgs& a, cudaStream_t s) {
    input_kernel<<<a.B, 256, 0, s>>>(a);
    return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// Mamba-2 step
// ------------------------------------------------------------------------------------------
static constexpr int kMambaThreads = 256;

__global__ void __launch_bounds__(kMambaThreads) mamba_step_kernel(const MambaStepArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ uint64_t bar;
    __shared__ float red[kMambaThreads / 32];
    pdl_trigger();

    const int h2 = blockIdx.x, b = blockIdx.y;
    const int h = h2 >> 1, half = h2 & 1;
    const int Ph = a.P / 2, p0 = half * Ph;
    const int slot = a.slots ? a.slots[b] : b;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = (int)((long long)h * a.G / a.H);

    float* S = reinterpret_cast<float*>(smem);                       // [Ph][N]
    float* xs = S + Ph * a.N;                                         // [Ph]
    float* Bs = xs + Ph;                                              // [N]
    float* Cs = Bs + a.N;                                             // [N]

    float* Sg = a.ssm + (((size_t)slot * a.H + h) * a.P + p0) * a.N;
    const uint32_t sbytes = (uint32_t)(Ph * a.N * 4);
    if (tid == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(&bar, sbytes);
        bulk_g2s(S, Sg, sbytes, &bar);
    }

    pdl_wait();
    const bool okb = a.ok ? a.ok[b] != 0 : true;
    const int t = a.ctx_len[slot];
    const uint16_t* zx = a.zx + (size_t)b * a.zx_ld;
    const uint16_t* xBC = zx + a.E;
    uint16_t* ring = a.conv + (size_t)slot * a.W * a.Cx;
    const bool writes_bc = (h % (a.H / a.G) == 0) && half == 0;

    // conv + silu for this CTA's x channels and its group's B, C channels
    auto conv_ch = [&](int c) -> float {
        float acc = a.conv_b[c];
        for (int k = 0; k < a.W - 1; ++k) {
            const int rs = ((t - (a.W - 1) + k) % a.W + a.W) % a.W;
            acc += a.conv_w[c * a.W + k] * bf16_bits_to_f(ring[(size_t)rs * a.Cx + c]);
        }
        acc += a.conv_w[c * a.W + a.W - 1] * bf16_bits_to_f(xBC[c]);
        return silu_f(acc);
    };
    for (int i = tid; i < Ph + 2 * a.N; i += kMambaThreads) {
        int c;
        float* dst;
        if (i < Ph) { c = h * a.P + p0 + i; dst = xs + i; }
        else if (i < Ph + a.N) { c = a.E + g * a.N + (i - Ph); dst = Bs + (i - Ph); }
        else { c = a.E + a.G * a.N + g * a.N + (i - Ph - a.N); dst = Cs + (i - Ph - a.N); }
        *dst = conv_ch(c);
    }
    __syncthreads();   // all window reads done before the ring slot t mod W is overwritten
    if (okb) {
        uint16_t* rw = ring + (size_t)(t % a.W) * a.Cx;
        for (int i = tid; i < Ph; i += kMambaThreads) rw[h * a.P + p0 + i] = xBC[h * a.P + p0 + i];
        if (writes_bc)
            for (int i = tid; i < 2 * a.N; i += kMambaThreads) {
                const int c = a.E + (i < a.N ? g * a.N + i : a.G * a.N + g * a.N + (i - a.N));
                rw[c] = xBC[c];
            }
    }

    const float dt = softplus_f(bf16_bits_to_f(zx[a.E + a.Cx + h]) + a.dt_bias[h]);
    const float A = -expf(a.A_log[h]);
    const float decay = expf(A * dt);
    const float Dh = a.D[h];

    if (!mbar_wait(&bar, 0, a.status)) return;

    float ss = 0.0f;
    for (int pr = warp; pr < Ph; pr += kMambaThreads / 32) {
        const float xv = xs[pr];
        const float dx = dt * xv;
        float y = 0.0f;
        float* Srow = S + pr * a.N;
        float* Sgrow = Sg + (size_t)pr * a.N;
        for (int n = lane; n < a.N; n += 32) {
            const float sn = fmaf(decay, Srow[n], dx * Bs[n]);
            if (okb) Sgrow[n] = sn;
            y = fmaf(Cs[n], sn, y);
        }
        y = warp_sum(y);
        if (lane == 0) {
            const int c = h * a.P + p0 + pr;
            y = fmaf(Dh, xv, y);
            const float v = y * silu_f(bf16_bits_to_f(zx[c]));
            ss += v * v;
            const float an = v * a.gnorm[c];
            a.act[(size_t)b * a.act_ld + c] = a.act_f16 ? act_bits<true>(an) : act_bits<false>(an);
        }
    }
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    if (tid == 0) {
        float tot = 0.0f;
        for (int w = 0; w < kMambaThreads / 32; ++w) tot += red[w];
        a.parts[(size_t)b * 2 * a.H + h2] = tot;
    }
}

cudaError_t launch_mamba_step(const MambaStepArgs& a, int pdl, cudaStream_t s) {
    const int Ph = a.P / 2;
    const size_t smem = (size_t)(Ph * a.N + Ph + 2 * a.N) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(mamba_step_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2 * a.H, a.B);
    cfg.blockDim = dim3(kMambaThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, mamba_step_kernel, a);
}

// ------------------------------------------------------------------------------------------
// GQA decode attention, split-K over keys
// ------------------------------------------------------------------------------------------
static constexpr int kAttnThreads = 128;
static constexpr int kMaxGQ = 8;

__global__ void __launch_bounds__(kAttnThreads) attn_decode_kernel(const AttnArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ uint64_t bar;
    __shared__ int last_flag;
    pdl_trigger();

    const int split = blockIdx.x, j = blockIdx.y, b = blockIdx.z;
    const int GQ = a.Hq / a.Hk, Dh = a.Dh;
    const int slot = a.slots ? a.slots[b] : b;
    const int t = a.ctx_len[slot];          // cached frames before this one; key t is the new frame
    const int nkeys = t + 1;
    const int nsplit = (nkeys + kAttnSplit - 1) / kAttnSplit;
    if (split >= nsplit || t >= a.cap) return;
    const int k0 = split * kAttnSplit, k1 = min(nkeys, k0 + kAttnSplit), nk = k1 - k0;
    const int tid = threadIdx.x;

    uint16_t* Ks = reinterpret_cast<uint16_t*>(smem);                // [64][Dh]
    uint16_t* Vs = Ks + kAttnSplit * Dh;                                // [64][Dh]
    float* qs = reinterpret_cast<float*>(Vs + kAttnSplit * Dh);         // [GQ][Dh]
    float* ps = qs + GQ * Dh;                                           // [GQ][64]

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
    pdl_wait();
    if (!a.ok[b]) return;
    // the new frame's key/value (written by this frame's qkv projection)
    if (k1 > t) {
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
                        const float* qr = qs + i * Dh + hf * hd + c * 8;
#pragma unroll
                        for (int e = 0; e < 8; ++e) s[i] = fmaf(qr[e], kf[e], s[i]);
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
    {
        const int warp = tid >> 5, lane = tid & 31;
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
    }
    __syncthreads();
    // unnormalised p . V
    for (int d = tid; d < Dh; d += kAttnThreads) {
        float o[kMaxGQ];
#pragma unroll
        for (int i = 0; i < kMaxGQ; ++i) o[i] = 0.0f;
        for (int k = 0; k < nk; ++k) {
            const float v = bf16_bits_to_f(Vs[k * Dh + d]);
#pragma unroll
            for (int i = 0; i < kMaxGQ; ++i)
                if (i < GQ) o[i] = fmaf(ps[i * kAttnSplit + k], v, o[i]);
        }
#pragma unroll
        for (int i = 0; i < kMaxGQ; ++i)
            if (i < GQ) part[i * (Dh + 2) + d] = o[i];
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
    for (int idx = tid; idx < GQ * Dh; idx += kAttnThreads) {
        const int i = idx / Dh, d = idx % Dh;
        float M = -INFINITY;
        for (int sp = 0; sp < nsplit; ++sp) M = fmaxf(M, __ldcg(base + ((size_t)sp * GQ + i) * (Dh + 2) + Dh));
        float L = 0.0f, O = 0.0f;
        for (int sp = 0; sp < nsplit; ++sp) {
            const float* p = base + ((size_t)sp * GQ + i) * (Dh + 2);
            const float w = expf(__ldcg(p + Dh) - M);
            L = fmaf(__ldcg(p + Dh + 1), w, L);
            O = fmaf(__ldcg(p + d), w, O);
        }
        const float o = O / L;
        const size_t col = (size_t)(j * GQ + i) * Dh + d;
        a.act[(size_t)b * a.act_ld + col] = a.act_f16 ? act_bits<true>(o) : act_bits<false>(o);
    }
}

cudaError_t launch_attn_decode(const AttnArgs& a, int pdl, cudaStream_t s) {
    const int GQ = a.Hq / a.Hk;
    const size_t smem = (size_t)2 * kAttnSplit * a.Dh * 2 + (size_t)GQ * a.Dh * 4 + (size_t)GQ * kAttnSplit * 4;
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
