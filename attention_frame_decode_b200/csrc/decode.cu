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
// by the previous frame) and written back once.  (GQA decode attention: attn_decode.cu.)
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
    const uint16_t* et = nullptr;
    const uint16_t* ef = nullptr;
    if (a.emb_t) {
        const int tt = a.tok_t[b], tf = a.tok_f[b];
        if (tt >= 0 && tt < a.Vt) et = a.emb_t + (size_t)tt * a.d;
        if (tf >= 0 && tf < a.Vf) ef = a.emb_f + (size_t)tf * a.d;
    }
    for (int k = threadIdx.x; k < a.d; k += blockDim.x) {
        float v = bf16_bits_to_f(a.x[(size_t)b * a.d + k]);
        if (a.emb_t) {
            if (et) v += bf16_bits_to_f(et[k]);
            if (ef) v += bf16_bits_to_f(ef[k]);
            v = bf16_bits_to_f(act_bits<false>(v));   // the fused input is a bf16 embedding
        }
        a.r[(size_t)b * a.d + k] = v;
        const float an = v * a.gamma[k];
        a.act[(size_t)b * a.act_ld + k] = a.act_f16 ? act_bits<true>(an) : act_bits<false>(an);
        if (a.tap) a.tap[(size_t)b * a.d + k] = v;
    }
    __syncthreads();   // r of this row complete (written by all threads of the CTA)
    for (int u = threadIdx.x; u < a.n_units; u += blockDim.x) {
        float ss = 0.0f;
        const int k1 = min(a.d, (u + 1) * a.unit_rows);
        for (int k = u * a.unit_rows; k < k1; ++k) {
            const float v = a.r[(size_t)b * a.d + k];
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

    // Before griddepcontrol.wait: everything that does not depend on this frame's in_proj output
    // (the frame counter, the W-1 previous pre-conv rows in the ring, the conv weights): the
    // partial conv sums of this CTA's x channels and its group's B, C channels.
    const int t = a.ctx_len[slot];   // advanced only by the last kernel of a step
    uint16_t* ring = a.conv + (size_t)slot * a.W * a.Cx;
    const bool writes_bc = (h % (a.H / a.G) == 0) && half == 0;
    auto channel = [&](int i, float*& dst) -> int {
        if (i < Ph) { dst = xs + i; return h * a.P + p0 + i; }
        if (i < Ph + a.N) { dst = Bs + (i - Ph); return a.E + g * a.N + (i - Ph); }
        dst = Cs + (i - Ph - a.N);
        return a.E + a.G * a.N + g * a.N + (i - Ph - a.N);
    };
    for (int i = tid; i < Ph + 2 * a.N; i += kMambaThreads) {
        float* dst;
        const int c = channel(i, dst);
        float acc = a.conv_b[c];
        for (int k = 0; k < a.W - 1; ++k) {
            const int rs = ((t - (a.W - 1) + k) % a.W + a.W) % a.W;
            acc += a.conv_w[c * a.W + k] * bf16_bits_to_f(ring[(size_t)rs * a.Cx + c]);
        }
        *dst = acc;
    }
    const float dt_bias = a.dt_bias[h], A = -expf(a.A_log[h]), Dh = a.D[h];

    pdl_wait();
    // one round trip for this frame's inputs: x/B/C pre-activations (kept raw for the ring),
    // the gate z and dt_raw; the ring slot t mod W is written at the end
    const bool okb = a.ok ? a.ok[b] != 0 : true;
    const uint16_t* zx = a.zx + (size_t)b * a.zx_ld;
    const uint16_t* xBC = zx + a.E;
    uint16_t raw[2];
    int chan[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        const int i = tid + q * kMambaThreads;
        chan[q] = -1;
        if (i < Ph + 2 * a.N) {
            float* dst;
            chan[q] = channel(i, dst);
            raw[q] = xBC[chan[q]];
        }
    }
    float* zs = Cs + a.N;   // [Ph] silu(z)
    for (int i = tid; i < Ph; i += kMambaThreads) zs[i] = silu_f(bf16_bits_to_f(zx[h * a.P + p0 + i]));
    const float dt_raw = bf16_bits_to_f(zx[a.E + a.Cx + h]);
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        if (chan[q] < 0) continue;
        float* dst;
        channel(tid + q * kMambaThreads, dst);
        *dst = silu_f(*dst + a.conv_w[chan[q] * a.W + a.W - 1] * bf16_bits_to_f(raw[q]));
    }
    __syncthreads();

    const float dt = softplus_f(dt_raw + dt_bias);
    const float decay = expf(A * dt);

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
            const float v = y * zs[pr];
            ss += v * v;
            const float an = v * a.gnorm[c];
            a.act[(size_t)b * a.act_ld + c] = a.act_f16 ? act_bits<true>(an) : act_bits<false>(an);
        }
    }
    if (lane == 0) red[warp] = ss;
    // the ring slot of frame t (disjoint from the W-1 slots any CTA reads this frame)
    if (okb) {
        uint16_t* rw = ring + (size_t)(t % a.W) * a.Cx;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int i = tid + q * kMambaThreads;
            if (chan[q] >= 0 && (i < Ph || writes_bc)) rw[chan[q]] = raw[q];
        }
    }
    __syncthreads();
    if (tid == 0) {
        float tot = 0.0f;
        for (int w = 0; w < kMambaThreads / 32; ++w) tot += red[w];
        a.parts[(size_t)b * 2 * a.H + h2] = tot;
    }
}

bool mamba_step_supported(int P, int N) { return P > 0 && N > 0 && P / 2 + 2 * N <= 2 * kMambaThreads; }

cudaError_t launch_mamba_step(const MambaStepArgs& a, int pdl, cudaStream_t s) {
    const int Ph = a.P / 2;
    if (Ph + 2 * a.N > 2 * kMambaThreads) return cudaErrorInvalidValue;
    const size_t smem = (size_t)(Ph * a.N + 2 * Ph + 2 * a.N) * sizeof(float);
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

}  // namespace vc
