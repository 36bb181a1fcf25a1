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
#include <algorithm>

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
// Mamba-2 step.  Work item = (session b, head h, half of the head's P channels); a persistent
// grid walks the items, each CTA its own in order, with the fp32 state slice of the next item
// bulk-copied into the second of two shared-memory buffers while the current one is updated, so
// the state stream keeps going across items.  The first item's state copy and conv partial sums
// (which depend only on the previous frames) are issued before griddepcontrol.wait.
// ------------------------------------------------------------------------------------------
static constexpr int kMambaThreads = 256;
static constexpr int kMambaCtasPerSm = 4;

struct MambaTile {
    float *S, *xs, *Bs, *Cs, *zs;   // [Ph][N], [Ph], [N], [N], [Ph]
};

__device__ __forceinline__ MambaTile mamba_tile(uint8_t* base, int Ph, int N) {
    MambaTile t;
    t.S = reinterpret_cast<float*>(base);
    t.xs = t.S + Ph * N;
    t.Bs = t.xs + Ph;
    t.Cs = t.Bs + N;
    t.zs = t.Cs + N;
    return t;
}

__host__ __device__ constexpr size_t mamba_tile_bytes(int Ph, int N) {
    return ((size_t)(Ph * N + 2 * Ph + 2 * N) * 4 + 127) / 128 * 128;
}

__global__ void __launch_bounds__(kMambaThreads, kMambaCtasPerSm) mamba_step_kernel(const MambaStepArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t bar[2];
    __shared__ float red[kMambaThreads / 32];
    pdl_trigger();

    const int Ph = a.P / 2;
    const int n_items = a.B * 2 * a.H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t tile_bytes = mamba_tile_bytes(Ph, a.N);
    const uint32_t sbytes = (uint32_t)(Ph * a.N * 4);
    const int hpg = a.H / a.G;

    // item i: (b, h2) with h2 = (h, half); its state slice and ring
    auto item_state = [&](int i) {
        const int b = i / (2 * a.H), h2 = i % (2 * a.H);
        const int slot = a.slots ? a.slots[b] : b;
        return a.ssm + (((size_t)slot * a.H + (h2 >> 1)) * a.P + (h2 & 1) * Ph) * a.N;
    };
    auto issue_state = [&](int i, int buf) {
        mbar_arrive_expect_tx(&bar[buf], sbytes);
        bulk_g2s(smem + (size_t)buf * tile_bytes, item_state(i), sbytes, &bar[buf]);
    };
    // the partial conv sums of an item's channels (its x half, its group's B and C) over the
    // W-1 ring rows before this frame
    auto channel = [&](const MambaTile& T, int h, int p0, int g, int i, float*& dst) -> int {
        if (i < Ph) { dst = T.xs + i; return h * a.P + p0 + i; }
        if (i < Ph + a.N) { dst = T.Bs + (i - Ph); return a.E + g * a.N + (i - Ph); }
        dst = T.Cs + (i - Ph - a.N);
        return a.E + a.G * a.N + g * a.N + (i - Ph - a.N);
    };
    auto conv_partial = [&](const MambaTile& T, int i) {
        const int b = i / (2 * a.H), h2 = i % (2 * a.H);
        const int h = h2 >> 1, p0 = (h2 & 1) * Ph, g = h / hpg;
        const int slot = a.slots ? a.slots[b] : b;
        const int t = a.ctx_len[slot];   // advanced only by the last kernel of a step
        const uint16_t* ring = a.conv + (size_t)slot * a.W * a.Cx;
        for (int k = tid; k < Ph + 2 * a.N; k += kMambaThreads) {
            float* dst;
            const int c = channel(T, h, p0, g, k, dst);
            float acc = a.conv_b[c];
            for (int q = 0; q < a.W - 1; ++q) {
                const int rs = ((t - (a.W - 1) + q) % a.W + a.W) % a.W;
                acc += a.conv_w[c * a.W + q] * bf16_bits_to_f(ring[(size_t)rs * a.Cx + c]);
            }
            *dst = acc;
        }
    };

    int first = blockIdx.x;
    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        fence_mbar_init();
        if (first < n_items) issue_state(first, 0);
        if (first + (int)gridDim.x < n_items) issue_state(first + gridDim.x, 1);
    }
    __syncthreads();
    if (first < n_items) conv_partial(mamba_tile(smem, Ph, a.N), first);

    pdl_wait();

    int k = 0;
    for (int i = first; i < n_items; i += gridDim.x, ++k) {
        const int buf = k & 1;
        const MambaTile T = mamba_tile(smem + (size_t)buf * tile_bytes, Ph, a.N);
        const int b = i / (2 * a.H), h2 = i % (2 * a.H);
        const int h = h2 >> 1, half = h2 & 1, p0 = half * Ph, g = h / hpg;
        const int slot = a.slots ? a.slots[b] : b;
        const int t = a.ctx_len[slot];
        uint16_t* ring = a.conv + (size_t)slot * a.W * a.Cx;
        const bool writes_bc = (h % hpg == 0) && half == 0;
        const bool okb = a.ok ? a.ok[b] != 0 : true;
        if (k > 0) conv_partial(T, i);   // the first item's were computed before the wait
        // this frame's inputs: x/B/C pre-activations (kept raw for the ring), the gate z, dt_raw
        const uint16_t* zx = a.zx + (size_t)b * a.zx_ld;
        const uint16_t* xBC = zx + a.E;
        uint16_t raw[2];
        int chan[2];
        __syncthreads();   // this buffer's conv partial sums are written
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int ci = tid + q * kMambaThreads;
            chan[q] = -1;
            if (ci < Ph + 2 * a.N) {
                float* dst;
                chan[q] = channel(T, h, p0, g, ci, dst);
                raw[q] = xBC[chan[q]];
                *dst = silu_f(*dst + a.conv_w[chan[q] * a.W + a.W - 1] * bf16_bits_to_f(raw[q]));
            }
        }
        for (int ci = tid; ci < Ph; ci += kMambaThreads) T.zs[ci] = silu_f(bf16_bits_to_f(zx[h * a.P + p0 + ci]));
        const float dt = softplus_f(bf16_bits_to_f(zx[a.E + a.Cx + h]) + a.dt_bias[h]);
        const float decay = expf(-expf(a.A_log[h]) * dt);
        const float Dh = a.D[h];
        __syncthreads();

        float* Sg = item_state(i);
        // every thread waits for the state copy; if it never arrives the CTA leaves together, after
        // a bounded wait for the other buffer's copy (no copy may land in a CTA that has exited)
        if (!__syncthreads_and(mbar_wait(&bar[buf], (uint32_t)(k >> 1) & 1u, a.status))) {
            if (tid == 0 && i + (int)gridDim.x < n_items) mbar_wait(&bar[buf ^ 1], (uint32_t)((k + 1) >> 1) & 1u, nullptr);
            return;
        }
        float ss = 0.0f;
        for (int pr = warp; pr < Ph; pr += kMambaThreads / 32) {
            const float xv = T.xs[pr];
            const float dx = dt * xv;
            float y = 0.0f;
            const float* Srow = T.S + pr * a.N;
            float* Sgrow = Sg + (size_t)pr * a.N;
            for (int n = lane; n < a.N; n += 32) {
                const float sn = fmaf(decay, Srow[n], dx * T.Bs[n]);
                if (okb) Sgrow[n] = sn;
                y = fmaf(T.Cs[n], sn, y);
            }
            y = warp_sum(y);
            if (lane == 0) {
                const int c = h * a.P + p0 + pr;
                y = fmaf(Dh, xv, y);
                const float v = y * T.zs[pr];
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
                const int ci = tid + q * kMambaThreads;
                if (chan[q] >= 0 && (ci < Ph || writes_bc)) rw[chan[q]] = raw[q];
            }
        }
        __syncthreads();   // the buffer is read; red is complete
        if (tid == 0) {
            float tot = 0.0f;
            for (int w = 0; w < kMambaThreads / 32; ++w) tot += red[w];
            a.parts[(size_t)b * 2 * a.H + h2] = tot;
            // the buffer's next item: the one after next of this CTA
            const int nx = i + 2 * (int)gridDim.x;
            if (nx < n_items) {
                fence_proxy_async();
                issue_state(nx, buf);
            }
        }
    }
}

bool mamba_step_supported(int P, int N) { return P > 0 && N > 0 && P / 2 + 2 * N <= 2 * kMambaThreads; }

cudaError_t launch_mamba_step(const MambaStepArgs& a, int pdl, cudaStream_t s) {
    const int Ph = a.P / 2;
    if (Ph + 2 * a.N > 2 * kMambaThreads) return cudaErrorInvalidValue;
    const size_t smem = 2 * mamba_tile_bytes(Ph, a.N);
    cudaError_t e = cudaFuncSetAttribute(mamba_step_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int n_items = a.B * 2 * a.H;
    const int grid = std::min(n_items, sms * kMambaCtasPerSm);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
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
