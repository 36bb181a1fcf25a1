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
// grid walks the items, each CTA its own in order.  Two shared-memory tiles alternate between
// items: while item i is updated in one, the fp32 state slice of the next item is bulk-copied into
// the other, and the next item's inputs (conv ring rows, this frame's x/B/C/z/dt_raw) are loaded
// into registers, so no item waits on a chain of global loads.  The first item's state copies are
// issued before griddepcontrol.wait.
// ------------------------------------------------------------------------------------------
static constexpr int kMambaThreads = 256;
static constexpr int kMambaCtasPerSm = 4;
static constexpr int kMambaMaxB = 16;

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
// (with P/2 a multiple of 2, the B and C rows of a tile start on 16-byte boundaries)

// one item's inputs for the thread's channels tid and tid + kMambaThreads (x half, then the
// group's B, then C): the conv sum over the W-1 ring rows before this frame, the last tap's
// weight, this frame's pre-conv value; the gate z of channel tid of the x half; dt_raw
struct MambaIn {
    float acc[2], wl[2], z, dtr;
    uint16_t raw[2];
    int chan[2];
};

// silu with a fast reciprocal-based division (2 ulp), used on the fp32 conv outputs and gates
VC_DEV float silu_fast(float x) { return __fdividef(x, 1.0f + __expf(-x)); }

// The shape is a template (0 = read from the arguments at run time): the Nano backbone's
// (W 4, N 128, P/2 40, H 128, G 8) gets loops with fixed trip counts and item indices by shifts.
template <int W_, int N_, int PH_, int H_, int G_>
__global__ void __launch_bounds__(kMambaThreads, kMambaCtasPerSm) mamba_step_kernel(const MambaStepArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t bar[2];
    __shared__ float red[kMambaThreads / 32];
    __shared__ int s_slot[kMambaMaxB], s_rb[kMambaMaxB], s_wr[kMambaMaxB], s_ok[kMambaMaxB];
    __shared__ float s_dt[2], s_decay[2];
    pdl_trigger();

    const int W = W_ ? W_ : a.W, N = N_ ? N_ : a.N, Ph = PH_ ? PH_ : a.P / 2, H = H_ ? H_ : a.H;
    const int G = G_ ? G_ : a.G;
    const int P = 2 * Ph, H2 = 2 * H;
    const int n_items = a.B * H2;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t tile_bytes = mamba_tile_bytes(Ph, N);
    const uint32_t sbytes = (uint32_t)(Ph * N * 4);
    const int hpg = H / G;
    const int nch = Ph + 2 * N;

    // per session: slot, the ring slot of the oldest of the W-1 rows before this frame and the
    // slot this frame's row goes to (frames cached come from earlier frames); ok after the wait
    for (int b = tid; b < a.B; b += kMambaThreads) {
        const int slot = a.slots ? a.slots[b] : b;
        const int t = a.ctx_len[slot];   // advanced only by the last kernel of a step
        s_slot[b] = slot;
        s_rb[b] = (t + 1) % W;           // (t - (W-1)) mod W
        s_wr[b] = t % W;
    }
    auto item_state = [&](int b, int h2) {
        return a.ssm + (((size_t)s_slot[b] * H + (h2 >> 1)) * P + (h2 & 1) * Ph) * N;
    };
    auto issue_state = [&](int i, int buf) {
        const int b = i / H2, h2 = i - b * H2;
        mbar_arrive_expect_tx(&bar[buf], sbytes);
        bulk_g2s(smem + (size_t)buf * tile_bytes, item_state(b, h2), sbytes, &bar[buf]);
    };
    auto channel = [&](int h, int p0, int g, int ci) -> int {
        if (ci < Ph) return h * P + p0 + ci;
        if (ci < Ph + N) return a.E + g * N + (ci - Ph);
        return a.E + G * N + g * N + (ci - Ph - N);
    };
    // the item's inputs into registers (issued loads; consumed by finish one item later)
    auto load = [&](int i, MambaIn& in) {
        const int b = i / H2, h2 = i - b * H2;
        const int h = h2 >> 1, p0 = (h2 & 1) * Ph, g = h / hpg;
        const int rb = s_rb[b];
        const uint16_t* ring = a.conv + (size_t)s_slot[b] * W * a.Cx;
        const uint16_t* zx = a.zx + (size_t)b * a.zx_ld;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int ci = tid + q * kMambaThreads;
            in.chan[q] = -1;
            in.acc[q] = in.wl[q] = 0.0f;
            in.raw[q] = 0;
            if (ci < nch) {
                const int c = channel(h, p0, g, ci);
                in.chan[q] = c;
                float acc = a.conv_b[c];
                int rs = rb;
#pragma unroll
                for (int w = 0; w < (W_ ? W_ - 1 : 7); ++w) {
                    if (!W_ && w >= W - 1) break;
                    acc += a.conv_w[c * W + w] * bf16_bits_to_f(ring[(size_t)rs * a.Cx + c]);
                    rs = rs + 1 == W ? 0 : rs + 1;
                }
                in.acc[q] = acc;
                in.wl[q] = a.conv_w[c * W + W - 1];
                in.raw[q] = zx[a.E + c];
            }
        }
        in.z = tid < Ph ? bf16_bits_to_f(zx[h * P + p0 + tid]) : 0.0f;
        in.dtr = bf16_bits_to_f(zx[a.E + a.Cx + h]);
    };
    // the loaded inputs into tile T: conv outputs, gate, dt and decay
    auto finish = [&](int i, const MambaIn& in, const MambaTile& T, int buf) {
        const int h = (i % H2) >> 1;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int ci = tid + q * kMambaThreads;
            if (in.chan[q] < 0) continue;
            float* dst = ci < Ph ? T.xs + ci : ci < Ph + N ? T.Bs + (ci - Ph) : T.Cs + (ci - Ph - N);
            *dst = silu_fast(in.acc[q] + in.wl[q] * bf16_bits_to_f(in.raw[q]));
        }
        if (tid < Ph) T.zs[tid] = silu_fast(in.z);
        if (tid == 0) {
            const float dt = softplus_f(in.dtr + a.dt_bias[h]);
            s_dt[buf] = dt;
            s_decay[buf] = expf(-expf(a.A_log[h]) * dt);
        }
    };

    const int first = blockIdx.x;
    __syncthreads();   // session table
    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        fence_mbar_init();
        if (first < n_items) issue_state(first, 0);
        if (first + (int)gridDim.x < n_items) issue_state(first + gridDim.x, 1);
    }
    pdl_wait();
    for (int b = tid; b < a.B; b += kMambaThreads) s_ok[b] = a.ok ? a.ok[b] != 0 : 1;
    __syncthreads();   // barriers, ok table
    MambaIn cur{};
    if (first < n_items) {
        load(first, cur);
        finish(first, cur, mamba_tile(smem, Ph, N), 0);
    }
    __syncthreads();

    int k = 0;
    for (int i = first; i < n_items; i += gridDim.x, ++k) {
        const int buf = k & 1;
        const MambaTile T = mamba_tile(smem + (size_t)buf * tile_bytes, Ph, N);
        const int b = i / H2, h2 = i - b * H2;
        const int h = h2 >> 1, half = h2 & 1, p0 = half * Ph;
        uint16_t* ring = a.conv + (size_t)s_slot[b] * W * a.Cx;
        const bool writes_bc = (h % hpg == 0) && half == 0;
        const bool okb = s_ok[b] != 0;
        const int nx = i + (int)gridDim.x;
        MambaIn nxt{};
        if (nx < n_items) load(nx, nxt);   // in flight during this item's update
        const float dt = s_dt[buf], decay = s_decay[buf], Dh = a.D[h];

        float* Sg = item_state(b, h2);
        // every thread waits for the state copy; if it never arrives the CTA leaves together, after
        // a bounded wait for the other buffer's copy (no copy may land in a CTA that has exited)
        if (!__syncthreads_and(mbar_wait(&bar[buf], (uint32_t)(k >> 1) & 1u, a.status))) {
            if (tid == 0 && nx < n_items) mbar_wait(&bar[buf ^ 1], (uint32_t)((k + 1) >> 1) & 1u, nullptr);
            return;
        }
        float ss = 0.0f;
        for (int pr = warp; pr < Ph; pr += kMambaThreads / 32) {
            const float xv = T.xs[pr];
            const float dx = dt * xv;
            float y = 0.0f;
            const float* Srow = T.S + pr * N;
            float* Sgrow = Sg + (size_t)pr * N;
            if constexpr (N_ == 128) {   // four consecutive states per lane: 16-byte accesses
                const float4 s4 = *reinterpret_cast<const float4*>(Srow + 4 * lane);
                const float4 b4 = *reinterpret_cast<const float4*>(T.Bs + 4 * lane);
                const float4 c4 = *reinterpret_cast<const float4*>(T.Cs + 4 * lane);
                float4 n4;
                n4.x = fmaf(decay, s4.x, dx * b4.x);
                n4.y = fmaf(decay, s4.y, dx * b4.y);
                n4.z = fmaf(decay, s4.z, dx * b4.z);
                n4.w = fmaf(decay, s4.w, dx * b4.w);
                if (okb) *reinterpret_cast<float4*>(Sgrow + 4 * lane) = n4;
                y = fmaf(c4.x, n4.x, fmaf(c4.y, n4.y, fmaf(c4.z, n4.z, c4.w * n4.w)));
            } else {
#pragma unroll
                for (int n0 = 0; n0 < (N_ ? N_ : 256); n0 += 32) {
                    if (!N_ && n0 >= N) break;
                    const int n = n0 + lane;
                    if (!N_ && n >= N) break;
                    const float sn = fmaf(decay, Srow[n], dx * T.Bs[n]);
                    if (okb) Sgrow[n] = sn;
                    y = fmaf(T.Cs[n], sn, y);
                }
            }
            y = warp_sum(y);
            if (lane == 0) {
                const int c = h * P + p0 + pr;
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
            uint16_t* rw = ring + (size_t)s_wr[b] * a.Cx;
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int ci = tid + q * kMambaThreads;
                if (cur.chan[q] >= 0 && (ci < Ph || writes_bc)) rw[cur.chan[q]] = cur.raw[q];
            }
        }
        __syncthreads();   // the buffer is read; red is complete
        if (tid == 0) {
            float tot = 0.0f;
            for (int w = 0; w < kMambaThreads / 32; ++w) tot += red[w];
            a.parts[(size_t)b * H2 + h2] = tot;
            // the buffer's next item: the one after next of this CTA
            if (i + 2 * (int)gridDim.x < n_items) {
                fence_proxy_async();
                issue_state(i + 2 * (int)gridDim.x, buf);
            }
        }
        if (nx < n_items) {
            finish(nx, nxt, mamba_tile(smem + (size_t)(buf ^ 1) * tile_bytes, Ph, N), buf ^ 1);
            cur = nxt;
        }
        __syncthreads();   // the next item's tile inputs are written
    }
}

bool mamba_step_supported(int P, int N) {
    return P > 0 && N > 0 && P / 2 + 2 * N <= 2 * kMambaThreads && P / 2 <= kMambaThreads && N <= 256;
}

cudaError_t launch_mamba_step(const MambaStepArgs& a, int pdl, cudaStream_t s) {
    const int Ph = a.P / 2;
    if (!mamba_step_supported(a.P, a.N) || a.B > kMambaMaxB || a.W > 8 || a.W < 1) return cudaErrorInvalidValue;
    const bool nano = a.W == 4 && a.N == 128 && Ph == 40 && a.H == 128 && a.G == 8;
    auto kern = nano ? mamba_step_kernel<4, 128, 40, 128, 8> : mamba_step_kernel<0, 0, 0, 0, 0>;
    const size_t smem = 2 * mamba_tile_bytes(Ph, a.N);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
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
    return cudaLaunchKernelEx(&cfg, kern, a);
}

}  // namespace vc
