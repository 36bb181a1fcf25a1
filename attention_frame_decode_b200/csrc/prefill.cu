// prefill.cu -- opening-context prefill of one session: all T frames layer by layer.
//
// A streaming session takes in its prompt as one block before the caller's speech
// ("NemotronLabs VoiceChat 11B: GPTQ 3-bit LLM, MLX", "Recipe"): the backbone consumes a context of
// T frames at once.  Per layer:
//   pre-RMSNorm rows (act = bf16(r * gamma), inv_rms per row)
//   Mamba-2 : in_proj GEMM (tcgen05) -> causal conv1d + SiLU over the frames (the last W-1 raw
//             rows go to the session's conv ring) -> chunked SSD (Dao & Gu, "Transformers are
//             SSMs", the SSD algorithm: per chunk of Q = 256 frames the chunk state
//             S_c = sum_j exp(Lam_end - Lam_j) dt_j x_j (outer) B_j, a scan over chunks
//             S_in(c+1) = exp(Lam_end(c)) S_in(c) + S_c, and the outputs
//             y_i = sum_{j<=i} (C_i.B_j) exp(Lam_i - Lam_j) dt_j x_j + exp(Lam_i) C_i.S_in + D x_i)
//             -> gated RMSNorm -> out_proj GEMM + residual
//   attention: qkv GEMM (k, v written to the KV cache rows 0..T-1) -> causal GQA softmax
//             attention -> o_proj GEMM + residual
//   MLP      : up GEMM with squared ReLU -> down GEMM + residual
// The projections (>95% of the FLOPs) run on tcgen05; the chunked SSD and the causal attention on
// warp-level MMA (prefill_mma.cuh); the scan over chunks, conv, norms in fp32 on CUDA cores.
// The call (re)initialises the slot: the SSM state ends as the scan's final state, the conv
// ring holds the last W-1 frames, KV rows 0..T-1 are written and ctx_len[slot] = T.
#include <string.h>

#include <algorithm>
#include <vector>

#include "common.cuh"
#include "gemm_tc.cuh"
#include "gemv.cuh"
#include "prefill_mma.cuh"
#include "prefill.cuh"

namespace vc {

static constexpr int kChunk = 256;   // SSD chunk length (frames)

static size_t al(size_t v) { return (v + 255) / 256 * 256; }

struct PfBufs {
    float *r, *inv, *xc, *dt, *lam, *y, *schunk;
    uint16_t *act_d, *act_big, *zx, *q, *xc16, *sin16;
    uint16_t* wdense[2];   // double buffer: the GEMM reads one while the next weight is unpacked
    int ld_d, ld_big;
};

static PfBufs carve_pf(uint8_t* base, int T, int d, int E, int Cx, int H, int P, int N, int Hq, int Hk, int Dh,
                       int F, size_t* total) {
    PfBufs b{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        uint8_t* p = base ? base + off : nullptr;
        off += al(bytes);
        return p;
    };
    const int nch = (T + kChunk - 1) / kChunk;
    b.ld_d = (d + 127) / 128 * 128;
    int big = std::max(std::max(E, F), Hq * Dh);
    b.ld_big = (big + 127) / 128 * 128;
    const int zxw = E + Cx + H;
    b.r = (float*)take((size_t)T * d * 4);
    b.inv = (float*)take((size_t)T * 4);
    b.act_d = (uint16_t*)take((size_t)T * b.ld_d * 2);
    b.act_big = (uint16_t*)take((size_t)T * b.ld_big * 2);
    b.zx = (uint16_t*)take((size_t)T * std::max(zxw, 1) * 2);
    b.q = (uint16_t*)take((size_t)T * std::max(Hq * Dh, 1) * 2);
    b.xc = (float*)take((size_t)T * std::max(Cx, 1) * 4);
    b.dt = (float*)take((size_t)T * std::max(H, 1) * 4);
    b.lam = (float*)take((size_t)T * std::max(H, 1) * 4);
    b.y = (float*)take((size_t)T * std::max(E, 1) * 4);
    b.schunk = (float*)take((size_t)nch * std::max(H * P * N, 1) * 4);
    b.sin16 = (uint16_t*)take((size_t)nch * std::max(H * P * N, 1) * 2);
    b.xc16 = (uint16_t*)take((size_t)T * std::max(Cx, 1) * 2);
    // the largest linear weight of a layer, unpacked to 16-bit row-major for the GEMM
    size_t wmax = std::max((size_t)zxw * d, (size_t)d * E);
    wmax = std::max(wmax, (size_t)(Hq + 2 * Hk) * Dh * d);
    wmax = std::max(wmax, (size_t)d * Hq * Dh);
    wmax = std::max(wmax, (size_t)F * d);
    b.wdense[0] = (uint16_t*)take(wmax * 2);
    b.wdense[1] = (uint16_t*)take(wmax * 2);
    if (total) *total = off;
    return b;
}

size_t prefill_workspace_bytes(int d, int L, int E, int Cx, int H, int P, int N, int G, int Hq, int Hk, int Dh, int F,
                               int cap) {
    (void)L; (void)G;
    size_t total = 0;
    carve_pf(nullptr, cap, d, E, Cx, H, P, N, Hq, Hk, Dh, F, &total);
    return total;
}

// ------------------------------------------------------------------------------------------
// row kernels
// ------------------------------------------------------------------------------------------
// r = x (first layer) or r (later layers); act = bf16(r * gamma); inv = rsqrt(mean(r^2) + eps)
__global__ void pf_rownorm_kernel(const uint16_t* x, float* r, const float* gamma, uint16_t* act, int ld, float* inv,
                                  int d, float eps, int f16) {
    const int t = blockIdx.x;
    float* rr = r + (size_t)t * d;
    uint16_t* ar = act + (size_t)t * ld;
    float ss = 0.0f;
    if ((d & 3) == 0 && (ld & 3) == 0) {   // 4 columns per step: 16-byte r, 8-byte act accesses
        for (int k = 4 * threadIdx.x; k < d; k += 4 * blockDim.x) {
            float4 v;
            if (x) {
                const uint2 xb = *reinterpret_cast<const uint2*>(x + (size_t)t * d + k);
                v = make_float4(bf16_bits_to_f((uint16_t)(xb.x & 0xFFFFu)), bf16_bits_to_f((uint16_t)(xb.x >> 16)),
                                bf16_bits_to_f((uint16_t)(xb.y & 0xFFFFu)), bf16_bits_to_f((uint16_t)(xb.y >> 16)));
                *reinterpret_cast<float4*>(rr + k) = v;
            } else {
                v = *reinterpret_cast<const float4*>(rr + k);
            }
            ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
            const float4 g = *reinterpret_cast<const float4*>(gamma + k);
            uint2 o;
            if (f16) {
                o.x = (uint32_t)act_bits<true>(v.x * g.x) | ((uint32_t)act_bits<true>(v.y * g.y) << 16);
                o.y = (uint32_t)act_bits<true>(v.z * g.z) | ((uint32_t)act_bits<true>(v.w * g.w) << 16);
            } else {
                o.x = (uint32_t)act_bits<false>(v.x * g.x) | ((uint32_t)act_bits<false>(v.y * g.y) << 16);
                o.y = (uint32_t)act_bits<false>(v.z * g.z) | ((uint32_t)act_bits<false>(v.w * g.w) << 16);
            }
            *reinterpret_cast<uint2*>(ar + k) = o;
        }
    } else {
        for (int k = threadIdx.x; k < d; k += blockDim.x) {
            float v;
            if (x) {
                v = bf16_bits_to_f(x[(size_t)t * d + k]);
                rr[k] = v;
            } else {
                v = rr[k];
            }
            ss += v * v;
            ar[k] = f16 ? act_bits<true>(v * gamma[k]) : act_bits<false>(v * gamma[k]);
        }
    }
    __shared__ float red[32];
    ss = warp_sum(ss);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x == 0) {
        float s = 0.0f;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s += red[w];
        inv[t] = rsqrtf(s / d + eps);
    }
}

// causal depthwise conv1d + SiLU over the frames (zero history), a tile of 64 frames x 256
// channels per CTA: each thread keeps its channel's W taps and last W-1 inputs in registers, so
// every input row is read once and every access is coalesced across the channels.  The last W-1
// raw pre-conv rows go to the conv ring (frame t in slot t mod W).
static constexpr int kConvTF = 64;

template <int WC>   // conv width when fixed at compile time (the backbone's 4), else 0: runtime W <= 8
__global__ void __launch_bounds__(256) pf_conv_kernel(const uint16_t* __restrict__ zx, int zxw, int T, int E, int Cx,
                                                      int Wr, const float* __restrict__ conv_w,
                                                      const float* __restrict__ conv_b, float* __restrict__ xc,
                                                      uint16_t* __restrict__ xc16, uint16_t* __restrict__ ring) {
    const int W = WC ? WC : Wr;
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= Cx) return;
    const int t0 = blockIdx.y * kConvTF, t1 = min(T, t0 + kConvTF);
    const uint16_t* col = zx + E + c;
    float w[8], hist[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        w[k] = k < W ? conv_w[c * W + k] : 0.0f;
        const int tt = t0 - (W - 1) + k;
        hist[k] = (k < W - 1 && tt >= 0) ? bf16_bits_to_f(col[(size_t)tt * zxw]) : 0.0f;
    }
    const float bias = conv_b[c];
    constexpr int U = 8;   // frames whose inputs are loaded together
    for (int tb = t0; tb < t1; tb += U) {
      uint16_t raws[U];
#pragma unroll
      for (int u = 0; u < U; ++u) raws[u] = tb + u < t1 ? col[(size_t)(tb + u) * zxw] : (uint16_t)0;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int t = tb + u;
        if (t >= t1) break;
        const uint16_t raw = raws[u];
        const float xv = bf16_bits_to_f(raw);
        float acc = bias;
#pragma unroll
        for (int k = 0; k < 7; ++k)
            if (k < W - 1) acc += w[k] * hist[k];
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (k == W - 1) acc += w[k] * xv;
#pragma unroll
        for (int k = 0; k < 7; ++k)
            if (k < W - 2) hist[k] = hist[k + 1];
#pragma unroll
        for (int k = 0; k < 7; ++k)
            if (k == W - 2) hist[k] = xv;
        const float v = silu_f(acc);
        xc[(size_t)t * Cx + c] = v;
        xc16[(size_t)t * Cx + c] = f16_bits(v);
        if (t >= T - (W - 1)) ring[(size_t)(t % W) * Cx + c] = raw;
      }
    }
}

// dt = softplus(dt_raw + dt_bias) for every frame and head
// the same for conv width 4 with 4 adjacent channels per thread (8-byte input loads, 16- and
// 8-byte output stores); requires E, Cx and the zx row width to be multiples of 4
__global__ void __launch_bounds__(256) pf_conv4x4_kernel(const uint16_t* __restrict__ zx, int zxw, int T, int E, int Cx,
                                                         const float* __restrict__ conv_w,
                                                         const float* __restrict__ conv_b, float* __restrict__ xc,
                                                         uint16_t* __restrict__ xc16, uint16_t* __restrict__ ring) {
    constexpr int W = 4;
    const int c = 4 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (c >= Cx) return;
    const int t0 = blockIdx.y * kConvTF, t1 = min(T, t0 + kConvTF);
    const uint16_t* col = zx + E + c;
    float w[4][W], hist[4][W - 1], bias[4];
    auto unpack = [](uint2 v, float (&f)[4]) {
        f[0] = bf16_bits_to_f((uint16_t)(v.x & 0xFFFFu));
        f[1] = bf16_bits_to_f((uint16_t)(v.x >> 16));
        f[2] = bf16_bits_to_f((uint16_t)(v.y & 0xFFFFu));
        f[3] = bf16_bits_to_f((uint16_t)(v.y >> 16));
    };
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
        bias[ch] = conv_b[c + ch];
#pragma unroll
        for (int k = 0; k < W; ++k) w[ch][k] = conv_w[(c + ch) * W + k];
    }
#pragma unroll
    for (int k = 0; k < W - 1; ++k) {
        const int tt = t0 - (W - 1) + k;
        float f[4] = {0.f, 0.f, 0.f, 0.f};
        if (tt >= 0) unpack(*reinterpret_cast<const uint2*>(col + (size_t)tt * zxw), f);
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) hist[ch][k] = f[ch];
    }
    constexpr int U = 8;   // frames whose inputs are loaded together
    for (int tb = t0; tb < t1; tb += U) {
        uint2 raws[U];
#pragma unroll
        for (int u = 0; u < U; ++u)
            raws[u] = tb + u < t1 ? *reinterpret_cast<const uint2*>(col + (size_t)(tb + u) * zxw) : make_uint2(0u, 0u);
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int t = tb + u;
            if (t >= t1) break;
            float xv[4], v[4];
            unpack(raws[u], xv);
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                float acc = bias[ch];
#pragma unroll
                for (int k = 0; k < W - 1; ++k) acc += w[ch][k] * hist[ch][k];
                acc += w[ch][W - 1] * xv[ch];
#pragma unroll
                for (int k = 0; k < W - 2; ++k) hist[ch][k] = hist[ch][k + 1];
                hist[ch][W - 2] = xv[ch];
                v[ch] = silu_f(acc);
            }
            *reinterpret_cast<float4*>(xc + (size_t)t * Cx + c) = make_float4(v[0], v[1], v[2], v[3]);
            *reinterpret_cast<uint2*>(xc16 + (size_t)t * Cx + c) =
                make_uint2((uint32_t)f16_bits(v[0]) | ((uint32_t)f16_bits(v[1]) << 16),
                           (uint32_t)f16_bits(v[2]) | ((uint32_t)f16_bits(v[3]) << 16));
            if (t >= T - (W - 1)) *reinterpret_cast<uint2*>(ring + (size_t)(t % W) * Cx + c) = raws[u];
        }
    }
}

__global__ void pf_dt_kernel(const uint16_t* __restrict__ zx, int zxw, int T, int off, int H,
                             const float* __restrict__ dt_bias, float* __restrict__ dt) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (long long)T * H) return;
    const int t = (int)(i / H), h = (int)(i % H);
    dt[i] = softplus_f(bf16_bits_to_f(zx[(size_t)t * zxw + off + h]) + dt_bias[h]);
}

// ------------------------------------------------------------------------------------------
// chunked SSD
// ------------------------------------------------------------------------------------------
// per (chunk, head): inclusive cumulative log decay Lam and the chunk state
//   S_c[p][n] = sum_j exp(Lam_end - Lam_j) dt_j x_j[p] B_j[n]
// in fp32 (the state the decode steps continue from), frames staged 32 at a time in shared
// memory; a 16 x 16 thread grid, each thread RP x RN outputs (p = pg + 16 r, n = ng + 16 q)
static constexpr int kStJ = 32;

template <int RP, int RN>
__global__ void __launch_bounds__(256) pf_ssd_state_kernel(const float* __restrict__ xc, const float* __restrict__ dt,
                                                           const float* __restrict__ A_log, int T, int H, int P, int N,
                                                           int G, int E, int Cx, float* __restrict__ lam,
                                                           float* __restrict__ schunk) {
    const int c = blockIdx.x, h = blockIdx.y;
    const int t0 = c * kChunk, len = min(kChunk, T - t0);
    const int g = (int)((long long)h * G / H);
    __shared__ float w[kChunk];
    __shared__ float lam_s[kChunk];
    __shared__ double lamd[kChunk];   // the same sums, unrounded
    extern __shared__ float stage[];   // xw [kStJ][P], bs [kStJ][N]
    float* xw = stage;
    float* bs = stage + kStJ * P;
    const float A = -expf(A_log[h]);
    // inclusive scan of A*dt over the chunk (one warp), summed in double (see the tensor-core
    // state kernel): each Lam is rounded to fp32 once
    if (threadIdx.x < 32) {
        double run = 0.0;
        for (int base = 0; base < len; base += 32) {
            const int i = base + threadIdx.x;
            double v = i < len ? (double)(A * dt[(size_t)(t0 + i) * H + h]) : 0.0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const double u = __shfl_up_sync(0xffffffffu, v, o);
                if ((int)threadIdx.x >= o) v += u;
            }
            v += run;
            if (i < len) {
                lam_s[i] = (float)v;
                lamd[i] = v;
            }
            run = __shfl_sync(0xffffffffu, v, 31);
        }
    }
    __syncthreads();
    const double lend = lamd[len - 1];   // weights from differences of the unrounded sums
    for (int i = threadIdx.x; i < len; i += blockDim.x) {
        w[i] = expf((float)(lend - lamd[i])) * dt[(size_t)(t0 + i) * H + h];
        lam[(size_t)(t0 + i) * H + h] = lam_s[i];
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ng = lane & 15, pg = warp * 2 + (lane >> 4);
    float acc[RP][RN];
#pragma unroll
    for (int r = 0; r < RP; ++r)
#pragma unroll
        for (int q = 0; q < RN; ++q) acc[r][q] = 0.0f;
    const float* xh = xc + (size_t)t0 * Cx + (size_t)h * P;
    const float* bg = xc + (size_t)t0 * Cx + E + (size_t)g * N;
    for (int jb = 0; jb < len; jb += kStJ) {
        const int nj = min(kStJ, len - jb);
        __syncthreads();   // w ready (first pass) / previous stage consumed
        const int P4 = P / 4, N4 = N / 4;
#pragma unroll 4
        for (int idx = threadIdx.x; idx < nj * P4; idx += blockDim.x) {
            const int j = idx / P4, q = idx - j * P4;
            float4 v = *reinterpret_cast<const float4*>(xh + (size_t)(jb + j) * Cx + 4 * q);
            const float wj = w[jb + j];
            v.x *= wj; v.y *= wj; v.z *= wj; v.w *= wj;
            *reinterpret_cast<float4*>(xw + j * P + 4 * q) = v;
        }
#pragma unroll 4
        for (int idx = threadIdx.x; idx < nj * N4; idx += blockDim.x) {
            const int j = idx / N4, q = idx - j * N4;
            *reinterpret_cast<float4*>(bs + j * N + 4 * q) =
                *reinterpret_cast<const float4*>(bg + (size_t)(jb + j) * Cx + 4 * q);
        }
        __syncthreads();
        for (int j = 0; j < nj; ++j) {
            float xv[RP], bv[RN];
#pragma unroll
            for (int r = 0; r < RP; ++r) xv[r] = pg + 16 * r < P ? xw[j * P + pg + 16 * r] : 0.0f;
#pragma unroll
            for (int q = 0; q < RN; ++q) bv[q] = ng + 16 * q < N ? bs[j * N + ng + 16 * q] : 0.0f;
#pragma unroll
            for (int r = 0; r < RP; ++r)
#pragma unroll
                for (int q = 0; q < RN; ++q) acc[r][q] = fmaf(xv[r], bv[q], acc[r][q]);
        }
    }
    float* S = schunk + ((size_t)c * H + h) * P * N;
#pragma unroll
    for (int r = 0; r < RP; ++r)
#pragma unroll
        for (int q = 0; q < RN; ++q) {
            const int p = pg + 16 * r, n = ng + 16 * q;
            if (p < P && n < N) S[(size_t)p * N + n] = acc[r][q];
        }
}

// scan over chunks: S_in(0) = 0, S_in(c+1) = exp(Lam_end(c)) S_in(c) + S_c; final -> ssm state.
// The chunk states and decays of 8 chunks are loaded before their part of the recurrence, so
// the loads overlap instead of following the chain one by one.
__global__ void pf_ssd_scan_kernel(const float* schunk, const float* lam, int T, int H, int P, int N,
                                   uint16_t* sin16, float* ssm_out) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long per_head = (long long)P * N;
    if (idx >= (long long)H * per_head) return;
    const int h = (int)(idx / per_head);
    const int nch = (T + kChunk - 1) / kChunk;
    const size_t cs = (size_t)H * per_head;
    float s = 0.0f;
    for (int c0 = 0; c0 < nch; c0 += 8) {
        float sc[8], dec[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int c = c0 + k;
            sc[k] = dec[k] = 0.0f;
            if (c < nch) {
                sc[k] = schunk[(size_t)c * cs + idx];
                dec[k] = lam[(size_t)(min(T, (c + 1) * kChunk) - 1) * H + h];
            }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (c0 + k < nch) {
                sin16[(size_t)(c0 + k) * cs + idx] = bf16_bits(s);
                s = expf(dec[k]) * s + sc[k];
            }
    }
    ssm_out[idx] = s;
}

// v = y * silu(z); per row and norm group: act = bf16(v * rsqrt(mean(v^2) + eps) * gamma).
// CTA = one frame, one warp per norm group (warp-level reductions only).  Groups of a multiple
// of 128 columns: each lane takes 4 consecutive columns per step (16-byte y, 8-byte z loads)
// and keeps v in registers between the two passes.
static constexpr int kGnMaxPerLane = 64;   // vector path: group size up to 32 x 64 columns

template <int STEPS>   // 128-column steps per group when fixed at compile time (the backbone's 10), else 0
__global__ void pf_gated_norm_kernel(const float* __restrict__ y, const uint16_t* __restrict__ zx, int zxw,
                                     const float* __restrict__ gnorm, int E, int NG, float eps,
                                     uint16_t* __restrict__ act, int ld, int f16) {
    const int t = blockIdx.x, q = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (q >= NG) return;
    const int gs = E / NG, c0 = q * gs;
    const float* yr = y + (size_t)t * E;
    const uint16_t* zr = zx + (size_t)t * zxw;
    uint16_t* ar = act + (size_t)t * ld;
    const bool vec = STEPS ? true
                           : (gs & 127) == 0 && gs / 32 <= kGnMaxPerLane && (zxw & 3) == 0 && (ld & 3) == 0 && (E & 3) == 0;
    if (vec) {
        float v[kGnMaxPerLane];
        const int steps = STEPS ? STEPS : gs / 128;
        float ss = 0.0f;
#pragma unroll
        for (int k = 0; k < kGnMaxPerLane / 4; ++k) {
            if (k >= steps) break;
            const int c = c0 + 128 * k + 4 * lane;
            const float4 y4 = *reinterpret_cast<const float4*>(yr + c);
            const uint2 z4 = *reinterpret_cast<const uint2*>(zr + c);
            v[4 * k] = y4.x * silu_f(bf16_bits_to_f((uint16_t)(z4.x & 0xFFFFu)));
            v[4 * k + 1] = y4.y * silu_f(bf16_bits_to_f((uint16_t)(z4.x >> 16)));
            v[4 * k + 2] = y4.z * silu_f(bf16_bits_to_f((uint16_t)(z4.y & 0xFFFFu)));
            v[4 * k + 3] = y4.w * silu_f(bf16_bits_to_f((uint16_t)(z4.y >> 16)));
            ss += v[4 * k] * v[4 * k] + v[4 * k + 1] * v[4 * k + 1] + v[4 * k + 2] * v[4 * k + 2] +
                  v[4 * k + 3] * v[4 * k + 3];
        }
        ss = warp_sum(ss);
        const float ginv = rsqrtf(ss / gs + eps);
#pragma unroll
        for (int k = 0; k < kGnMaxPerLane / 4; ++k) {
            if (k >= steps) break;
            const int c = c0 + 128 * k + 4 * lane;
            const float4 g4 = *reinterpret_cast<const float4*>(gnorm + c);
            const float u0 = v[4 * k] * ginv * g4.x, u1 = v[4 * k + 1] * ginv * g4.y;
            const float u2 = v[4 * k + 2] * ginv * g4.z, u3 = v[4 * k + 3] * ginv * g4.w;
            uint2 o;
            if (f16) {
                o.x = (uint32_t)act_bits<true>(u0) | ((uint32_t)act_bits<true>(u1) << 16);
                o.y = (uint32_t)act_bits<true>(u2) | ((uint32_t)act_bits<true>(u3) << 16);
            } else {
                o.x = (uint32_t)act_bits<false>(u0) | ((uint32_t)act_bits<false>(u1) << 16);
                o.y = (uint32_t)act_bits<false>(u2) | ((uint32_t)act_bits<false>(u3) << 16);
            }
            *reinterpret_cast<uint2*>(ar + c) = o;
        }
        return;
    }
    float ss = 0.0f;
#pragma unroll 4
    for (int c = c0 + lane; c < c0 + gs; c += 32) {
        const float v = yr[c] * silu_f(bf16_bits_to_f(zr[c]));
        ss += v * v;
    }
    ss = warp_sum(ss);
    const float ginv = rsqrtf(ss / gs + eps);
#pragma unroll 4
    for (int c = c0 + lane; c < c0 + gs; c += 32) {
        const float u = yr[c] * silu_f(bf16_bits_to_f(zr[c])) * ginv * gnorm[c];
        ar[c] = f16 ? act_bits<true>(u) : act_bits<false>(u);
    }
}

// ------------------------------------------------------------------------------------------
// causal GQA attention for head dimensions without a tensor-core instance (multiples of 32 up
// to 256): fp32, online softmax, one warp per (frame, query head) over the KV cache rows just
// written
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) pf_attn_scalar_kernel(const uint16_t* q, const uint16_t* kc, const uint16_t* vc, int T,
                                                      int Hq, int Hk, int Dh, int cap, uint16_t* out, int ld,
                                                      int f16) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + warp;
    const int i = blockIdx.y;
    if (t >= T) return;
    const int j = (int)((long long)i * Hk / Hq);
    const float scale = rsqrtf((float)Dh);
    const int per = Dh / 32;   // dims per lane (Dh <= 256)
    float qv[8], o[8];
    for (int e = 0; e < per; ++e) {
        qv[e] = bf16_bits_to_f(q[(size_t)t * Hq * Dh + (size_t)i * Dh + lane * per + e]) * scale;
        o[e] = 0.0f;
    }
    const uint16_t* K = kc + (size_t)j * cap * Dh;
    const uint16_t* V = vc + (size_t)j * cap * Dh;
    float m = -INFINITY, l = 0.0f;
    for (int tau = 0; tau <= t; ++tau) {
        float s = 0.0f;
        for (int e = 0; e < per; ++e) s = fmaf(qv[e], bf16_bits_to_f(K[(size_t)tau * Dh + lane * per + e]), s);
        s = warp_sum(s);
        const float mn = fmaxf(m, s);
        const float corr = expf(m - mn), p = expf(s - mn);
        l = l * corr + p;
        for (int e = 0; e < per; ++e) o[e] = o[e] * corr + p * bf16_bits_to_f(V[(size_t)tau * Dh + lane * per + e]);
        m = mn;
    }
    for (int e = 0; e < per; ++e) {
        const float u = o[e] / l;
        out[(size_t)t * ld + (size_t)i * Dh + lane * per + e] = f16 ? act_bits<true>(u) : act_bits<false>(u);
    }
}

__global__ void pf_finish_kernel(int32_t* ctx_len, int slot, int T) { ctx_len[slot] = T; }

// ------------------------------------------------------------------------------------------
// Mamba-2 mixer over the frames (conv -> chunked SSD -> gated norm), shared by the prefill and
// its kernel-level test entry
// ------------------------------------------------------------------------------------------
size_t prefill_mixer_scratch_bytes(int T, int E, int Cx, int H, int P, int N) {
    const size_t nch = (size_t)(T + kChunk - 1) / kChunk;
    return al((size_t)T * Cx * 4) + 2 * al((size_t)T * H * 4) + al((size_t)T * E * 4) + al(nch * H * P * N * 4) +
           al(nch * H * P * N * 2) + al((size_t)T * Cx * 2) + al(4);
}

void carve_mixer(PfMixer& m, uint8_t* base) {
    const size_t nch = (size_t)(m.T + kChunk - 1) / kChunk;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        uint8_t* p = base + off;
        off += al(bytes);
        return (float*)p;
    };
    m.xc = take((size_t)m.T * m.Cx * 4);
    m.dt = take((size_t)m.T * m.H * 4);
    m.lam = take((size_t)m.T * m.H * 4);
    m.y = take((size_t)m.T * m.E * 4);
    m.schunk = take(nch * m.H * m.P * m.N * 4);
    m.sin16 = (uint16_t*)take(nch * m.H * m.P * m.N * 2);
    m.xc16 = (uint16_t*)take((size_t)m.T * m.Cx * 2);
    m.status = (int*)take(4);
}

cudaError_t prefill_mixer(const PfMixer& m, cudaStream_t s) {
    const int T = m.T, E = m.E, Cx = m.Cx, H = m.H, P = m.P, N = m.N, W = m.W;
    const int zxw = E + Cx + H;
    const int nch = (T + kChunk - 1) / kChunk;
    const vc_layer_weights& Lw = *m.Lw;
    if (P % 8 || P > 128 || N % 16 || N > 256 || H % m.G) return cudaErrorNotSupported;
    const SsdLayout SL = ssd_layout(N, P);
    if (SL.total > 227 * 1024) return cudaErrorNotSupported;
    cudaError_t e = cudaFuncSetAttribute(pf_ssd_out_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SL.total);
    if (e != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(m.ring, 0, (size_t)W * Cx * 2, s)) != cudaSuccess) return e;
    if (W > 8 || m.NG > 32) return cudaErrorNotSupported;
    const dim3 cg((Cx + 255) / 256, (T + kConvTF - 1) / kConvTF);
    if (W == 4 && E % 4 == 0 && Cx % 4 == 0 && zxw % 4 == 0)
        pf_conv4x4_kernel<<<dim3((Cx / 4 + 255) / 256, (T + kConvTF - 1) / kConvTF), 256, 0, s>>>(
            m.zx, zxw, T, E, Cx, Lw.conv_w, Lw.conv_b, m.xc, m.xc16, m.ring);
    else if (W == 4)
        pf_conv_kernel<4><<<cg, 256, 0, s>>>(m.zx, zxw, T, E, Cx, W, Lw.conv_w, Lw.conv_b, m.xc, m.xc16, m.ring);
    else
        pf_conv_kernel<0><<<cg, 256, 0, s>>>(m.zx, zxw, T, E, Cx, W, Lw.conv_w, Lw.conv_b, m.xc, m.xc16, m.ring);
    pf_dt_kernel<<<(unsigned)(((long long)T * H + 255) / 256), 256, 0, s>>>(m.zx, zxw, T, E + Cx, H, Lw.dt_bias, m.dt);
    const size_t st_smem = (size_t)kStJ * (P + N) * 4;
    const dim3 sg(nch, H);
    const bool st_mma = N % 16 == 0 && N <= 128 && (P == 80 || P == 32);
    const StateLayout STL = state_layout(N, P);
    if (m.status && ssd_state_tc_supported(N, P, E, Cx)) {
        if ((e = launch_ssd_state_tc(m.xc, m.dt, Lw.A_log, T, H, P, N, m.G, E, Cx, m.lam, m.schunk, m.status, s)) !=
            cudaSuccess)
            return e;
    } else if (st_mma) {
        auto kst = P == 80 ? pf_ssd_state_mma_kernel<5> : pf_ssd_state_mma_kernel<2>;
        if ((e = cudaFuncSetAttribute(kst, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)STL.total)) != cudaSuccess)
            return e;
        kst<<<sg, 256, STL.total, s>>>(m.xc, m.dt, Lw.A_log, T, H, P, N, m.G, E, Cx, m.lam, m.schunk);
    } else if (P <= 80 && P > 64 && N <= 128 && N > 112)
        pf_ssd_state_kernel<5, 8><<<sg, 256, st_smem, s>>>(m.xc, m.dt, Lw.A_log, T, H, P, N, m.G, E, Cx, m.lam,
                                                             m.schunk);
    else if (P <= 32 && N <= 16)
        pf_ssd_state_kernel<2, 1><<<sg, 256, st_smem, s>>>(m.xc, m.dt, Lw.A_log, T, H, P, N, m.G, E, Cx, m.lam,
                                                             m.schunk);
    else
        pf_ssd_state_kernel<8, 16><<<sg, 256, st_smem, s>>>(m.xc, m.dt, Lw.A_log, T, H, P, N, m.G, E, Cx, m.lam,
                                                              m.schunk);
    const long long n = (long long)H * P * N;
    pf_ssd_scan_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(m.schunk, m.lam, T, H, P, N, m.sin16, m.ssm);
    if (m.status && ssd_out_tc_supported(N, P, E, Cx)) {
        if ((e = launch_ssd_out_tc(m.xc16, m.sin16, m.dt, m.lam, Lw.D, m.y, T, H, P, N, m.G, E, Cx, m.status, s)) !=
            cudaSuccess)
            return e;
    } else {
        pf_ssd_out_mma_kernel<<<dim3(nch, m.G, kChunk / kSsdTi), 256, SL.total, s>>>(m.xc, m.xc16, m.dt, m.lam, m.sin16,
                                                                                     Lw.D, T, H, P, N, m.G, E, Cx, m.y);
    }
    // groups of 1280 columns (the backbone's) with aligned rows: the fixed-step instance, whose
    // ten 16-byte loads per lane are all issued before the first is used
    if (E / m.NG == 1280 && E % m.NG == 0 && zxw % 4 == 0 && m.act_ld % 4 == 0 && E % 4 == 0)
        pf_gated_norm_kernel<10><<<T, 32 * m.NG, 0, s>>>(m.y, m.zx, zxw, Lw.gnorm, E, m.NG, m.eps, m.act, m.act_ld,
                                                         m.f16);
    else
        pf_gated_norm_kernel<0><<<T, 32 * m.NG, 0, s>>>(m.y, m.zx, zxw, Lw.gnorm, E, m.NG, m.eps, m.act, m.act_ld,
                                                        m.f16);
    return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// orchestration
// ------------------------------------------------------------------------------------------
// The projections of one prefill, in order.  Weight i is unpacked (device layout -> row-major
// 16-bit) into buffer i % 2 on the side stream while GEMM i - 1 runs on the caller's stream:
//   side: wait "GEMM i-2 done" -> unpack i -> record "unpacked i % 2"
//   main: wait "unpacked i % 2" -> GEMM i -> record "GEMM done i % 2"
struct PfGemm {
    const PrefillCtx& c;
    const PfBufs& b;
    int f16;
    cudaStream_t s;
    std::vector<const vc_qmat*> seq;
    size_t next = 0;   // index of the next GEMM

    cudaError_t unpack(size_t i) {
        if (i >= seq.size()) return cudaSuccess;
        const vc_qmat& w = *seq[i];
        const int k = (int)(i & 1);
        cudaError_t e = cudaStreamWaitEvent(c.side, i >= 2 ? c.ev[2 + k] : c.ev[4], 0);
        if (e == cudaSuccess)
            e = launch_unpack16(w.fmt, w.fmt == VC_W_BF16 ? 64 : w.group, w.N, w.K, (const uint8_t*)w.data,
                                b.wdense[k], w.K, f16, c.side);
        if (e == cudaSuccess) e = cudaEventRecord(c.ev[k], c.side);
        return e;
    }
    cudaError_t start() {
        cudaError_t e = cudaEventRecord(c.ev[4], s);   // buffers free once the caller's prior work is done
        if (e == cudaSuccess) e = unpack(0);
        return e;
    }
    // out = epilogue(A . w^T) for the next weight of the sequence
    cudaError_t operator()(int epi, const uint16_t* A, int lda, int M, const vc_qmat& w, const float* row_scale,
                           uint16_t* out, int ldo, float* out32, int ldo32, const GemmArgs* qkv = nullptr) {
        const size_t i = next++;
        if (i >= seq.size() || seq[i] != &w) return cudaErrorInvalidValue;
        const int k = (int)(i & 1);
        cudaError_t e = cudaStreamWaitEvent(s, c.ev[k], 0);
        if (e != cudaSuccess) return e;
        GemmArgs a = qkv ? *qkv : GemmArgs{};
        a.f16 = f16; a.out_f16 = f16;
        a.A = A; a.lda = lda; a.M = M;
        a.W = b.wdense[k]; a.ldw = w.K; a.N = w.N; a.K = w.K;
        a.row_scale = row_scale; a.out = out; a.ldo = ldo; a.out_f32 = out32; a.ldo32 = ldo32; a.status = c.status;
        if ((e = launch_gemm_tc(epi, a, s)) != cudaSuccess) return e;
        if ((e = cudaEventRecord(c.ev[2 + k], s)) != cudaSuccess) return e;
        return unpack(i + 1);
    }
};

cudaError_t run_prefill(const PrefillCtx& c, const uint16_t* x, int T, int slot, cudaStream_t s) {
    const int d = c.d, E = c.E, Cx = c.Cx, H = c.H, P = c.P, N = c.N, W = c.W;
    const int zxw = E + Cx + H;
    if (T < 1 || T > c.cap) return cudaErrorInvalidValue;
    if (strchr(c.cfg->pattern, '*') && (c.Dh % 32 || c.Dh > 256)) return cudaErrorNotSupported;
    const PfBufs b = carve_pf(c.ws, T, d, E, Cx, H, P, N, c.Hq, c.Hk, c.Dh, c.F, nullptr);
    const int f16 = c.cfg->wfmt != VC_W_BF16;   // quantized weights: fp16 operands, as in the decode GEMV
    PfGemm gemm{c, b, f16, s, {}, 0};
    for (int l = 0; l < c.L; ++l) {
        const vc_layer_weights& Lw = c.layers[l];
        const char kind = c.cfg->pattern[l];
        if (kind == 'M') gemm.seq.insert(gemm.seq.end(), {&Lw.in_proj, &Lw.out_proj});
        else if (kind == '*') gemm.seq.insert(gemm.seq.end(), {&Lw.qkv, &Lw.o});
        else gemm.seq.insert(gemm.seq.end(), {&Lw.up, &Lw.down});
    }
    const float eps = c.cfg->eps;
    cudaError_t e = gemm.start();
    if (e != cudaSuccess) return e;
    pf_rownorm_kernel<<<T, 256, 0, s>>>(x, b.r, c.layers[0].norm, b.act_d, b.ld_d, b.inv, d, eps, f16);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t rbytes = (size_t)T * d * 4;
    if (c.tap && (e = cudaMemcpyAsync(c.tap, b.r, rbytes, cudaMemcpyDeviceToDevice, s)) != cudaSuccess) return e;
    int mi = 0, ai = 0;
    for (int l = 0; l < c.L; ++l) {
        const vc_layer_weights& Lw = c.layers[l];
        const char kind = c.cfg->pattern[l];
        if (l > 0) {
            pf_rownorm_kernel<<<T, 256, 0, s>>>(nullptr, b.r, Lw.norm, b.act_d, b.ld_d, b.inv, d, eps, f16);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
        if (kind == 'M') {
            PfMixer m{};
            m.T = T; m.E = E; m.Cx = Cx; m.H = H; m.P = P; m.N = N; m.G = c.G; m.W = W; m.NG = c.NG;
            m.eps = eps; m.f16 = f16; m.Lw = &Lw;
            m.xc = b.xc; m.dt = b.dt; m.lam = b.lam; m.y = b.y; m.schunk = b.schunk; m.sin16 = b.sin16; m.xc16 = b.xc16;
            m.ssm = c.ssm + ((size_t)mi * c.n_slots + slot) * H * P * N;
            m.ring = c.conv + ((size_t)mi * c.n_slots + slot) * W * Cx;
            m.act = b.act_big; m.act_ld = b.ld_big;
            m.status = c.status;
            // the GEMM's GE_ROWSCALE outputs are the bf16 in_proj values (the decode path's zx)
            if ((e = gemm(GE_ROWSCALE, b.act_d, b.ld_d, T, Lw.in_proj, b.inv, b.zx, zxw, nullptr, 0))) return e;
            m.zx = b.zx;
            if (c.tap_zx && (e = cudaMemcpyAsync(c.tap_zx + (size_t)mi * T * zxw, b.zx, (size_t)T * zxw * 2,
                                                 cudaMemcpyDeviceToDevice, s)))
                return e;
            if ((e = prefill_mixer(m, s))) return e;
            if ((e = gemm(GE_RESID, b.act_big, b.ld_big, T, Lw.out_proj, nullptr, nullptr, 0, b.r, d))) return e;
            mi++;
        } else if (kind == '*') {
            const size_t kvl = ((size_t)ai * c.n_slots + slot) * c.Hk * c.cap * c.Dh;
            GemmArgs qa{};
            qa.Hq = c.Hq; qa.Hk = c.Hk; qa.Dh = c.Dh; qa.cap = c.cap; qa.t0 = 0;
            qa.kcache = c.k + kvl; qa.vcache = c.v + kvl;
            if ((e = gemm(GE_QKV, b.act_d, b.ld_d, T, Lw.qkv, b.inv, b.q, c.Hq * c.Dh, nullptr, 0, &qa))) return e;
            if (c.Dh == 128)
                pf_flash_kernel<128><<<dim3((T + 63) / 64, c.Hq), 128, 0, s>>>(b.q, qa.kcache, qa.vcache, T, c.Hq, c.Hk,
                                                                               c.cap, b.act_big, b.ld_big, f16);
            else if (c.Dh == 64)
                pf_flash_kernel<64><<<dim3((T + 63) / 64, c.Hq), 128, 0, s>>>(b.q, qa.kcache, qa.vcache, T, c.Hq, c.Hk,
                                                                              c.cap, b.act_big, b.ld_big, f16);
            else
                pf_attn_scalar_kernel<<<dim3((T + 7) / 8, c.Hq), 256, 0, s>>>(b.q, qa.kcache, qa.vcache, T, c.Hq, c.Hk,
                                                                              c.Dh, c.cap, b.act_big, b.ld_big, f16);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
            if ((e = gemm(GE_RESID, b.act_big, b.ld_big, T, Lw.o, nullptr, nullptr, 0, b.r, d))) return e;
            ai++;
        } else {
            if ((e = gemm(GE_RELU2, b.act_d, b.ld_d, T, Lw.up, b.inv, b.act_big, b.ld_big, nullptr, 0))) return e;
            if ((e = gemm(GE_RESID, b.act_big, b.ld_big, T, Lw.down, nullptr, nullptr, 0, b.r, d))) return e;
        }
        if (c.tap && (e = cudaMemcpyAsync(c.tap + (size_t)(l + 1) * T * d, b.r, rbytes, cudaMemcpyDeviceToDevice, s)))
            return e;
    }
    pf_finish_kernel<<<1, 1, 0, s>>>(c.ctx_len, slot, T);
    return cudaGetLastError();
}

}  // namespace vc
