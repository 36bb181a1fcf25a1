// prefill_mma.cuh -- the chunk contractions of the prefill on warp-level tensor-core MMA
// (mma.sync m16n8k16, 16-bit operands, fp32 accumulation): the chunked SSD outputs and causal
// flash attention.  Together they are ~2.5% of the prefill's FLOPs (the projections, on tcgen05,
// are the rest), on tiles whose head dimensions (P = 80, Dh = 128) are small, so register-fragment
// MMA with shared-memory staging keeps them off the critical path without a TMEM pipeline.
//
// Fragment layouts of m16n8k16 (g = lane / 4, t = lane % 4):
//   A 16x16 row-major: a0 = A[g][2t..2t+1], a1 = A[g+8][2t..], a2 = A[g][2t+8..], a3 = A[g+8][2t+8..]
//   B 16x8  (k x n):   b0 = B[2t..2t+1][g], b1 = B[2t+8..2t+9][g]
//   C 16x8:            c0 = C[g][2t], c1 = C[g][2t+1], c2 = C[g+8][2t], c3 = C[g+8][2t+1]
// Shared-memory rows are padded so the 8 rows a fragment load touches fall in distinct banks.
#pragma once
#include "common.cuh"

namespace vc {

VC_DEV uint32_t lds32(const uint16_t* p) { return *reinterpret_cast<const uint32_t*>(p); }

VC_DEV uint16_t bf16_bits(float v) {
    __nv_bfloat16 b = __float2bfloat16_rn(v);
    return *reinterpret_cast<uint16_t*>(&b);
}

VC_DEV uint32_t pack_bf16x2(float lo, float hi) { return (uint32_t)bf16_bits(lo) | ((uint32_t)bf16_bits(hi) << 16); }

VC_DEV void ldsm_x4_trans(uint32_t (&r)[4], const uint16_t* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}

// fp16 bits, saturated to the finite range
VC_DEV uint16_t f16_bits(float v) {
    __half h = __float2half_rn(fminf(fmaxf(v, -65504.0f), 65504.0f));
    return *reinterpret_cast<uint16_t*>(&h);
}

// ------------------------------------------------------------------------------------------
// chunked SSD, outputs.  CTA = (chunk c, B/C group g, 64-row tile of the chunk), two CTAs per
// SM.  The group's C.B^T block (64 x j) is formed once (fragments read straight from the fp16
// image of the conv outputs, which the chunk's CTAs share through L2) and kept in shared memory
// as fp16; the H/G heads of the group then reuse it:
//   y_i[p] = sum_{j<=i} (C_i.B_j) exp(Lam_i - Lam_j) dt_j x_j[p]      (intra-chunk, W . X)
//          + exp(Lam_i) sum_n C_i[n] S_in[p][n]                        (state entering the chunk)
//          + D x_i[p]
// The decay-weighted W fragments are built in registers from the fp16 C.B^T, so only x is
// staged per head.  The intra-chunk products take fp16 operands (C, B, W and x: 11-bit
// significands; y is heavy-tailed, and bf16's 8 bits leave its largest elements ~10% of the
// RMS off), the entering-state product bf16 operands (the state's range).
// ------------------------------------------------------------------------------------------
static constexpr int kSsdChunk = 256;
static constexpr int kSsdTi = 64;

VC_DEV uint32_t pack_f16x2(float lo, float hi) { return (uint32_t)f16_bits(lo) | ((uint32_t)f16_bits(hi) << 16); }

struct SsdLayout {
    int scb, sx, sc;             // row strides (elements): C.B^T fp16 [64][scb], x fp16 [j][sx], C bf16 [64][sc]
    size_t off_cb, off_x, off_c, off_l, total;
};

__host__ __device__ inline SsdLayout ssd_layout(int N, int P) {
    (void)N;
    SsdLayout L{};
    L.scb = kSsdChunk + 8;
    L.sx = P + 8;
    L.sc = N + 8;
    auto a16 = [](size_t v) { return (v + 15) / 16 * 16; };
    L.off_cb = 0;
    L.off_x = a16((size_t)kSsdTi * L.scb * 2);
    L.off_c = L.off_x + a16((size_t)kSsdChunk * L.sx * 2);
    L.off_l = L.off_c + a16((size_t)kSsdTi * L.sc * 2);
    L.total = L.off_l + 2 * kSsdChunk * 4;
    return L;
}

__global__ void __launch_bounds__(256, 2) pf_ssd_out_mma_kernel(const float* __restrict__ xc,
                                                                const uint16_t* __restrict__ xc16,
                                                                const float* __restrict__ dt,
                                                                const float* __restrict__ lam,
                                                                const uint16_t* __restrict__ sin16,
                                                                const float* __restrict__ Dv, int T, int H, int P,
                                                                int N, int G, int E, int Cx, float* __restrict__ y) {
    extern __shared__ __align__(16) unsigned char smraw[];
    const int c = blockIdx.x, g = blockIdx.y, it = blockIdx.z;
    const int t0 = c * kSsdChunk, len = min(kSsdChunk, T - t0);
    const int i0 = it * kSsdTi;
    if (i0 >= len) return;
    const int i1 = min(len, i0 + kSsdTi);
    const int jn = i1;                       // frames j < jn are visible to some row of the tile
    const int jn16 = (jn + 15) & ~15;
    const SsdLayout L = ssd_layout(N, P);
    uint16_t* CB = reinterpret_cast<uint16_t*>(smraw + L.off_cb);    // C_i.B_j, fp16 [64][scb]
    uint16_t* Xs = reinterpret_cast<uint16_t*>(smraw + L.off_x);     // x rows of the head, fp16 [j][p]
    uint16_t* Cb = reinterpret_cast<uint16_t*>(smraw + L.off_c);     // C rows of the tile, bf16 [64][sc]
    float* lam_s = reinterpret_cast<float*>(smraw + L.off_l);
    float* dts = lam_s + kSsdChunk;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gq = lane >> 2, tq = lane & 3;
    const uint16_t* C16 = xc16 + (size_t)t0 * Cx + E + (size_t)G * N + (size_t)g * N;
    const uint16_t* B16 = xc16 + (size_t)t0 * Cx + E + (size_t)g * N;
    const float* C32 = xc + (size_t)t0 * Cx + E + (size_t)G * N + (size_t)g * N;
    const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
    auto ldg32 = [](const uint16_t* p) { return __ldg(reinterpret_cast<const unsigned int*>(p)); };

    // 0. the tile's C rows as bf16, for the entering-state product of every head
    for (int idx = tid; idx < kSsdTi * (N / 4); idx += blockDim.x) {
        const int ii = idx / (N / 4), q = idx - ii * (N / 4);
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i0 + ii < i1) v = __ldg(reinterpret_cast<const float4*>(C32 + (size_t)(i0 + ii) * Cx + 4 * q));
        *reinterpret_cast<uint2*>(Cb + ii * L.sc + 4 * q) = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
    }
    // 1. CB[ii][j] = C_i . B_j: warp w forms columns 32w .. 32w+31 of all 64 rows
    if (32 * warp < jn) {
        float acc[4][4][4];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[a][b][e] = 0.0f;
        for (int k0 = 0; k0 < N; k0 += 16) {
            uint32_t af[4][4];
#pragma unroll
            for (int mt = 0; mt < 4; ++mt) {
                const int ra = i0 + mt * 16 + gq, rb = ra + 8;
                const uint16_t* pa = C16 + (size_t)ra * Cx + k0 + 2 * tq;
                const uint16_t* pb = C16 + (size_t)rb * Cx + k0 + 2 * tq;
                af[mt][0] = ra < i1 ? ldg32(pa) : 0u;
                af[mt][1] = rb < i1 ? ldg32(pb) : 0u;
                af[mt][2] = ra < i1 ? ldg32(pa + 8) : 0u;
                af[mt][3] = rb < i1 ? ldg32(pb + 8) : 0u;
            }
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const int j = 32 * warp + nt * 8 + gq;
                const uint16_t* pbj = B16 + (size_t)j * Cx + k0 + 2 * tq;
                const uint32_t b0 = j < jn ? ldg32(pbj) : 0u, b1 = j < jn ? ldg32(pbj + 8) : 0u;
#pragma unroll
                for (int mt = 0; mt < 4; ++mt) mma_f16(acc[mt][nt], af[mt], b0, b1);
            }
        }
#pragma unroll
        for (int mt = 0; mt < 4; ++mt)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                uint16_t* r = CB + (mt * 16 + gq) * L.scb + 32 * warp + nt * 8 + 2 * tq;
                *reinterpret_cast<uint32_t*>(r) = pack_f16x2(acc[mt][nt][0], acc[mt][nt][1]);
                *reinterpret_cast<uint32_t*>(r + 8 * L.scb) = pack_f16x2(acc[mt][nt][2], acc[mt][nt][3]);
            }
    }

    // 2. the heads of the group
    const int hpg = H / G;
    const int nt8 = P / 8;
    const int wm = warp & 3, wn = warp >> 2;
    const int half = (nt8 + 1) / 2;
    const int q0 = wn * half;
    const int qn = min(nt8, q0 + half) - q0;
    const int kend = min(jn16, i0 + wm * 16 + 16);   // rows of this warp see j < i0 + 16 (wm + 1)
    const int lk = (lane & 7) + 8 * ((lane >> 3) & 1);
    const int lp = 8 * (lane >> 4);
    const int p8 = P / 8;
    const int ia = wm * 16 + gq, ib = ia + 8;          // the lane's two rows within the tile
    for (int hh = 0; hh < hpg; ++hh) {
        const int h = g * hpg + hh;
        __syncthreads();   // C.B^T ready (first head) / previous head's x consumed
        for (int j = tid; j < jn16; j += blockDim.x) {
            lam_s[j] = j < jn ? lam[(size_t)(t0 + j) * H + h] : 0.0f;
            dts[j] = j < jn ? dt[(size_t)(t0 + j) * H + h] : 0.0f;
        }
        const uint16_t* xh16 = xc16 + (size_t)t0 * Cx + (size_t)h * P;
#pragma unroll 4
        for (int idx = tid; idx < jn16 * p8; idx += blockDim.x) {
            const int j = idx / p8, c8 = idx - j * p8;
            *reinterpret_cast<uint4*>(Xs + j * L.sx + c8 * 8) =
                j < jn ? *reinterpret_cast<const uint4*>(xh16 + (size_t)j * Cx + c8 * 8) : z4;
        }
        __syncthreads();
        const float la = lam_s[min(i0 + ia, jn - 1)], lb = lam_s[min(i0 + ib, jn - 1)];
        float acc[8][4], acc2[8][4];
#pragma unroll
        for (int q = 0; q < 8; ++q)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[q][e] = acc2[q][e] = 0.0f;
        for (int k0 = 0; k0 < kend; k0 += 16) {
            // W fragments: W[i][j] = CB[i][j] exp(Lam_i - Lam_j) dt_j for j <= i < i1, else 0
            uint32_t af[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int ii = (e & 1) ? ib : ia;
                const int j = k0 + 2 * tq + 8 * (e >> 1);
                const float li = (e & 1) ? lb : la;
                const __half2 cb = *reinterpret_cast<const __half2*>(CB + ii * L.scb + j);
                const float2 lj = *reinterpret_cast<const float2*>(lam_s + j);
                const float2 dj = *reinterpret_cast<const float2*>(dts + j);
                const int i = i0 + ii;
                const float w0 = (i < i1 && j <= i) ? __low2float(cb) * __expf(li - lj.x) * dj.x : 0.0f;
                const float w1 = (i < i1 && j + 1 <= i) ? __high2float(cb) * __expf(li - lj.y) * dj.y : 0.0f;
                af[e] = pack_f16x2(w0, w1);
            }
#pragma unroll
            for (int q = 0; q < 8; q += 2)
                if (q < qn) {
                    uint32_t xb[4];
                    ldsm_x4_trans(xb, Xs + (k0 + lk) * L.sx + (q0 + q) * 8 + lp);
                    mma_f16(acc[q], af, xb[0], xb[1]);
                    if (q + 1 < qn) mma_f16(acc[q + 1], af, xb[2], xb[3]);
                }
        }
        // C . S_in^T: C rows (bf16, staged once), S_in rows p (bf16) from L2
        const uint16_t* Sh = sin16 + ((size_t)c * H + h) * P * N;
        for (int k0 = 0; k0 < N; k0 += 16) {
            uint32_t af[4];
            const uint16_t* r = Cb + ia * L.sc + k0 + 2 * tq;
            af[0] = lds32(r);
            af[1] = lds32(r + 8 * L.sc);
            af[2] = lds32(r + 8);
            af[3] = lds32(r + 8 * L.sc + 8);
#pragma unroll
            for (int q = 0; q < 8; ++q)
                if (q < qn) {
                    const uint16_t* br = Sh + (size_t)((q0 + q) * 8 + gq) * N + k0 + 2 * tq;
                    mma_bf16(acc2[q], af, ldg32(br), ldg32(br + 8));
                }
        }
        const float Dh_ = Dv[h];
        const float* xh = xc + (size_t)t0 * Cx + (size_t)h * P;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int i = i0 + (r ? ib : ia);
            if (i < i1) {
                const float el = __expf(lam_s[i]);
                const float* xi = xh + (size_t)i * Cx;
                float* yi = y + (size_t)(t0 + i) * E + (size_t)h * P;
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    if (q < qn) {
                        const int p = (q0 + q) * 8 + 2 * tq;
                        const float2 xv = *reinterpret_cast<const float2*>(xi + p);
                        float2 o;
                        o.x = acc[q][2 * r] + el * acc2[q][2 * r] + Dh_ * xv.x;
                        o.y = acc[q][2 * r + 1] + el * acc2[q][2 * r + 1] + Dh_ * xv.y;
                        *reinterpret_cast<float2*>(yi + p) = o;
                    }
            }
        }
    }
}

// ------------------------------------------------------------------------------------------
// chunked SSD, chunk states on tensor cores:  S_c[p][n] = sum_j (w_j x_j[p]) B_j[n],
// w_j = exp(Lam_end - Lam_j) dt_j.  The state decode continues from must meet the fp32 bound, so
// each operand is split into two fp16 halves (v = hi + lo, lo = v - hi) and the product is
// hi.hi + hi.lo + lo.hi (the dropped lo.lo term is ~2^-22 of the product), accumulated in fp32.
// CTA = (chunk, head); frames staged 64 at a time; warp w owns state columns 16 w .. 16 w + 15
// (two n8 tiles) for all P rows (MT m16 tiles).  Both operands are loaded with transposing
// 8x8 matrix loads from their natural [frame][channel] rows.
// ------------------------------------------------------------------------------------------
static constexpr int kStTile = 64;

struct StateLayout {
    int sx, sb;
    size_t off_xh, off_xl, off_bh, off_bl, off_w, off_ld, total;
};

__host__ __device__ inline StateLayout state_layout(int N, int P) {
    StateLayout L{};
    L.sx = P + 8;
    L.sb = N + 8;
    auto a16 = [](size_t v) { return (v + 15) / 16 * 16; };
    const size_t rx = a16((size_t)kStTile * L.sx * 2), rb = a16((size_t)kStTile * L.sb * 2);
    L.off_xh = 0;
    L.off_xl = rx;
    L.off_bh = 2 * rx;
    L.off_bl = 2 * rx + rb;
    L.off_w = 2 * rx + 2 * rb;
    L.off_ld = a16(L.off_w + 2 * kSsdChunk * 4);
    L.total = L.off_ld + kSsdChunk * 8;
    return L;
}

VC_DEV void split_f16(float v, uint16_t& hi, uint16_t& lo) {
    hi = f16_bits(v);
    const __half h = *reinterpret_cast<const __half*>(&hi);
    lo = f16_bits(v - __half2float(h));
}

template <int MT>
__global__ void __launch_bounds__(256) pf_ssd_state_mma_kernel(const float* __restrict__ xc, const float* __restrict__ dt,
                                                               const float* __restrict__ A_log, int T, int H, int P,
                                                               int N, int G, int E, int Cx, float* __restrict__ lam,
                                                               float* __restrict__ schunk) {
    extern __shared__ __align__(16) unsigned char smraw[];
    const int c = blockIdx.x, h = blockIdx.y;
    const int t0 = c * kSsdChunk, len = min(kSsdChunk, T - t0);
    const int g = (int)((long long)h * G / H);
    const StateLayout L = state_layout(N, P);
    uint16_t* Xh = reinterpret_cast<uint16_t*>(smraw + L.off_xh);
    uint16_t* Xl = reinterpret_cast<uint16_t*>(smraw + L.off_xl);
    uint16_t* Bh = reinterpret_cast<uint16_t*>(smraw + L.off_bh);
    uint16_t* Bl = reinterpret_cast<uint16_t*>(smraw + L.off_bl);
    float* lam_s = reinterpret_cast<float*>(smraw + L.off_w);
    float* w = lam_s + kSsdChunk;
    double* lamd = reinterpret_cast<double*>(smraw + L.off_ld);   // the same sums, unrounded
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gq = lane >> 2, tq = lane & 3;
    const float A = -expf(A_log[h]);
    // inclusive scan of A*dt over the chunk (one warp), summed in double: over 256 frames the
    // cumulative log decay of a fast head reaches ~100, where fp32 partial sums would carry ~1e-4
    // of absolute error into every decay factor exp(Lam_i - Lam_j); each Lam is rounded once
    if (warp == 0) {
        double run = 0.0;
        for (int base = 0; base < len; base += 32) {
            const int i = base + lane;
            double v = i < len ? (double)(A * dt[(size_t)(t0 + i) * H + h]) : 0.0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const double u = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += u;
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
    // the state weights from differences of the unrounded sums: in fp32, two sums of magnitude
    // ~200 would leave ~1e-5 of absolute error in the small differences that matter most
    const double lend = lamd[len - 1];
    for (int i = tid; i < len; i += blockDim.x) {
        w[i] = expf((float)(lend - lamd[i])) * dt[(size_t)(t0 + i) * H + h];
        lam[(size_t)(t0 + i) * H + h] = lam_s[i];
    }
    const int npairs = N / 16;   // pairs of n8 tiles
    float acc[MT][2][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[mt][q][e] = 0.0f;
    const float* xh = xc + (size_t)t0 * Cx + (size_t)h * P;
    const float* bg = xc + (size_t)t0 * Cx + E + (size_t)g * N;
    const int P4 = P / 4, N4 = N / 4;
    // A fragments (rows p, k = frame) from Xw[j][p]: lanes 0-7 frames 0-7 at p0, 8-15 frames 0-7 at
    // p0 + 8, 16-23 frames 8-15 at p0, 24-31 frames 8-15 at p0 + 8
    const int ar = (lane & 7) + 8 * (lane >> 4), ac = 8 * ((lane >> 3) & 1);
    // B fragments (k = frame, n) from B[j][n]: lanes 0-7 frames 0-7, 8-15 frames 8-15 (n0),
    // 16-31 the same frames at n0 + 8
    const int br = (lane & 7) + 8 * ((lane >> 3) & 1), bc = 8 * (lane >> 4);
    for (int jb = 0; jb < len; jb += kStTile) {
        const int nj = min(kStTile, len - jb);
        const int nj16 = (nj + 15) & ~15;
        __syncthreads();   // w ready (first tile) / previous tile consumed
        for (int idx = tid; idx < nj16 * P4; idx += blockDim.x) {
            const int j = idx / P4, q = idx - j * P4;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (j < nj) {
                v = *reinterpret_cast<const float4*>(xh + (size_t)(jb + j) * Cx + 4 * q);
                const float wj = w[jb + j];
                v.x *= wj; v.y *= wj; v.z *= wj; v.w *= wj;
            }
            uint16_t hh[4], ll[4];
            split_f16(v.x, hh[0], ll[0]); split_f16(v.y, hh[1], ll[1]);
            split_f16(v.z, hh[2], ll[2]); split_f16(v.w, hh[3], ll[3]);
            *reinterpret_cast<uint2*>(Xh + j * L.sx + 4 * q) =
                make_uint2(hh[0] | ((uint32_t)hh[1] << 16), hh[2] | ((uint32_t)hh[3] << 16));
            *reinterpret_cast<uint2*>(Xl + j * L.sx + 4 * q) =
                make_uint2(ll[0] | ((uint32_t)ll[1] << 16), ll[2] | ((uint32_t)ll[3] << 16));
        }
        for (int idx = tid; idx < nj16 * N4; idx += blockDim.x) {
            const int j = idx / N4, q = idx - j * N4;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (j < nj) v = *reinterpret_cast<const float4*>(bg + (size_t)(jb + j) * Cx + 4 * q);
            uint16_t hh[4], ll[4];
            split_f16(v.x, hh[0], ll[0]); split_f16(v.y, hh[1], ll[1]);
            split_f16(v.z, hh[2], ll[2]); split_f16(v.w, hh[3], ll[3]);
            *reinterpret_cast<uint2*>(Bh + j * L.sb + 4 * q) =
                make_uint2(hh[0] | ((uint32_t)hh[1] << 16), hh[2] | ((uint32_t)hh[3] << 16));
            *reinterpret_cast<uint2*>(Bl + j * L.sb + 4 * q) =
                make_uint2(ll[0] | ((uint32_t)ll[1] << 16), ll[2] | ((uint32_t)ll[3] << 16));
        }
        __syncthreads();
        if (warp < npairs) {
            const int pr = warp;
            for (int k0 = 0; k0 < nj16; k0 += 16) {
                uint32_t bh[4], bl[4];
                ldsm_x4_trans(bh, Bh + (k0 + br) * L.sb + 16 * pr + bc);
                ldsm_x4_trans(bl, Bl + (k0 + br) * L.sb + 16 * pr + bc);
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    uint32_t ah[4], al[4];
                    ldsm_x4_trans(ah, Xh + (k0 + ar) * L.sx + 16 * mt + ac);
                    ldsm_x4_trans(al, Xl + (k0 + ar) * L.sx + 16 * mt + ac);
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        mma_f16(acc[mt][q], ah, bh[2 * q], bh[2 * q + 1]);
                        mma_f16(acc[mt][q], ah, bl[2 * q], bl[2 * q + 1]);
                        mma_f16(acc[mt][q], al, bh[2 * q], bh[2 * q + 1]);
                    }
                }
            }
        }
    }
    // write the chunk state (each warp its column pair; N <= 128, so every pair has one owner)
    if (warp < npairs) {
        float* S = schunk + ((size_t)c * H + h) * P * N;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int n = 16 * warp + 8 * q + 2 * tq;
                const int p = 16 * mt + gq;
                *reinterpret_cast<float2*>(S + (size_t)p * N + n) = make_float2(acc[mt][q][0], acc[mt][q][1]);
                *reinterpret_cast<float2*>(S + (size_t)(p + 8) * N + n) = make_float2(acc[mt][q][2], acc[mt][q][3]);
            }
    }
}

// ------------------------------------------------------------------------------------------
// causal GQA attention (flash form): CTA = (64 query frames, q head), 4 warps of 16 rows; keys
// and values in tiles of 64 frames from the KV cache rows the qkv projection just wrote; online
// softmax in fp32 (exp2 with the 1/sqrt(Dh) scale folded in), P rounded to bf16 for P.V.
// q head i reads KV head floor(i Hk / Hq); no positional encoding.
// ------------------------------------------------------------------------------------------

template <int DH>
__global__ void __launch_bounds__(128) pf_flash_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ kc,
                                                       const uint16_t* __restrict__ vc, int T, int Hq, int Hk, int cap,
                                                       uint16_t* __restrict__ out, int ld, int f16) {
    constexpr int SK = DH + 8;
    __shared__ __align__(16) uint16_t Ks[64 * SK];
    __shared__ __align__(16) uint16_t Vs[64 * SK];
    const int nqt = (T + 63) / 64;
    const int qt = nqt - 1 - (int)blockIdx.x;   // the longest rows first
    const int hq = blockIdx.y;
    const int hk = (int)((long long)hq * Hk / Hq);
    const int r0 = qt * 64;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gq = lane >> 2, tq = lane & 3;
    const uint16_t* K = kc + (size_t)hk * cap * DH;
    const uint16_t* V = vc + (size_t)hk * cap * DH;
    const int qld = Hq * DH;

    uint32_t qa[DH / 16][4];
    {
        const int ra = r0 + warp * 16 + gq, rb = ra + 8;
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
            const int col = hq * DH + kk * 16 + 2 * tq;
            qa[kk][0] = ra < T ? lds32(q + (size_t)ra * qld + col) : 0u;
            qa[kk][1] = rb < T ? lds32(q + (size_t)rb * qld + col) : 0u;
            qa[kk][2] = ra < T ? lds32(q + (size_t)ra * qld + col + 8) : 0u;
            qa[kk][3] = rb < T ? lds32(q + (size_t)rb * qld + col + 8) : 0u;
        }
    }
    float o[DH / 8][4];
#pragma unroll
    for (int d = 0; d < DH / 8; ++d)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[d][e] = 0.0f;
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.0f, 0.0f};
    const float sl2 = rsqrtf((float)DH) * 1.4426950408889634f;
    const int row[2] = {r0 + warp * 16 + gq, r0 + warp * 16 + gq + 8};

    for (int kt = 0; kt <= qt; ++kt) {
        const int key0 = kt * 64;
        __syncthreads();
        for (int idx = tid; idx < 64 * DH / 8; idx += blockDim.x) {
            const int key = idx / (DH / 8), c8 = idx - key * (DH / 8);
            uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
            if (key0 + key < T) {
                kv = *reinterpret_cast<const uint4*>(K + (size_t)(key0 + key) * DH + c8 * 8);
                vv = *reinterpret_cast<const uint4*>(V + (size_t)(key0 + key) * DH + c8 * 8);
            }
            *reinterpret_cast<uint4*>(Ks + key * SK + c8 * 8) = kv;
            *reinterpret_cast<uint4*>(Vs + key * SK + c8 * 8) = vv;
        }
        __syncthreads();
        float s[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[nt][e] = 0.0f;
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk)
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                const uint16_t* br = Ks + (nt * 8 + gq) * SK + kk * 16 + 2 * tq;
                mma_bf16(s[nt], qa[kk], lds32(br), lds32(br + 8));
            }
        // causal mask (keys beyond the row or beyond T) and the running max of each row
        const bool diag = kt == qt;
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int key = key0 + nt * 8 + 2 * tq + (e & 1);
                const int r = e >> 1;
                if ((diag && key > row[r]) || key >= T) s[nt][e] = -INFINITY;
                mx[r] = fmaxf(mx[r], s[nt][e]);
            }
        float corr[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
            mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
            const float mn = fmaxf(m[r], mx[r]);
            corr[r] = m[r] == -INFINITY ? 0.0f : exp2f((m[r] - mn) * sl2);
            m[r] = mn;
        }
        float ls[2] = {0.0f, 0.0f};
        uint32_t pa[4][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            float p[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = e >> 1;
                p[e] = s[nt][e] == -INFINITY ? 0.0f : exp2f((s[nt][e] - m[r]) * sl2);
                ls[r] += p[e];
            }
            // C fragment of key tile nt -> A fragment (keys 16 kb .. 16 kb + 15) of P . V
            const int kb = nt >> 1;
            if ((nt & 1) == 0) {
                pa[kb][0] = pack_bf16x2(p[0], p[1]);
                pa[kb][1] = pack_bf16x2(p[2], p[3]);
            } else {
                pa[kb][2] = pack_bf16x2(p[0], p[1]);
                pa[kb][3] = pack_bf16x2(p[2], p[3]);
            }
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) l[r] = l[r] * corr[r] + ls[r];
#pragma unroll
        for (int d = 0; d < DH / 8; ++d) {
            o[d][0] *= corr[0];
            o[d][1] *= corr[0];
            o[d][2] *= corr[1];
            o[d][3] *= corr[1];
        }
        // O += P . V; V fragments by transposing 8x8 loads: lanes 0-7 keys 0-7, 8-15 keys 8-15
        // (dims d0..d0+7), 16-23 and 24-31 the same keys at dims d0+8..d0+15
        const int lk = (lane & 7) + 8 * ((lane >> 3) & 1);
        const int ld8 = 8 * (lane >> 4);
#pragma unroll
        for (int kb = 0; kb < 4; ++kb)
#pragma unroll
            for (int d = 0; d < DH / 8; d += 2) {
                uint32_t vb[4];
                ldsm_x4_trans(vb, Vs + (kb * 16 + lk) * SK + d * 8 + ld8);
                mma_bf16(o[d], pa[kb], vb[0], vb[1]);
                mma_bf16(o[d + 1], pa[kb], vb[2], vb[3]);
            }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        l[r] += __shfl_xor_sync(0xffffffffu, l[r], 1);
        l[r] += __shfl_xor_sync(0xffffffffu, l[r], 2);
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        if (row[r] >= T) continue;
        const float inv = 1.0f / l[r];
        uint16_t* orow = out + (size_t)row[r] * ld + (size_t)hq * DH;
#pragma unroll
        for (int d = 0; d < DH / 8; ++d) {
            const float u0 = o[d][2 * r] * inv, u1 = o[d][2 * r + 1] * inv;
            const uint32_t w = f16 ? ((uint32_t)act_bits<true>(u0) | ((uint32_t)act_bits<true>(u1) << 16))
                                   : ((uint32_t)act_bits<false>(u0) | ((uint32_t)act_bits<false>(u1) << 16));
            *reinterpret_cast<uint32_t*>(orow + d * 8 + 2 * tq) = w;
        }
    }
}

}  // namespace vc
