// ssd_tc.cu -- the chunked SSD of the prefill on tcgen05 tensor cores: chunk outputs and chunk
// states (the scan over chunks between them is elementwise, prefill.cu).
//
// Dao & Gu, "Transformers are SSMs", the SSD algorithm: within a chunk of Q = 256 frames the
// output of head h is a masked, decay-weighted attention-like product plus the contribution of
// the state entering the chunk,
//   y_i = sum_{j<=i} (C_i . B_j) exp(Lam_i - Lam_j) dt_j x_j  +  exp(Lam_i) C_i . S_in  +  D x_i,
// with Lam the within-chunk cumulative log decay (A dt summed).  Written as matrices per chunk,
// row tile of 128 frames and B/C group g (whose H/G heads share B and C):
//   G   = C B^T                      [128 x jn]  over the state dimension (once per tile)
//   M_h = G o L_h                    [128 x jn]  L_h[i][j] = exp(Lam_i - Lam_j) dt_j (j <= i), else 0
//   Y_h = M_h X_h + diag(exp Lam) C S_in,h^T  (+ D x)
// where jn = 128 for the first row half of the chunk and 256 for the second.  Each is a dense
// contraction, so each runs on tcgen05.mma with the accumulator in tensor memory:
//   * TMA brings C and B of the group (fp16 image of the conv outputs, 128-byte swizzle) and,
//     per head, x (the B operand of M X, MN-major with 32-byte swizzle) and S_in (bf16);
//   * one thread issues G = C B^T into TMEM columns [0, jn);
//   * per head, the 256 threads read G back (each thread one row = one TMEM lane, warps w and
//     w + 4 share a lane quarter and split the columns), apply the decay mask with one ex2 per
//     element, and write M_h as fp16 into shared memory in the K-major swizzled layout; one
//     thread then issues M_h X_h (fp16) into columns [256, 256 + P) and C S_in^T (bf16) into
//     [384, 384 + P); the threads read both back, add exp(Lam_i) x the second and D x_i, store y;
//     the next head's x and S_in are copied while its M_h is formed.
// The C rows are converted to bf16 in place once G is done (the entering-state product keeps
// bf16 operands: the state's range).  Every wait is bounded; a timeout sets the status word,
// the CTA waits (bounded) for its copies in flight and frees its TMEM.
#include "common.cuh"
#include "prefill.cuh"
#include "tc.cuh"

namespace vc {

static constexpr int kQ = 256;          // chunk length (frames)
static constexpr int kRows = 128;       // frames of one CTA's output tile (TMEM lanes)
static constexpr int kOutThreads = 256;
static constexpr uint32_t kTmemCols = 512;
static constexpr uint32_t kColY1 = 256, kColY2 = 384;

// shared-memory plan of the output kernel (byte offsets from a 1024-aligned base)
struct SsdOutPlan {
    int NA, PA;                                 // 64-wide atoms of N, 16-wide blocks of P
    uint32_t off_c, off_bm, off_x, off_s, total;
};

__host__ __device__ inline SsdOutPlan ssd_out_plan(int N, int P) {
    SsdOutPlan L{};
    L.NA = N / 64;
    L.PA = P / 16;
    L.off_c = 0;                                               // C rows: NA atoms x 128 rows x 128 B
    const uint32_t bm = (uint32_t)L.NA * 32768u > 65536u ? (uint32_t)L.NA * 32768u : 65536u;
    L.off_bm = L.off_c + (uint32_t)L.NA * 16384u;              // B rows (NA x 256 x 128 B), later M_h (4 x 128 x 128 B)
    L.off_x = L.off_bm + bm;                                   // x_h: PA blocks x 256 rows x 32 B
    L.off_s = L.off_x + (uint32_t)L.PA * 8192u;                // S_in,h: NA atoms x P rows x 128 B
    L.total = L.off_s + (uint32_t)L.NA * (uint32_t)P * 128u;
    return L;
}

VC_DEV float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

VC_DEV uint32_t pack_f16x2_sat(float lo, float hi) {
    lo = fminf(fmaxf(lo, -65504.0f), 65504.0f);
    hi = fminf(fmaxf(hi, -65504.0f), 65504.0f);
    return h2_as_u32(__floats2half2_rn(lo, hi));
}

VC_DEV uint32_t f16x2_to_bf16x2(uint32_t v) {
    const __half2 h = u32_as_h2(v);
    const __nv_bfloat162 b = __floats2bfloat162_rn(__low2float(h), __high2float(h));
    return *reinterpret_cast<const uint32_t*>(&b);
}

struct SsdOutArgs {
    const float* dt;    // [T][H]
    const float* lam;   // [T][H] within-chunk cumulative A dt
    const float* Dv;    // [H]
    float* y;           // [T][E]
    int T, H, P, N, G, E;
    int* status;
};

__global__ void __launch_bounds__(kOutThreads, 1)
    pf_ssd_out_tc_kernel(const __grid_constant__ CUtensorMap mC, const __grid_constant__ CUtensorMap mB,
                         const __grid_constant__ CUtensorMap mX, const __grid_constant__ CUtensorMap mS,
                         const SsdOutArgs a) {
    extern __shared__ uint8_t smraw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t bar_cb, bar_g, bar_x, bar_y;
    __shared__ uint32_t tmem_base;
    __shared__ float lam2[kQ], dts[kQ];

    const int H = a.H, P = a.P, N = a.N, G = a.G;
    const int nch = (a.T + kQ - 1) / kQ;
    int bid = blockIdx.x;
    const int it = bid < nch * G ? 1 : 0;   // the second (longer) row halves first
    bid -= it ? 0 : nch * G;
    const int c = bid / G, g = bid - c * G;
    const int t0 = c * kQ, len = min(kQ, a.T - t0);
    const int i0 = it * kRows;
    if (i0 >= len) return;
    const int jn = it ? 2 * kRows : kRows;   // frames j < jn of the chunk reach the tile's rows
    const SsdOutPlan L = ssd_out_plan(N, P);
    uint8_t* sC = sm + L.off_c;
    uint8_t* sBM = sm + L.off_bm;
    uint8_t* sX = sm + L.off_x;
    uint8_t* sS = sm + L.off_s;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int hpg = H / G, nkN = N / 16;

    if (tid == 0) {
        mbar_init(&bar_cb, 1);
        mbar_init(&bar_g, 1);
        mbar_init(&bar_x, 1);
        mbar_init(&bar_y, 1);
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(&tmem_base, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;

    bool cb_pending = false, x_pending = false;   // copies in flight (thread 0)
    uint32_t x_phase = 0;
    auto issue_xs = [&](int h, uint32_t phase) {
        mbar_arrive_expect_tx(&bar_x, (uint32_t)L.PA * 8192u + (uint32_t)L.NA * (uint32_t)P * 128u);
        for (int q = 0; q < L.PA; ++q) tma_load_2d(sX + q * 8192, &mX, h * P + 16 * q, t0, &bar_x);
        for (int q = 0; q < L.NA; ++q) tma_load_2d(sS + q * P * 128, &mS, 64 * q, (c * H + h) * P, &bar_x);
        x_pending = true;
        x_phase = phase;
    };
    if (tid == 0) {
        mbar_arrive_expect_tx(&bar_cb, (uint32_t)L.NA * (16384u + 32768u));
        for (int q = 0; q < L.NA; ++q) {
            tma_load_2d(sC + q * 16384, &mC, a.E + (G + g) * N + 64 * q, t0 + i0, &bar_cb);
            tma_load_2d(sBM + q * 32768, &mB, a.E + g * N + 64 * q, t0, &bar_cb);
        }
        cb_pending = true;
        issue_xs(g * hpg, 0);
        if (mbar_wait(&bar_cb, 0, a.status)) {
            cb_pending = false;
            tc_fence_after();
            // G = C B^T (fp16 operands, both K-major) into TMEM columns [0, jn)
            for (int k = 0; k < nkN; ++k)
                tc_mma(tmem, desc_sw128(smem_u32(sC + (k >> 2) * 16384 + (k & 3) * 32)),
                       desc_sw128(smem_u32(sBM + (k >> 2) * 32768 + (k & 3) * 32)), umma_idesc(false, false, kRows, jn),
                       k > 0);
            tc_commit(&bar_g);
        }
    }
    bool ok = __syncthreads_and(mbar_wait(&bar_g, 0, a.status));
    tc_fence_after();
    if (ok) {
        // the C rows to bf16 in place (same swizzled positions): the G MMAs have consumed them
        for (int q = tid; q < L.NA * 1024; q += kOutThreads) {
            uint4* p = reinterpret_cast<uint4*>(sC) + q;
            uint4 v = *p;
            v.x = f16x2_to_bf16x2(v.x);
            v.y = f16x2_to_bf16x2(v.y);
            v.z = f16x2_to_bf16x2(v.z);
            v.w = f16x2_to_bf16x2(v.w);
            *p = v;
        }
    }

    const int lb = 32 * (warp & 3);      // the warp's TMEM lane quarter
    const int r = lb + lane;             // tile row = TMEM lane
    const int i = i0 + r;                // frame within the chunk
    const int ilim = i < len ? i : -1;   // columns j <= ilim are unmasked
    const int jh = jn / 2, jbeg = warp < 4 ? 0 : jh;
    const int wmax = i0 + lb + 31;       // the warp's last row
    const int qh = (L.PA + 1) / 2;
    const int qa = warp < 4 ? 0 : qh, qb = warp < 4 ? qh : L.PA;
    const uint32_t trow = tmem + ((uint32_t)lb << 16);
    constexpr float kLog2e = 1.4426950408889634f;

    for (int hh = 0; hh < hpg && ok; ++hh) {
        const int h = g * hpg + hh;
        for (int j = tid; j < kQ; j += kOutThreads) {
            lam2[j] = j < len ? a.lam[(size_t)(t0 + j) * H + h] * kLog2e : 0.0f;
            dts[j] = j < len ? a.dt[(size_t)(t0 + j) * H + h] : 0.0f;
        }
        __syncthreads();
        // M_h[i][j] = G[i][j] 2^(lam2_i - lam2_j) dt_j for j <= i, fp16, K-major 128-byte swizzle
        {
            const float li = lam2[min(i, kQ - 1)];
            for (int j0 = jbeg; j0 < jbeg + jh; j0 += 32) {
                uint32_t pk[16];
                if (j0 > wmax) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) pk[e] = 0u;
                } else {
                    float gv[32];
                    tc_ld32(trow + (uint32_t)j0, gv);
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const int j = j0 + e;
                        const float v0 = j <= ilim ? gv[e] * ex2_approx(li - lam2[j]) * dts[j] : 0.0f;
                        const float v1 = j + 1 <= ilim ? gv[e + 1] * ex2_approx(li - lam2[j + 1]) * dts[j + 1] : 0.0f;
                        pk[e >> 1] = pack_f16x2_sat(v0, v1);
                    }
                }
                uint8_t* rowp = sBM + (j0 >> 6) * 16384 + r * 128;
                const int c0 = (j0 & 63) >> 3;
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<uint4*>(rowp + (((c0 + q) ^ (r & 7)) << 4)) =
                        make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
            }
        }
        fence_proxy_async();   // the generic-proxy writes of M_h (and C) -> the tensor core's reads
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            if (mbar_wait(&bar_x, x_phase, a.status)) {
                x_pending = false;
                tc_fence_after();
                // Y1 = M_h X_h: fp16, x MN-major (16-wide blocks 8 KB apart, 8-frame groups 256 B apart)
                for (int k = 0; k < jn / 16; ++k)
                    tc_mma(tmem + kColY1, desc_sw128(smem_u32(sBM + (k >> 2) * 16384 + (k & 3) * 32)),
                           umma_desc(smem_u32(sX + k * 512), 8192, 256, UMMA_SW32), umma_idesc(false, true, kRows, P),
                           k > 0);
                // Y2 = C S_in^T: bf16, both K-major
                for (int k = 0; k < nkN; ++k)
                    tc_mma(tmem + kColY2, desc_sw128(smem_u32(sC + (k >> 2) * 16384 + (k & 3) * 32)),
                           desc_sw128(smem_u32(sS + (k >> 2) * P * 128 + (k & 3) * 32)), umma_idesc(true, false, kRows, P),
                           k > 0);
                tc_commit(&bar_y);
            }
        }
        ok = __syncthreads_and(mbar_wait(&bar_y, (uint32_t)(hh & 1), a.status));
        tc_fence_after();
        if (!ok) break;
        // y_i = Y1 + exp(Lam_i) Y2 + D x_i; x_i from the staged fp16 tile (32-byte swizzle: the two
        // 16-byte halves of row j swap when bit 2 of j is set)
        {
            const float el = ex2_approx(lam2[min(i, kQ - 1)]);
            const float Dh = a.Dv[h];
            float* yrow = a.y + (size_t)(t0 + min(i, len - 1)) * a.E + (size_t)h * P;
            const uint32_t sw = ((uint32_t)i >> 2) & 1u;
            for (int q = qa; q < qb; ++q) {
                float y1[16], y2[16];
                tc_ld16(trow + kColY1 + 16 * q, y1);
                tc_ld16(trow + kColY2 + 16 * q, y2);
                const uint8_t* xr = sX + q * 8192 + i * 32;
                const uint4 xa = *reinterpret_cast<const uint4*>(xr + (sw << 4));
                const uint4 xb = *reinterpret_cast<const uint4*>(xr + ((sw ^ 1u) << 4));
                const uint32_t xw[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
                if (i < len) {
#pragma unroll
                    for (int e4 = 0; e4 < 4; ++e4) {
                        const __half2 p0 = u32_as_h2(xw[2 * e4]), p1 = u32_as_h2(xw[2 * e4 + 1]);
                        const float xv[4] = {__low2float(p0), __high2float(p0), __low2float(p1), __high2float(p1)};
                        float4 o;
                        o.x = fmaf(Dh, xv[0], fmaf(el, y2[4 * e4], y1[4 * e4]));
                        o.y = fmaf(Dh, xv[1], fmaf(el, y2[4 * e4 + 1], y1[4 * e4 + 1]));
                        o.z = fmaf(Dh, xv[2], fmaf(el, y2[4 * e4 + 2], y1[4 * e4 + 2]));
                        o.w = fmaf(Dh, xv[3], fmaf(el, y2[4 * e4 + 3], y1[4 * e4 + 3]));
                        reinterpret_cast<float4*>(yrow + 16 * q)[e4] = o;
                    }
                }
            }
        }
        tc_fence_before();
        __syncthreads();   // TMEM, x and lam2 reads done before the next head's copies and writes
        // the next head's x and S_in: the buffers are free (MMAs complete, epilogue read x); the
        // copies overlap the next head's M_h
        if (tid == 0 && hh + 1 < hpg) issue_xs(h + 1, (uint32_t)((hh + 1) & 1));
    }
    // a failed wait may leave copies in flight: give them a bounded chance to land
    if (tid == 0) {
        if (cb_pending) mbar_wait(&bar_cb, 0, nullptr);
        if (x_pending) mbar_wait(&bar_x, x_phase, nullptr);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------------------------------
// chunk states:  S_c[p][n] = sum_j w_j x_j[p] B_j[n],  w_j = exp(Lam_end - Lam_j) dt_j
// As a contraction over the chunk's frames with M = n (the state dimension, 128 TMEM lanes),
// N = p and K = j, both operands MN-major (their frame rows are n- and p-contiguous):
//   A = B_g^T: 128-byte swizzle, two 64-wide n blocks;  B = (w x_h): 32-byte swizzle, P/16 blocks.
// The state that decode continues from must meet the fp32 bound, so each operand is split into
// two fp16 halves (v = hi + lo, lo = v - hi) and the product is hi.hi + hi.lo + lo.hi (the dropped
// lo.lo term is ~2^-22 of the product), accumulated in fp32 in TMEM.  CTA = (chunk, head), frames
// in slabs of 64 staged by the threads (the split needs the fp32 values); a few CTAs per SM
// overlap one CTA's staging with another's MMAs.  The within-chunk cumulative log decay is
// scanned in double precision (one warp), as the decay weights come from its differences.
// ------------------------------------------------------------------------------------------
static constexpr int kStSlab = 64;
static constexpr int kStThreads = 256;
static constexpr uint32_t kStTmemCols = 128;

struct SsdStPlan {
    uint32_t off_ah, off_al, off_xh, off_xl, total;
};

__host__ __device__ inline SsdStPlan ssd_st_plan(int P) {
    SsdStPlan L{};
    L.off_ah = 0;                                 // B_g^T hi: 2 blocks x 64 rows x 128 B
    L.off_al = 16384;                             //          lo
    L.off_xh = 32768;                             // (w x) hi: P/16 blocks x 64 rows x 32 B
    L.off_xl = L.off_xh + (uint32_t)P * 128u;     //          lo
    L.total = L.off_xl + (uint32_t)P * 128u;
    return L;
}

VC_DEV void split_f16x8(const float (&v)[8], uint4& hi, uint4& lo) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const __half2 hh = __floats2half2_rn(v[2 * e], v[2 * e + 1]);
        const __half2 ll = __floats2half2_rn(v[2 * e] - __low2float(hh), v[2 * e + 1] - __high2float(hh));
        h[e] = h2_as_u32(hh);
        l[e] = h2_as_u32(ll);
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

__global__ void __launch_bounds__(kStThreads) pf_ssd_state_tc_kernel(const float* __restrict__ xc,
                                                                     const float* __restrict__ dt,
                                                                     const float* __restrict__ A_log, int T, int H,
                                                                     int P, int G, int E, int Cx,
                                                                     float* __restrict__ lam,
                                                                     float* __restrict__ schunk, int* status) {
    constexpr int N = 128;
    extern __shared__ uint8_t smraw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
    __shared__ double lamd[kQ];
    __shared__ float w[kQ];
    __shared__ uint64_t bar_mma;
    __shared__ uint32_t tmem_base;
    const int c = blockIdx.x, h = blockIdx.y;
    const int t0 = c * kQ, len = min(kQ, T - t0);
    const int g = (int)((long long)h * G / H);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const SsdStPlan L = ssd_st_plan(P);
    const float A = -expf(A_log[h]);

    if (tid == 0) {
        mbar_init(&bar_mma, 1);
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(&tmem_base, kStTmemCols);
    // inclusive scan of A dt over the chunk (warp 0), summed in double; each Lam rounded once
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
                lamd[i] = v;
                lam[(size_t)(t0 + i) * H + h] = (float)v;
            }
            run = __shfl_sync(0xffffffffu, v, 31);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;
    // decay weights from differences of the unrounded sums
    const double lend = lamd[len - 1];
    for (int i = tid; i < kQ; i += kStThreads)
        w[i] = i < len ? expf((float)(lend - lamd[i])) * dt[(size_t)(t0 + i) * H + h] : 0.0f;
    __syncthreads();

    const float* xh = xc + (size_t)t0 * Cx + (size_t)h * P;
    const float* bg = xc + (size_t)t0 * Cx + E + (size_t)g * N;
    const int p8 = P / 8;
    const uint32_t idesc = umma_idesc(false, true, N, P, true);
    const int nsl = (len + kStSlab - 1) / kStSlab;
    bool ok = true;
    for (int sl = 0; sl < nsl; ++sl) {
        if (sl > 0) {   // the previous slab's MMAs have read the staging buffers
            ok = __syncthreads_and(mbar_wait(&bar_mma, (uint32_t)((sl - 1) & 1), status));
            if (!ok) break;
        }
        const int f0 = sl * kStSlab;
        for (int idx = tid; idx < kStSlab * (N / 8); idx += kStThreads) {
            const int j = idx >> 4, nc = idx & 15;
            float v[8];
            if (f0 + j < len) {
                const float4 a0 = *reinterpret_cast<const float4*>(bg + (size_t)(f0 + j) * Cx + 8 * nc);
                const float4 a1 = *reinterpret_cast<const float4*>(bg + (size_t)(f0 + j) * Cx + 8 * nc + 4);
                v[0] = a0.x; v[1] = a0.y; v[2] = a0.z; v[3] = a0.w; v[4] = a1.x; v[5] = a1.y; v[6] = a1.z; v[7] = a1.w;
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) v[e] = 0.0f;
            }
            uint4 hi, lo;
            split_f16x8(v, hi, lo);
            const uint32_t off = (uint32_t)(nc >> 3) * 8192u + (uint32_t)j * 128u + ((uint32_t)((nc & 7) ^ (j & 7)) << 4);
            *reinterpret_cast<uint4*>(sm + L.off_ah + off) = hi;
            *reinterpret_cast<uint4*>(sm + L.off_al + off) = lo;
        }
        for (int idx = tid; idx < kStSlab * p8; idx += kStThreads) {
            const int j = idx / p8, pc = idx - j * p8;
            float v[8];
            if (f0 + j < len) {
                const float wj = w[f0 + j];
                const float4 a0 = *reinterpret_cast<const float4*>(xh + (size_t)(f0 + j) * Cx + 8 * pc);
                const float4 a1 = *reinterpret_cast<const float4*>(xh + (size_t)(f0 + j) * Cx + 8 * pc + 4);
                v[0] = a0.x * wj; v[1] = a0.y * wj; v[2] = a0.z * wj; v[3] = a0.w * wj;
                v[4] = a1.x * wj; v[5] = a1.y * wj; v[6] = a1.z * wj; v[7] = a1.w * wj;
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) v[e] = 0.0f;
            }
            uint4 hi, lo;
            split_f16x8(v, hi, lo);
            const uint32_t off = (uint32_t)(pc >> 1) * 2048u + (uint32_t)j * 32u + ((uint32_t)((pc & 1) ^ ((j >> 2) & 1)) << 4);
            *reinterpret_cast<uint4*>(sm + L.off_xh + off) = hi;
            *reinterpret_cast<uint4*>(sm + L.off_xl + off) = lo;
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const uint32_t ah = smem_u32(sm + L.off_ah), al = smem_u32(sm + L.off_al);
            const uint32_t bh = smem_u32(sm + L.off_xh), bl = smem_u32(sm + L.off_xl);
#pragma unroll
            for (int k = 0; k < kStSlab / 16; ++k) {
                const uint64_t dah = umma_desc(ah + k * 2048, 8192, 1024, UMMA_SW128);
                const uint64_t dal = umma_desc(al + k * 2048, 8192, 1024, UMMA_SW128);
                const uint64_t dbh = umma_desc(bh + k * 512, 2048, 256, UMMA_SW32);
                const uint64_t dbl = umma_desc(bl + k * 512, 2048, 256, UMMA_SW32);
                tc_mma(tmem, dah, dbh, idesc, (sl | k) != 0);
                tc_mma(tmem, dah, dbl, idesc, 1);
                tc_mma(tmem, dal, dbh, idesc, 1);
            }
            tc_commit(&bar_mma);
        }
    }
    if (ok) ok = __syncthreads_and(mbar_wait(&bar_mma, (uint32_t)((nsl - 1) & 1), status));
    tc_fence_after();
    if (ok) {
        // thread = state row n (TMEM lane); warps w and w + 4 split the P columns in blocks of 16
        const int lb = 32 * (warp & 3), n = lb + lane;
        const int PA = P / 16, qh = (PA + 1) / 2;
        const int qa = warp < 4 ? 0 : qh, qb = warp < 4 ? qh : PA;
        float* S = schunk + ((size_t)c * H + h) * P * N;
        for (int q = qa; q < qb; ++q) {
            float v[16];
            tc_ld16(tmem + ((uint32_t)lb << 16) + 16 * q, v);
#pragma unroll
            for (int e = 0; e < 16; ++e) S[(size_t)(16 * q + e) * N + n] = v[e];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kStTmemCols);
    }
}

bool ssd_state_tc_supported(int N, int P, int E, int Cx) {
    return N == 128 && P % 16 == 0 && P >= 16 && P <= 256 && E % 4 == 0 && Cx % 4 == 0;
}

cudaError_t launch_ssd_state_tc(const float* xc, const float* dt, const float* A_log, int T, int H, int P, int N, int G,
                                int E, int Cx, float* lam, float* schunk, int* status, cudaStream_t s) {
    if (!ssd_state_tc_supported(N, P, E, Cx) || T < 1 || !status || (((uintptr_t)xc) & 15)) return cudaErrorInvalidValue;
    const size_t smem = (size_t)ssd_st_plan(P).total + 1024;
    cudaError_t e =
        cudaFuncSetAttribute(pf_ssd_state_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int nch = (T + kQ - 1) / kQ;
    pf_ssd_state_tc_kernel<<<dim3(nch, H), kStThreads, smem, s>>>(xc, dt, A_log, T, H, P, G, E, Cx, lam, schunk,
                                                                  status);
    return cudaGetLastError();
}

bool ssd_out_tc_supported(int N, int P, int E, int Cx) {
    return N % 64 == 0 && N >= 64 && N <= 128 && P % 16 == 0 && P >= 16 && P <= 128 && E % 8 == 0 && Cx % 8 == 0;
}

cudaError_t launch_ssd_out_tc(const uint16_t* xc16, const uint16_t* sin16, const float* dt, const float* lam,
                              const float* Dv, float* y, int T, int H, int P, int N, int G, int E, int Cx, int* status,
                              cudaStream_t s) {
    if (!ssd_out_tc_supported(N, P, E, Cx) || H % G || T < 1 || !status) return cudaErrorInvalidValue;
    if ((((uintptr_t)xc16) & 15) || (((uintptr_t)sin16) & 15)) return cudaErrorInvalidValue;
    const int nch = (T + kQ - 1) / kQ;
    CUtensorMap mC, mB, mX, mS;
    if (!tma_map_2d(&mC, xc16, T, Cx, Cx, 64, kRows, true, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !tma_map_2d(&mB, xc16, T, Cx, Cx, 64, kQ, true, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !tma_map_2d(&mX, xc16, T, Cx, Cx, 16, kQ, true, CU_TENSOR_MAP_SWIZZLE_32B) ||
        !tma_map_2d(&mS, sin16, nch * H * P, N, N, 64, P, false, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const size_t smem = (size_t)ssd_out_plan(N, P).total + 1024;
    cudaError_t e = cudaFuncSetAttribute(pf_ssd_out_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    SsdOutArgs a{};
    a.dt = dt; a.lam = lam; a.Dv = Dv; a.y = y;
    a.T = T; a.H = H; a.P = P; a.N = N; a.G = G; a.E = E;
    a.status = status;
    pf_ssd_out_tc_kernel<<<2 * nch * G, kOutThreads, smem, s>>>(mC, mB, mX, mS, a);
    return cudaGetLastError();
}

}  // namespace vc
