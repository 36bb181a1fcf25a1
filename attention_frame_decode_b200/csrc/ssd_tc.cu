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
//     x and S_in are double-buffered: the next head's copies run under this head's work.
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
static_assert(kQ == kOutThreads, "one thread per frame of the chunk stages the decay of a head");

// shared-memory plan of the output kernel (byte offsets from a 1024-aligned base)
struct SsdOutPlan {
    int NA, PA;                                 // 64-wide atoms of N, 16-wide blocks of P
    uint32_t off_c, off_bm, off_x0, off_s0, off_x1, off_s1, total;
};

__host__ __device__ inline SsdOutPlan ssd_out_plan(int N, int P) {
    SsdOutPlan L{};
    L.NA = N / 64;
    L.PA = P / 16;
    L.off_c = 0;                                               // C rows: NA atoms x 128 rows x 128 B
    const uint32_t bm = (uint32_t)L.NA * 32768u > 65536u ? (uint32_t)L.NA * 32768u : 65536u;
    L.off_bm = L.off_c + (uint32_t)L.NA * 16384u;              // B rows (NA x 256 x 128 B), then M_h (4 x 128 x 128 B)
                                                               // and the y staging tile (PA x 128 rows x 64 B)
    // two buffers (heads alternate) of x_h (PA blocks x 256 rows x 32 B) and S_in,h (NA atoms x P
    // rows x 128 B)
    const uint32_t xb = (uint32_t)L.PA * 8192u, sb = (uint32_t)L.NA * (uint32_t)P * 128u;
    L.off_x0 = L.off_bm + bm;
    L.off_s0 = L.off_x0 + xb;
    L.off_x1 = L.off_s0 + sb;
    L.off_s1 = L.off_x1 + xb;
    L.total = L.off_s1 + sb;
    return L;
}

VC_DEV float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

VC_DEV float lg2_approx(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// fp16 pair (lo in the low half), saturated to the finite range
VC_DEV uint32_t pack_f16x2_sat(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

VC_DEV uint32_t f16x2_to_bf16x2(uint32_t v) {
    const __half2 h = u32_as_h2(v);
    const __nv_bfloat162 b = __floats2bfloat162_rn(__low2float(h), __high2float(h));
    return *reinterpret_cast<const uint32_t*>(&b);
}

VC_DEV void tma_store_2d(const CUtensorMap* map, const void* src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(map), "r"(x),
                 "r"(y), "r"(smem_u32(src))
                 : "memory");
}
VC_DEV void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
VC_DEV void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
VC_DEV void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

struct SsdOutArgs {
    const float* dt;    // [T][H]
    const float* lam;   // [T][H] within-chunk cumulative A dt
    const float* Dv;    // [H]
    int T, H, P, N, G, E;
    int* status;
};

// warp 4 (whose rows see the fewest unmasked columns) issues the copies, one per lane (the TMA
// engine works on several boxes at once), and its lane 0 the MMAs
static constexpr int kIssuerWarp = 4;

__global__ void __launch_bounds__(kOutThreads, 1)
    pf_ssd_out_tc_kernel(const __grid_constant__ CUtensorMap mBC, const __grid_constant__ CUtensorMap mX,
                         const __grid_constant__ CUtensorMap mS, const __grid_constant__ CUtensorMap mY,
                         const SsdOutArgs a) {
    extern __shared__ uint8_t smraw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t bar_cb, bar_g, bar_x[2], bar_y;
    __shared__ uint32_t tmem_base;
    __shared__ __align__(16) float lam2[kQ];   // log2 of the cumulative decay, per frame
    __shared__ __align__(16) float qv[kQ];     // lam2_j - log2(dt_j): 2^(lam2_i - qv_j) = decay x dt_j

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
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int hpg = H / G, nkN = N / 16;
    const bool iwarp = warp == kIssuerWarp, issuer = iwarp && lane == 0;

    if (tid == 0) {
        mbar_init(&bar_cb, 1);
        mbar_init(&bar_g, 1);
        mbar_init(&bar_x[0], 1);
        mbar_init(&bar_x[1], 1);
        mbar_init(&bar_y, 1);
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(&tmem_base, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;

    // copies of head hh's x and S_in go to buffer hh & 1 (completion phase (hh >> 1) & 1); the
    // issuer warp calls this together: lane 0 registers the bytes, then each lane issues one box
    const int nrh = jn / kRows;   // 128-row halves of the frames j < jn
    bool cb_pending = false;
    uint32_t x_pend = 0u, x_ph = 0u;   // copies in flight per buffer (bit b) and their phases
    auto issue_xs = [&](int hh) {
        const int b = hh & 1, h = g * hpg + hh;
        uint64_t* bar = &bar_x[b];
        uint8_t* sX = sm + (b ? L.off_x1 : L.off_x0);
        uint8_t* sS = sm + (b ? L.off_s1 : L.off_s0);
        if (lane == 0)
            mbar_arrive_expect_tx(bar, (uint32_t)L.PA * (uint32_t)jn * 32u + (uint32_t)L.NA * (uint32_t)P * 128u);
        __syncwarp();
        const int nx = L.PA * nrh;
        if (lane < nx) {
            const int q = lane / nrh, r0 = (lane - q * nrh) * kRows;
            tma_load_2d(sX + q * 8192 + r0 * 32, &mX, h * P + 16 * q, t0 + r0, bar);
        } else if (lane < nx + L.NA) {
            const int q = lane - nx;
            tma_load_2d(sS + q * P * 128, &mS, 64 * q, (c * H + h) * P, bar);
        }
        x_pend |= 1u << b;
        x_ph = (x_ph & ~(1u << b)) | ((uint32_t)((hh >> 1) & 1) << b);
    };
    if (iwarp) {
        // C rows of the tile; B rows of the frames j < jn (128-row boxes)
        if (lane == 0) mbar_arrive_expect_tx(&bar_cb, (uint32_t)L.NA * (16384u + (uint32_t)jn * 128u));
        __syncwarp();
        if (lane < L.NA) {
            tma_load_2d(sC + lane * 16384, &mBC, a.E + (G + g) * N + 64 * lane, t0 + i0, &bar_cb);
        } else if (lane < L.NA + L.NA * nrh) {
            const int q = (lane - L.NA) / nrh, r0 = (lane - L.NA - q * nrh) * kRows;
            tma_load_2d(sBM + q * 32768 + r0 * 128, &mBC, a.E + g * N + 64 * q, t0 + r0, &bar_cb);
        }
        cb_pending = true;
        issue_xs(0);
    }
    if (issuer) {
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
    const int wmin = i0 + lb, wmax = wmin + 31;   // the warp's rows
    const bool wfull = wmax < len;                 // every row of the warp is a frame of the chunk
    const int qh = (L.PA + 1) / 2;
    const int qa = warp < 4 ? 0 : qh, qb = warp < 4 ? qh : L.PA;
    const uint32_t trow = tmem + ((uint32_t)lb << 16);
    constexpr float kLog2e = 1.4426950408889634f;
    // Lam and dt of frame tid for the next head, loaded one head ahead (kQ == kOutThreads)
    const bool fr = tid < len;
    float nl = fr ? a.lam[(size_t)(t0 + tid) * H + g * hpg] : 0.0f;
    float nd = fr ? a.dt[(size_t)(t0 + tid) * H + g * hpg] : 0.0f;

    for (int hh = 0; hh < hpg && ok; ++hh) {
        const int h = g * hpg + hh, b = hh & 1;
        uint8_t* sX = sm + (b ? L.off_x1 : L.off_x0);
        uint8_t* sS = sm + (b ? L.off_s1 : L.off_s0);
        {
            const float l2 = nl * kLog2e;
            lam2[tid] = l2;
            qv[tid] = nd > 0.0f ? l2 - lg2_approx(nd) : INFINITY;
            if (hh + 1 < hpg && fr) {
                nl = a.lam[(size_t)(t0 + tid) * H + h + 1];
                nd = a.dt[(size_t)(t0 + tid) * H + h + 1];
            }
        }
        const float Dh = a.Dv[h];
        // the previous head's y store has read the staging tile (the M_h buffer)
        if (iwarp && hh > 0 && lane < L.PA) bulk_wait_read0();
        __syncthreads();
        // the next head's copies into the other buffer (its last reader, head hh - 1, is done)
        if (iwarp && hh + 1 < hpg) issue_xs(hh + 1);
        // M_h[i][j] = G[i][j] 2^(lam2_i - qv_j) for j <= i, fp16, K-major 128-byte swizzle
        {
            const float li = lam2[min(i, kQ - 1)];
            for (int j0 = jbeg; j0 < jbeg + jh; j0 += 64) {
                uint32_t pk[32];
                if (j0 > wmax) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) pk[e] = 0u;
                } else {
                    float gv[64];
                    tc_ld64(trow + (uint32_t)j0, gv);
                    if (wfull && j0 + 63 <= wmin) {   // below the diagonal for every row of the warp
#pragma unroll
                        for (int e = 0; e < 64; e += 4) {
                            const float4 q4 = *reinterpret_cast<const float4*>(qv + j0 + e);
                            pk[e >> 1] = pack_f16x2_sat(gv[e] * ex2_approx(li - q4.x), gv[e + 1] * ex2_approx(li - q4.y));
                            pk[(e >> 1) + 1] =
                                pack_f16x2_sat(gv[e + 2] * ex2_approx(li - q4.z), gv[e + 3] * ex2_approx(li - q4.w));
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 64; e += 4) {
                            const int j = j0 + e;
                            const float4 q4 = *reinterpret_cast<const float4*>(qv + j);
                            const float v0 = j <= ilim ? gv[e] * ex2_approx(li - q4.x) : 0.0f;
                            const float v1 = j + 1 <= ilim ? gv[e + 1] * ex2_approx(li - q4.y) : 0.0f;
                            const float v2 = j + 2 <= ilim ? gv[e + 2] * ex2_approx(li - q4.z) : 0.0f;
                            const float v3 = j + 3 <= ilim ? gv[e + 3] * ex2_approx(li - q4.w) : 0.0f;
                            pk[e >> 1] = pack_f16x2_sat(v0, v1);
                            pk[(e >> 1) + 1] = pack_f16x2_sat(v2, v3);
                        }
                    }
                }
                uint8_t* rowp = sBM + (j0 >> 6) * 16384 + r * 128;
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    *reinterpret_cast<uint4*>(rowp + ((q ^ (r & 7)) << 4)) =
                        make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
            }
        }
        fence_proxy_async();   // the generic-proxy writes of M_h (and C) -> the tensor core's reads
        tc_fence_before();
        __syncthreads();
        if (issuer) {
            if (mbar_wait(&bar_x[b], (uint32_t)((hh >> 1) & 1), a.status)) {
                x_pend &= ~(1u << b);
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
        // y_i = Y1 + exp(Lam_i) Y2 + D x_i into the staging tile (the M_h buffer is free): block q of
        // 16 columns is 128 rows x 64 B with the 64-byte swizzle (16-byte chunk c of row r at
        // c ^ ((r >> 1) & 3)).  x_i comes from the staged fp16 tile (32-byte swizzle: the two
        // 16-byte halves of row j swap when bit 2 of j is set).
        {
            const float el = ex2_approx(lam2[min(i, kQ - 1)]);
            const uint32_t sw = ((uint32_t)i >> 2) & 1u;
            for (int q = qa; q < qb; ++q) {
                float y1[16], y2[16];
                tc_ld16x2(trow + kColY1 + 16 * q, trow + kColY2 + 16 * q, y1, y2);
                const uint8_t* xr = sX + q * 8192 + i * 32;
                const uint4 xa = *reinterpret_cast<const uint4*>(xr + (sw << 4));
                const uint4 xb = *reinterpret_cast<const uint4*>(xr + ((sw ^ 1u) << 4));
                const uint32_t xw[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
                uint8_t* yr = sBM + q * 8192 + r * 64;
#pragma unroll
                for (int e4 = 0; e4 < 4; ++e4) {
                    const __half2 p0 = u32_as_h2(xw[2 * e4]), p1 = u32_as_h2(xw[2 * e4 + 1]);
                    float4 o;
                    o.x = fmaf(Dh, __low2float(p0), fmaf(el, y2[4 * e4], y1[4 * e4]));
                    o.y = fmaf(Dh, __high2float(p0), fmaf(el, y2[4 * e4 + 1], y1[4 * e4 + 1]));
                    o.z = fmaf(Dh, __low2float(p1), fmaf(el, y2[4 * e4 + 2], y1[4 * e4 + 2]));
                    o.w = fmaf(Dh, __high2float(p1), fmaf(el, y2[4 * e4 + 3], y1[4 * e4 + 3]));
                    *reinterpret_cast<float4*>(yr + ((e4 ^ ((r >> 1) & 3)) << 4)) = o;
                }
            }
        }
        fence_proxy_async();   // the staging tile -> the TMA store's reads
        tc_fence_before();
        __syncthreads();       // TMEM, x, lam2 and staging done before the store and the next head
        if (iwarp && lane < L.PA) {   // rows beyond T are clipped by the store
            tma_store_2d(&mY, sBM + lane * 8192, h * P + 16 * lane, t0 + i0);
            bulk_commit();
        }
    }
    // a failed wait may leave copies in flight: give them a bounded chance to land
    if (iwarp && lane < L.PA) bulk_wait0();
    if (issuer) {
        if (cb_pending) mbar_wait(&bar_cb, 0, nullptr);
        for (int b = 0; b < 2; ++b)
            if (x_pend & (1u << b)) mbar_wait(&bar_x[b], (x_ph >> b) & 1u, nullptr);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

bool ssd_out_tc_supported(int N, int P, int E, int Cx) {
    return N % 64 == 0 && N >= 64 && N <= 128 && P % 16 == 0 && P >= 16 && P <= 128 && E % 8 == 0 && Cx % 8 == 0;
}

cudaError_t launch_ssd_out_tc(const uint16_t* xc16, const uint16_t* sin16, const float* dt, const float* lam,
                              const float* Dv, float* y, int T, int H, int P, int N, int G, int E, int Cx, int* status,
                              cudaStream_t s) {
    if (!ssd_out_tc_supported(N, P, E, Cx) || H % G || T < 1 || !status) return cudaErrorInvalidValue;
    if ((((uintptr_t)xc16) & 15) || (((uintptr_t)sin16) & 15) || (((uintptr_t)y) & 15)) return cudaErrorInvalidValue;
    const int nch = (T + kQ - 1) / kQ;
    CUtensorMap mBC, mX, mS, mY;
    if (!tma_map_2d(&mBC, xc16, T, Cx, Cx, 64, kRows, true, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !tma_map_2d(&mX, xc16, T, Cx, Cx, 16, kRows, true, CU_TENSOR_MAP_SWIZZLE_32B) ||
        !tma_map_2d(&mS, sin16, nch * H * P, N, N, 64, P, false, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !tma_map_2d_f32(&mY, y, T, E, E, 16, kRows, CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    const size_t smem = (size_t)ssd_out_plan(N, P).total + 1024;
    cudaError_t e = cudaFuncSetAttribute(pf_ssd_out_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    SsdOutArgs a{};
    a.dt = dt; a.lam = lam; a.Dv = Dv;
    a.T = T; a.H = H; a.P = P; a.N = N; a.G = G; a.E = E;
    a.status = status;
    pf_ssd_out_tc_kernel<<<2 * nch * G, kOutThreads, smem, s>>>(mBC, mX, mS, mY, a);
    return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// chunk states:  S_c[p][n] = sum_j w_j x_j[p] B_j[n],  w_j = exp(Lam_end - Lam_j) dt_j
// As a contraction over the chunk's frames with M = n (the state dimension, 128 TMEM lanes),
// N = p and K = j, both operands MN-major (their frame rows are n- and p-contiguous):
//   A = B_g^T: 128-byte swizzle, two 64-wide n blocks;  B = (w x_h): 32-byte swizzle, P/16 blocks.
// The state that decode continues from must meet the fp32 bound, so each operand is split into
// two fp16 halves (v = hi + lo, lo = v - hi) and the product is hi.hi + hi.lo + lo.hi (the dropped
// lo.lo term is ~2^-22 of the product), accumulated in fp32 in TMEM: the hi.hi products in one
// accumulator and the two correction products, ~2^-11 smaller, in a second one, added in fp32 at
// the end, so that the corrections are not rounded against the much larger main sums.  CTA = (chunk, head), frames
// in slabs of 64 staged by the threads (the split needs the fp32 values); a few CTAs per SM
// overlap one CTA's staging with another's MMAs.  The within-chunk cumulative log decay is
// scanned in double precision (one warp), as the decay weights come from its differences.
// ------------------------------------------------------------------------------------------
static constexpr int kStSlab = 64;
static constexpr int kStThreads = 256;
static constexpr uint32_t kStTmemCols = 256;   // hi.hi sums in [0, P), hi.lo + lo.hi sums in [128, 128 + P)

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
    constexpr int AR = kStSlab * (N / 8) / kStThreads;   // B rows: 8-value items per thread and slab
    constexpr int XR = kStSlab * (128 / 8) / kStThreads; // x rows: up to P = 128
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
    const float* xh = xc + (size_t)t0 * Cx + (size_t)h * P;
    const float* bg = xc + (size_t)t0 * Cx + E + (size_t)g * N;
    const int p8 = P / 8;

    // the next slab's rows, prefetched into registers while the tensor core works on this one
    float4 ra[AR][2], rx[XR][2];
    auto load = [&](int f0) {
#pragma unroll
        for (int m = 0; m < AR; ++m) {
            const int idx = tid + m * kStThreads, j = idx >> 4, nc = idx & 15;
            ra[m][0] = ra[m][1] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (f0 + j < len) {
                const float* src = bg + (size_t)(f0 + j) * Cx + 8 * nc;
                ra[m][0] = *reinterpret_cast<const float4*>(src);
                ra[m][1] = *reinterpret_cast<const float4*>(src + 4);
            }
        }
#pragma unroll
        for (int m = 0; m < XR; ++m) {
            const int idx = tid + m * kStThreads, j = idx / p8, pc = idx - j * p8;
            rx[m][0] = rx[m][1] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (j < kStSlab && f0 + j < len) {
                const float* src = xh + (size_t)(f0 + j) * Cx + 8 * pc;
                rx[m][0] = *reinterpret_cast<const float4*>(src);
                rx[m][1] = *reinterpret_cast<const float4*>(src + 4);
            }
        }
    };
    // split into fp16 halves and write the MN-major swizzled tiles (x scaled by w_j)
    auto store = [&](int f0) {
#pragma unroll
        for (int m = 0; m < AR; ++m) {
            const int idx = tid + m * kStThreads, j = idx >> 4, nc = idx & 15;
            const float v[8] = {ra[m][0].x, ra[m][0].y, ra[m][0].z, ra[m][0].w,
                                ra[m][1].x, ra[m][1].y, ra[m][1].z, ra[m][1].w};
            uint4 hi, lo;
            split_f16x8(v, hi, lo);
            const uint32_t off = (uint32_t)(nc >> 3) * 8192u + (uint32_t)j * 128u + ((uint32_t)((nc & 7) ^ (j & 7)) << 4);
            *reinterpret_cast<uint4*>(sm + L.off_ah + off) = hi;
            *reinterpret_cast<uint4*>(sm + L.off_al + off) = lo;
        }
#pragma unroll
        for (int m = 0; m < XR; ++m) {
            const int idx = tid + m * kStThreads, j = idx / p8, pc = idx - j * p8;
            if (j >= kStSlab) continue;
            const float wj = f0 + j < len ? w[f0 + j] : 0.0f;
            const float v[8] = {rx[m][0].x * wj, rx[m][0].y * wj, rx[m][0].z * wj, rx[m][0].w * wj,
                                rx[m][1].x * wj, rx[m][1].y * wj, rx[m][1].z * wj, rx[m][1].w * wj};
            uint4 hi, lo;
            split_f16x8(v, hi, lo);
            const uint32_t off = (uint32_t)(pc >> 1) * 2048u + (uint32_t)j * 32u + ((uint32_t)((pc & 1) ^ ((j >> 2) & 1)) << 4);
            *reinterpret_cast<uint4*>(sm + L.off_xh + off) = hi;
            *reinterpret_cast<uint4*>(sm + L.off_xl + off) = lo;
        }
    };

    load(0);   // in flight during the scan
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
    for (int i = tid; i < len; i += kStThreads) w[i] = expf((float)(lend - lamd[i])) * dt[(size_t)(t0 + i) * H + h];
    __syncthreads();

    const uint32_t idesc = umma_idesc(false, true, N, P, true);
    const int nsl = (len + kStSlab - 1) / kStSlab;
    bool ok = true;
    for (int sl = 0; sl < nsl; ++sl) {
        if (sl > 0) {   // the previous slab's MMAs have read the staging buffers
            ok = __syncthreads_and(mbar_wait(&bar_mma, (uint32_t)((sl - 1) & 1), status));
            if (!ok) break;
        }
        store(sl * kStSlab);
        if (sl + 1 < nsl) load((sl + 1) * kStSlab);
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
                tc_mma(tmem + 128, dah, dbl, idesc, (sl | k) != 0);
                tc_mma(tmem + 128, dal, dbh, idesc, 1);
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
            float v[16], cr[16];
            tc_ld16x2(tmem + ((uint32_t)lb << 16) + 16 * q, tmem + ((uint32_t)lb << 16) + 128 + 16 * q, v, cr);
#pragma unroll
            for (int e = 0; e < 16; ++e) S[(size_t)(16 * q + e) * N + n] = v[e] + cr[e];
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
    return N == 128 && P % 16 == 0 && P >= 16 && P <= 128 && E % 4 == 0 && Cx % 4 == 0;
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

}  // namespace vc
