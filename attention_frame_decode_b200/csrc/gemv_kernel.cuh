// gemv_kernel.cuh -- streaming weight GEMV for the per-frame decode step (B <= 16 sessions).
//
// The per-frame LLM step is bound by memory bandwidth, and its time falls with the bits per
// weight (NemotronLabs VoiceChat 11B: GPTQ 3-bit LLM, MLX, the measurement bullets of the
// introduction), so the kernel is built to read every weight byte exactly once at full HBM rate:
//   * persistent grid (two 8-warp CTAs per SM for up to 8 batch rows, one for 9..16); each warp
//     is a worker that owns one contiguous
//     byte range of the matrix (see layout.cuh) and streams it through its own ring of shared
//     memory slots with 1-D bulk copies (cp.async.bulk, TMA engine) completing on mbarriers;
//   * the weight copies of the first ring slots are issued before griddepcontrol.wait, so they
//     overlap the tail of the previous kernel (programmatic dependent launch);
//   * dequantization is a few lop3/prmt + one fp16 op per pair of weights (exponent-field
//     trick: OR a code into the mantissa of 1024.0, subtract 1024 + z) feeding mma.sync
//     m16n8k16 with fp32 accumulation; quantization-group scales multiply the fp32 group sums;
//   * a unit (16R rows) cut between workers is finished by the last of them (atomic counter):
//     in the step the contributors add their fp32 sums into a per-unit accumulator with vector
//     reductions and the last one reads the total once; without an accumulator (test entries)
//     the last one adds the others' fp32 partials in worker order (deterministic); then it runs
//     the fused epilogue.
#pragma once
#include "common.cuh"
#include "gemv.cuh"
#include "layout.cuh"

namespace vc {

static constexpr int kWarps = 16;   // upper bound of warps per CTA (sizes the partial-sum scratch)
// warps per CTA: 8 for every batch size
__host__ __device__ constexpr int warps_for(int) { return 8; }
// CTAs per SM: two 8-warp CTAs for up to 8 rows (<= 128 registers, <= ~105 KB shared memory each),
// so that under programmatic dependent launch the next kernel's CTAs can become resident and
// start their weight copies while this kernel drains; one CTA for 9..16 rows
__host__ __device__ constexpr int ctas_per_sm(int NT) { return NT == 1 ? 2 : 1; }
static constexpr int kMaxB = 16;
static constexpr int kMaxSlots = 8;          // ring slots per warp (upper bound)
static constexpr int kRingBudget = 210 * 1024; // dynamic shared memory for the rings of one CTA

// ------------------------------------------------------------------------------------------
// partition helpers (worker w of W owns flat blocks [w*T/W, (w+1)*T/W))
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ long long llmin(long long a, long long b) { return a < b ? a : b; }
// With T (W + 1) < 2^32 (every shape of the backbone) the same integer quotients are taken in
// 32-bit arithmetic, which costs a fraction of a 64-bit division.
__device__ __forceinline__ long long part_begin(long long w, long long T, long long W, bool s32) {
    if (s32) return (long long)((uint32_t)w * (uint32_t)T / (uint32_t)W);
    return w * T / W;
}
// largest worker whose range starts at or before block f (always a non-empty range)
__device__ __forceinline__ long long part_owner(long long f, long long T, long long W, bool s32) {
    if (s32) return (long long)(((uint32_t)(f + 1) * (uint32_t)W + (uint32_t)T - 1u) / (uint32_t)T) - 1;
    return ((f + 1) * W + T - 1) / T - 1;
}

// ------------------------------------------------------------------------------------------
// A-fragment extraction, one 16x64 tile per call: a[step][reg]
// ------------------------------------------------------------------------------------------
struct QConst {
    uint32_t zg, zh;       // (1024 + z) pairs, rows g and g+8
    uint32_t f16g, f16h;   // -(64 + z)          (W4 high nibble)
    uint32_t f8g, f8h;     // -(128 + z)         (W3 field 1, 4)
    uint32_t f64g, f64h;   // -(16 + z)          (W3 field 2)
};

__device__ __forceinline__ uint32_t h2bits(float v) {
    __half h = __float2half_rn(v);
    uint16_t b = *reinterpret_cast<uint16_t*>(&h);
    return (uint32_t)b | ((uint32_t)b << 16);
}

template <int FMT>
__device__ __forceinline__ void load_tile_frags(const uint8_t* tile, int lane, const QConst& qc, uint32_t (&a)[4][4]) {
    const uint32_t M = 0x64006400u;
    if constexpr (FMT == FMT_BF16) {
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            uint4 v = *reinterpret_cast<const uint4*>(tile + (s * 32 + lane) * 16);
            a[s][0] = v.x; a[s][1] = v.y; a[s][2] = v.z; a[s][3] = v.w;
        }
    } else if constexpr (FMT == FMT_W8) {
        const uint32_t K1152 = 0x64806480u;   // 1024 + 128 as an fp16 pair
        const uint32_t M8 = 0x64646464u;      // prmt source of the 0x64 exponent byte
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            uint4 v = *reinterpret_cast<const uint4*>(tile + (c * 32 + lane) * 16);
            uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                int s = 2 * c + h;
                uint32_t A = w[2 * h], B = w[2 * h + 1];
                a[s][0] = hsub2_u32(prmt(A, M8, 0x4240), K1152);
                a[s][1] = hsub2_u32(prmt(B, M8, 0x4240), K1152);
                a[s][2] = hsub2_u32(prmt(A, M8, 0x4341), K1152);
                a[s][3] = hsub2_u32(prmt(B, M8, 0x4341), K1152);
            }
        }
    } else if constexpr (FMT == FMT_W4) {
        const uint32_t R16 = h2bits(1.0f / 16.0f);
        uint4 v = *reinterpret_cast<const uint4*>(tile + lane * 16);
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            uint32_t x = w[s], y = w[s] >> 8;
            a[s][0] = hsub2_u32(and_or(x, 0x000F000Fu, M), qc.zg);
            a[s][1] = hfma2_u32(and_or(x, 0x00F000F0u, M), R16, qc.f16h);
            a[s][2] = hsub2_u32(and_or(y, 0x000F000Fu, M), qc.zg);
            a[s][3] = hfma2_u32(and_or(y, 0x00F000F0u, M), R16, qc.f16h);
        }
    } else {  // W3
        const uint32_t R8 = h2bits(1.0f / 8.0f), R64 = h2bits(1.0f / 64.0f);
        uint2 v01 = *reinterpret_cast<const uint2*>(tile + lane * 8);
        uint32_t w[3] = {v01.x, v01.y, *reinterpret_cast<const uint32_t*>(tile + 256 + lane * 4)};
#pragma unroll
        for (int p = 0; p < 16; ++p) {
            const int s = p / 4, reg = p % 4;
            const bool hi = reg & 1;
            const uint32_t z = hi ? qc.zh : qc.zg, f8 = hi ? qc.f8h : qc.f8g, f64 = hi ? qc.f64h : qc.f64g;
            uint32_t r;
            if (p < 15) {
                const uint32_t x = w[p / 5];
                const int i = p % 5;
                if (i == 0) r = hsub2_u32(and_or(x, 0x00070007u, M), z);
                else if (i == 1) r = hfma2_u32(and_or(x, 0x00380038u, M), R8, f8);
                else if (i == 2) r = hfma2_u32(and_or(x, 0x01C001C0u, M), R64, f64);
                else if (i == 3) r = hsub2_u32(and_or(x >> 9, 0x00070007u, M), z);
                else r = hfma2_u32(and_or(x >> 9, 0x00380038u, M), R8, f8);
            } else {
                uint32_t c = ((w[0] >> 15) & 0x00010001u) | ((w[1] >> 14) & 0x00020002u) | ((w[2] >> 13) & 0x00040004u);
                r = hsub2_u32(c | M, z);
            }
            a[s][reg] = r;
        }
    }
}

template <int FMT>
__device__ __forceinline__ void mma_step(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    if constexpr (FMT == FMT_BF16) mma_bf16(d, a, b0, b1, d);
    else mma_f16(d, a, b0, b1, d);
}

// ------------------------------------------------------------------------------------------
// the kernel
// ------------------------------------------------------------------------------------------
struct RingGeom {
    int slots;        // ring slots per warp
    int slot_bytes;   // weights (bps blocks) [+ activation rows when act_smem == 0]
    int act_row;      // bytes per staged activation row (KS*2 + 16)
    int act_smem;     // 1: the whole activation [B][act_ld] is copied to shared memory once per CTA
    int act_stride;   // bytes per activation row in shared memory (act_ld*2 + 16)
};

template <int FMT, int GRP, int NT, int EPI>
__global__ void __launch_bounds__(warps_for(NT) * 32, ctas_per_sm(NT)) gemv_kernel(const GemvArgs args, const RingGeom rg) {
    constexpr int WARPS = warps_for(NT);
    constexpr LayoutInfo L = layout_info(FMT, GRP);
    constexpr int R = L.R, SUB = L.SUB, KS = L.KS;
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t bars[WARPS][kMaxSlots];
    __shared__ float insc_tab[kMaxB * 16];

    pdl_trigger();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int B = args.B;

    // ---- worker range -------------------------------------------------------------------
    const long long Wall = (long long)gridDim.x * WARPS;
    const long long wid = (long long)blockIdx.x * WARPS + warp;
    int m = 0;
    long long Wm = Wall, wl = wid, wbase = 0;
    if (args.nmat == 2) {
        long long W0 = Wall / 2;
        if (wid >= W0) { m = 1; wl = wid - W0; Wm = Wall - W0; wbase = W0; }
        else Wm = W0;
    }
    const GemvMat M = args.mat[m];
    const long long T = (long long)M.NU * M.KT;
    // with fewer blocks than warps only the first T workers get (one-block) ranges, so that every
    // worker between the first and last contributor of a unit is a contributor
    if (Wm > T) Wm = T;
    const bool idle = wl >= Wm;
    // block indices fit in 32 bits (at most a few 10^5 blocks per matrix); positions advance
    // incrementally so the hot loop has no integer division
    const bool s32 = (unsigned long long)T * (unsigned long long)(Wm + 1) < (1ull << 32);
    const int f0 = idle ? 0 : (int)part_begin(wl, T, Wm, s32), f1 = idle ? 0 : (int)part_begin(wl + 1, T, Wm, s32);
    const int bps = L.bps;
    const int nstages = (f1 - f0 + bps - 1) / bps;
    const int KT = M.KT;

    uint8_t* ring = smem + (size_t)warp * rg.slots * rg.slot_bytes;
    uint64_t* bar = bars[warp];
    const int act_rows = B;

    // stage i covers blocks [f0 + i*bps, min(f0 + (i+1)*bps, f1)) and lives in ring slot i mod slots
    auto issue_weights = [&](int i, int slot) {
        const int fb = f0 + i * bps;
        const int nb = min(bps, f1 - fb);
        const uint32_t wbytes = nb * L.block_bytes;
        const uint32_t abytes = rg.act_smem ? 0u : (uint32_t)(nb * act_rows * KS * 2);
        mbar_arrive_expect_tx(&bar[slot], wbytes + abytes);
        bulk_g2s(ring + (size_t)slot * rg.slot_bytes, M.w + (size_t)fb * L.block_bytes, wbytes, &bar[slot]);
    };
    int act_kt = f0 % KT;   // k-step of the next block whose activation slice is issued
    auto issue_act = [&](int i, int slot) {
        const int nb = min(bps, f1 - (f0 + i * bps));
        uint8_t* abase = ring + (size_t)slot * rg.slot_bytes + bps * L.block_bytes;
        for (int j = 0; j < nb; ++j) {
            for (int b = 0; b < act_rows; ++b)
                bulk_g2s(abase + (j * act_rows + b) * rg.act_row,
                         args.act + (size_t)b * args.act_ld + (size_t)act_kt * KS, KS * 2, &bar[slot]);
            if (++act_kt == KT) act_kt = 0;
        }
    };

    if (lane == 0) {
        for (int s = 0; s < rg.slots; ++s) mbar_init(&bar[s], 1);
        fence_mbar_init();
        for (int i = 0; i < nstages && i < rg.slots; ++i) issue_weights(i, i);
    }
    __syncwarp();

    pdl_wait();

    // ---- input-scale table (per CTA): one warp per (row b, norm group q) --------------------
    const int ng = args.insc.parts ? args.insc.n_groups : 1;
    for (int idx = warp; idx < B * ng; idx += WARPS) {
        float v = 1.0f;
        if (args.insc.parts) {
            const int b = idx / ng, q = idx % ng;
            const float* p = args.insc.parts + ((size_t)b * ng + q) * args.insc.per_group;
            float s = 0.0f;
            for (int i = lane; i < args.insc.per_group; i += 32) s += p[i];
            s = warp_sum(s);
            v = rsqrtf(s * args.insc.inv_width + args.insc.eps);
        }
        if (lane == 0) insc_tab[idx] = v;
    }
    uint8_t* act_s = smem + (size_t)WARPS * rg.slots * rg.slot_bytes;
    if (rg.act_smem) {
        const int row16 = args.act_ld / 8;   // 16-byte chunks per row
        for (int idx = threadIdx.x; idx < B * row16; idx += WARPS * 32) {
            const int b = idx / row16, c = idx % row16;
            *reinterpret_cast<uint4*>(act_s + (size_t)b * rg.act_stride + c * 16) =
                *reinterpret_cast<const uint4*>(args.act + (size_t)b * args.act_ld + (size_t)c * 8);
        }
    }
    __syncthreads();

    if (lane == 0 && !rg.act_smem)
        for (int i = 0; i < nstages && i < rg.slots; ++i) issue_act(i, i);

    // ---- accumulation state ---------------------------------------------------------------
    float acc[R][NT][4];
    unsigned long long best[NT][2];
#pragma unroll
    for (int j = 0; j < NT; ++j) best[j][0] = best[j][1] = 0ull;

    auto zero_acc = [&]() {
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int j = 0; j < NT; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[r][j][e] = 0.0f;
    };

    // epilogue of a finished unit (values in v)
    auto epilogue = [&](int u, float (&v)[R][NT][4]) {
        const int row0 = (int)(u * 16 * R);
        if constexpr (EPI == EPI_ARGMAX) {
#pragma unroll
            for (int j = 0; j < NT; ++j)
#pragma unroll
                for (int e2 = 0; e2 < 2; ++e2) {
                    const int b = 8 * j + 2 * t + e2;
                    unsigned long long k = 0ull;
#pragma unroll
                    for (int r = 0; r < R; ++r)
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int row = row0 + 16 * r + g + 8 * h;
                            const float x = v[r][j][2 * h + e2];
                            if (row < M.N && b < B) {
                                if (!isfinite(x)) atomicOr(args.status, VC_DEV_NONFINITE);
                                unsigned long long kk = argmax_key(x, row);
                                k = kk > k ? kk : k;
                                if (args.tap) args.tap[((size_t)m * B + b) * args.tap_ld + row] = x;
                            }
                        }
#pragma unroll
                    for (int o = 4; o < 32; o <<= 1) {
                        unsigned long long kk = __shfl_xor_sync(0xffffffffu, k, o);
                        k = kk > k ? kk : k;
                    }
                    best[j][e2] = k > best[j][e2] ? k : best[j][e2];
                }
        } else if constexpr (EPI == EPI_RESID) {
#pragma unroll
            for (int j = 0; j < NT; ++j)
#pragma unroll
                for (int e2 = 0; e2 < 2; ++e2) {
                    const int b = 8 * j + 2 * t + e2;
                    float ss = 0.0f;
#pragma unroll
                    for (int r = 0; r < R; ++r)
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int row = row0 + 16 * r + g + 8 * h;
                            if (row < M.N && b < B) {
                                float* rp = args.resid + (size_t)b * args.resid_ld + row;
                                const float rn = *rp + v[r][j][2 * h + e2];
                                *rp = rn;
                                ss += rn * rn;
                                const float an = rn * args.gamma_next[row];
                                args.act_next[(size_t)b * args.act_next_ld + row] =
                                    args.act_next_f16 ? act_bits<true>(an) : act_bits<false>(an);
                                if (args.tap) args.tap[(size_t)b * args.tap_ld + row] = rn;
                            }
                        }
#pragma unroll
                    for (int o = 4; o < 32; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
                    if (g == 0 && b < B) args.parts_next[(size_t)b * args.parts_ld + u] = ss;
                }
        } else {
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int j = 0; j < NT; ++j)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int row = row0 + 16 * r + g + 8 * (e >> 1);
                        const int b = 8 * j + 2 * t + (e & 1);
                        if (row >= M.N || b >= B) continue;
                        float x = v[r][j][e];
                        if constexpr (EPI == EPI_RELU2) {
                            x = fmaxf(x, 0.0f);
                            x = x * x;
                        }
                        if constexpr (EPI == EPI_QKV) {
                            const int qrows = args.Hq * args.Dh;
                            if (row < qrows) {
                                args.q_out[(size_t)b * args.q_ld + row] = act_bits<false>(x);
                            } else if (args.ok[b]) {
                                const int rr = row - qrows, kvsel = rr / (args.Hk * args.Dh);
                                const int jj = (rr % (args.Hk * args.Dh)) / args.Dh, d = rr % args.Dh;
                                const int slot = args.slots ? args.slots[b] : b;
                                const int pos = args.ctx_len[slot];
                                uint16_t* cache = kvsel == 0 ? args.kcache : args.vcache;
                                cache[(((size_t)slot * args.Hk + jj) * args.cap + pos) * args.Dh + d] = act_bits<false>(x);
                            }
                        } else {
                            if (args.out)
                                args.out[(size_t)b * args.out_ld + row] = args.out_f16 ? act_bits<true>(x) : act_bits<false>(x);
                            if (args.tap) args.tap[(size_t)b * args.tap_ld + row] = x;
                        }
                    }
        }
    };

    // a unit leaves this worker: finish it here or hand a partial to the last contributor
    auto flush = [&](int u) {
        const long long lo = part_owner((long long)u * M.KT, T, Wm, s32),
                        hi = part_owner((long long)(u + 1) * M.KT - 1, T, Wm, s32);
        if (lo == hi) {
            epilogue(u, acc);
            return;
        }
        if (args.accum) {
            float* au = args.accum + ((size_t)(m ? args.mat[0].NU : 0) + u) * (R * NT * 128);
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int j = 0; j < NT; ++j)
                    red_add_v4(au + ((r * NT + j) * 32 + lane) * 4, acc[r][j][0], acc[r][j][1], acc[r][j][2],
                               acc[r][j][3]);
            __threadfence();
            __syncwarp();
            int old = 0;
            int* cnt = args.counters + (m ? args.mat[0].NU : 0) + u;
            if (lane == 0) old = atomicAdd(cnt, 1);
            old = __shfl_sync(0xffffffffu, old, 0);
            if (old != (int)(hi - lo)) return;
            __threadfence();
            float tot[R][NT][4];
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    float4* p4 = reinterpret_cast<float4*>(au + ((r * NT + j) * 32 + lane) * 4);
                    const float4 v = __ldcg(p4);
                    __stcg(p4, make_float4(0.0f, 0.0f, 0.0f, 0.0f));
                    tot[r][j][0] = v.x; tot[r][j][1] = v.y; tot[r][j][2] = v.z; tot[r][j][3] = v.w;
                }
            if (lane == 0) *cnt = 0;
            epilogue(u, tot);
            return;
        }
        const long long first_u = f0 / M.KT;
        float* mine = args.partials + ((size_t)(wbase + wl) * 2 + (u == first_u ? 0 : 1)) * (R * NT * 128);
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int j = 0; j < NT; ++j)
                *reinterpret_cast<float4*>(mine + ((r * NT + j) * 32 + lane) * 4) =
                    make_float4(acc[r][j][0], acc[r][j][1], acc[r][j][2], acc[r][j][3]);
        __threadfence();
        __syncwarp();
        int old = 0;
        int* cnt = args.counters + (m ? args.mat[0].NU : 0) + u;
        if (lane == 0) old = atomicAdd(cnt, 1);
        old = __shfl_sync(0xffffffffu, old, 0);
        if (old != (int)(hi - lo)) return;
        __threadfence();
        float tot[R][NT][4];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int j = 0; j < NT; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) tot[r][j][e] = 0.0f;
        for (long long w0 = lo; w0 <= hi; w0 += 2) {
            float4 x[2][R * NT];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const long long w2 = w0 + q;
                if (w2 > hi) break;
                const long long fu = part_begin(w2, T, Wm, s32) / M.KT;
                const float* p = args.partials + ((size_t)(wbase + w2) * 2 + (u == fu ? 0 : 1)) * (R * NT * 128);
#pragma unroll
                for (int rj = 0; rj < R * NT; ++rj) x[q][rj] = __ldcg(reinterpret_cast<const float4*>(p + (rj * 32 + lane) * 4));
            }
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                if (w0 + q > hi) break;
#pragma unroll
                for (int r = 0; r < R; ++r)
#pragma unroll
                    for (int j = 0; j < NT; ++j) {
                        const float4 v = x[q][r * NT + j];
                        tot[r][j][0] += v.x; tot[r][j][1] += v.y; tot[r][j][2] += v.z; tot[r][j][3] += v.w;
                    }
            }
        }
        if (lane == 0) *cnt = 0;
        epilogue(u, tot);
    };

    zero_acc();
    bool alive = true;
    int cur_u = f0 / KT, kt = f0 % KT;   // unit and k-step of the next block to consume
    bool pending = false;                 // acc holds contributions of cur_u not yet flushed
    int slot = 0;
    uint32_t phase = 0;
    float sc[NT][2];
    int sc_next = kt;   // first k-step at which sc must be (re)loaded
    for (int i = 0; i < nstages; ++i) {
        if (!mbar_wait(&bar[slot], phase, args.status)) { alive = false; break; }
        const uint8_t* base = ring + (size_t)slot * rg.slot_bytes;
        const int nb = min(bps, f1 - (f0 + i * bps));
        for (int jb = 0; jb < nb; ++jb) {
            const uint8_t* blk = base + jb * L.block_bytes;
            const uint8_t* arow = base + bps * L.block_bytes + (size_t)jb * act_rows * rg.act_row;
            // input scales of this k-step (norm group qg) for the lane's batch columns
            if (kt == sc_next) {
                const int qg = ng > 1 ? (kt * KS) / args.insc.group_cols : 0;
                sc_next = ng > 1 ? min(KT, ((qg + 1) * args.insc.group_cols) / KS) : KT;
#pragma unroll
                for (int j = 0; j < NT; ++j)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int b = 8 * j + 2 * t + e;
                        sc[j][e] = b < B ? insc_tab[b * ng + qg] : 0.0f;
                    }
            }
            // activation B-fragments
            uint32_t bf[SUB][NT][4][2];
#pragma unroll
            for (int st = 0; st < SUB; ++st)
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    const int b = 8 * j + g;
                    uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
                    if (b < B) {
                        const uint8_t* p = rg.act_smem
                            ? act_s + (size_t)b * rg.act_stride + ((size_t)kt * KS + 64 * st + 16 * t) * 2
                            : arow + b * rg.act_row + (64 * st + 16 * t) * 2;
                        v0 = *reinterpret_cast<const uint4*>(p);
                        v1 = *reinterpret_cast<const uint4*>(p + 16);
                    }
                    bf[st][j][0][0] = v0.x; bf[st][j][0][1] = v0.y;
                    bf[st][j][1][0] = v0.z; bf[st][j][1][1] = v0.w;
                    bf[st][j][2][0] = v1.x; bf[st][j][2][1] = v1.y;
                    bf[st][j][3][0] = v1.z; bf[st][j][3][1] = v1.w;
                }
#pragma unroll
            for (int r = 0; r < R; ++r) {
                QConst qc{};
                float s_lo = 1.0f, s_hi = 1.0f;
                if constexpr (FMT != FMT_BF16) {
                    const uint8_t* meta = blk + R * SUB * L.tile_bytes + r * L.meta_bytes;
                    const __half2 sp = *reinterpret_cast<const __half2*>(meta + g * 4);
                    s_lo = __low2float(sp);
                    s_hi = __high2float(sp);
                    if constexpr (FMT == FMT_W4 || FMT == FMT_W3) {
                        const uint32_t zb = meta[32 + g];
                        const uint32_t zl = (zb & 15u) | 0x6400u, zh = (zb >> 4) | 0x6400u;
                        qc.zg = zl | (zl << 16);
                        qc.zh = zh | (zh << 16);
                        qc.f16g = hsub2_u32(h2bits(960.0f), qc.zg);
                        qc.f16h = hsub2_u32(h2bits(960.0f), qc.zh);
                        qc.f8g = hsub2_u32(h2bits(896.0f), qc.zg);
                        qc.f8h = hsub2_u32(h2bits(896.0f), qc.zh);
                        qc.f64g = hsub2_u32(h2bits(1008.0f), qc.zg);
                        qc.f64h = hsub2_u32(h2bits(1008.0f), qc.zh);
                    }
                }
                float c[NT][4];
#pragma unroll
                for (int j = 0; j < NT; ++j) c[j][0] = c[j][1] = c[j][2] = c[j][3] = 0.0f;
#pragma unroll
                for (int st = 0; st < SUB; ++st) {
                    uint32_t a[4][4];
                    load_tile_frags<FMT>(blk + (r * SUB + st) * L.tile_bytes, lane, qc, a);
#pragma unroll
                    for (int s = 0; s < 4; ++s)
#pragma unroll
                        for (int j = 0; j < NT; ++j) mma_step<FMT>(c[j], a[s], bf[st][j][s][0], bf[st][j][s][1]);
                }
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    acc[r][j][0] = fmaf(s_lo * sc[j][0], c[j][0], acc[r][j][0]);
                    acc[r][j][1] = fmaf(s_lo * sc[j][1], c[j][1], acc[r][j][1]);
                    acc[r][j][2] = fmaf(s_hi * sc[j][0], c[j][2], acc[r][j][2]);
                    acc[r][j][3] = fmaf(s_hi * sc[j][1], c[j][3], acc[r][j][3]);
                }
            }
            pending = true;
            if (++kt == KT) {   // the unit's last k-step: finish it (or hand over the partial)
                flush(cur_u);
                zero_acc();
                pending = false;
                kt = 0;
                ++cur_u;
                if (ng > 1) sc_next = 0;
            }
        }
        __syncwarp();
        if (lane == 0 && i + rg.slots < nstages) {
            fence_proxy_async();
            issue_weights(i + rg.slots, slot);
            if (!rg.act_smem) issue_act(i + rg.slots, slot);
        }
        if (++slot == rg.slots) { slot = 0; phase ^= 1u; }
    }
    if (alive && pending) flush(cur_u);

    if constexpr (EPI == EPI_ARGMAX) {
        // publish this worker's best keys, then the last worker of the launch emits the tokens
        if (g == 0) {
#pragma unroll
            for (int j = 0; j < NT; ++j)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int b = 8 * j + 2 * t + e;
                    if (b < B && best[j][e]) atomicMax(&args.keys[m * kMaxB + b], best[j][e]);
                }
        }
        __threadfence();
        __syncwarp();
        int old = 0;
        if (lane == 0) old = atomicAdd(args.done, 1);
        old = __shfl_sync(0xffffffffu, old, 0);
        if (old == (int)Wall - 1) {
            __threadfence();
            if (lane < B) {
                const int b = lane;
                const int slot = args.slots ? args.slots[b] : b;
                const bool okb = args.ok[b] != 0;
                for (int mm = 0; mm < args.nmat; ++mm) {
                    const unsigned long long k = atomicExch(&args.keys[mm * kMaxB + b], 0ull);
                    args.tok[mm][b] = okb ? argmax_key_index(k) : -1;
                }
                if (okb && args.ctx_len_mut) args.ctx_len_mut[slot] += 1;
            }
            if (lane == 0) *args.done = 0;
        }
    }
}

template <int FMT, int GRP, int NT, int EPI>
cudaError_t launch_t(const GemvLaunch& Lh, const GemvArgs& a, cudaStream_t s) {
    constexpr LayoutInfo L = layout_info(FMT, GRP);
    RingGeom rg{};
    rg.act_row = L.KS * 2 + 16;
    rg.act_stride = a.act_ld * 2 + 16;
    const int act_total = a.B * rg.act_stride;
    rg.act_smem = act_total <= 32 * 1024;
    const int wbytes = L.bps * L.block_bytes;
    rg.slot_bytes = round_up(wbytes + (rg.act_smem ? 0 : L.bps * a.B * rg.act_row), 128);
    // as many 4 KB-class slots per warp as the budget allows: the bytes in flight per SM
    // (warps x (slots - 1) x slot) must cover HBM latency x per-SM bandwidth (~60-100 KB)
    constexpr int WARPS = warps_for(NT);
    const int budget = kRingBudget / ctas_per_sm(NT) - 4096;   // two CTAs must fit one SM
    rg.slots = (budget - (rg.act_smem ? act_total : 0)) / (WARPS * rg.slot_bytes);
    if (rg.slots > kMaxSlots) rg.slots = kMaxSlots;
    if (rg.slots < 2) rg.slots = 2;
    const size_t smem = (size_t)WARPS * rg.slots * rg.slot_bytes + (rg.act_smem ? act_total : 0);
    if (smem > 220 * 1024) return cudaErrorInvalidValue;
    auto kern = gemv_kernel<FMT, GRP, NT, EPI>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(Lh.num_sms * ctas_per_sm(NT));
    cfg.blockDim = dim3(WARPS * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = Lh.pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a, rg);
}

template <int FMT, int GRP, int NT>
cudaError_t launch_epi(const GemvLaunch& L, const GemvArgs& a, cudaStream_t s) {
    switch (L.epi) {
        case EPI_STORE: return launch_t<FMT, GRP, NT, EPI_STORE>(L, a, s);
        case EPI_RELU2: return launch_t<FMT, GRP, NT, EPI_RELU2>(L, a, s);
        case EPI_RESID: return launch_t<FMT, GRP, NT, EPI_RESID>(L, a, s);
        case EPI_QKV: return launch_t<FMT, GRP, NT, EPI_QKV>(L, a, s);
        case EPI_ARGMAX: return launch_t<FMT, GRP, NT, EPI_ARGMAX>(L, a, s);
    }
    return cudaErrorInvalidValue;
}

template <int FMT, int GRP>
cudaError_t launch_nt(const GemvLaunch& L, const GemvArgs& a, cudaStream_t s) {
    if (a.B <= 8) return launch_epi<FMT, GRP, 1>(L, a, s);
    return launch_epi<FMT, GRP, 2>(L, a, s);
}

cudaError_t launch_gemv_bf16(const GemvLaunch& L, const GemvArgs& a, cudaStream_t s);
cudaError_t launch_gemv_w8(const GemvLaunch& L, const GemvArgs& a, cudaStream_t s);
cudaError_t launch_gemv_w4(const GemvLaunch& L, const GemvArgs& a, cudaStream_t s);
cudaError_t launch_gemv_w3(const GemvLaunch& L, const GemvArgs& a, cudaStream_t s);

}  // namespace vc
