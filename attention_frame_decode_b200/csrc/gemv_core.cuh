// gemv_core.cuh -- the per-warp building blocks of the streaming weight GEMV (y = W u for
// B <= 16 activation rows), shared by the standalone GEMV kernel (gemv_kernel.cuh) and the
// persistent frame kernel (frame_kernel.cuh).
//
// A matrix in the device layout (layout.cuh) is a sequence of T = NU * KT blocks (unit u of 16R
// rows, k-step kt); the warps of a launch split that sequence into equal contiguous ranges
// (worker w of W owns blocks [w T / W, (w+1) T / W)).  A warp walks its range block by block:
//   * the A fragments of a 16x64 tile are formed in registers (bf16 as stored; W8/W4/W3 the exact
//     fp16 values q - z by the exponent-field trick: OR a code into the mantissa of 1024.0 and
//     subtract 1024 + z) and multiplied on mma.sync m16n8k16 with fp32 accumulation; the fp32
//     group sums are scaled by the group's fp16 scale and by the input scale of the activation row;
//   * a unit whose k-steps all belong to this warp is finished here (fused epilogue); a unit cut
//     between warps is finished by its last contributor (atomic counter), which adds the others'
//     contributions: with an accumulator area through fp32 vector reductions (summation order
//     varies between runs), without one from the contributors' partials in worker order.
#pragma once
#include "common.cuh"
#include "gemv.cuh"
#include "layout.cuh"

namespace vc {

static constexpr int kWarps = 16;   // upper bound of warps per CTA (sizes the partial-sum scratch)

// the 16-bit type of the activations a weight format multiplies: bf16 (the values the step stores)
// for bf16 weights, fp16 (the same values widened, exact in fp16's normal range) for the quantized
// formats, whose dequantized codes are fp16
__host__ __device__ constexpr bool act_f16_for(int fmt) { return fmt != 0; }
static constexpr int kMaxB = 16;
static constexpr int kMaxSlots = 8;  // ring slots per warp (upper bound)

// ------------------------------------------------------------------------------------------
// partition helpers (worker w of W owns flat blocks [w*T/W, (w+1)*T/W))
// ------------------------------------------------------------------------------------------
// With T (W + 1) < 2^32 (every shape of the backbone) the same integer quotients are taken in
// 32-bit arithmetic, which costs a fraction of a 64-bit division.
__host__ __device__ __forceinline__ long long part_begin(long long w, long long T, long long W, bool s32) {
    if (s32) return (long long)((uint32_t)w * (uint32_t)T / (uint32_t)W);
    return w * T / W;
}
// largest worker whose range starts at or before block f (always a non-empty range)
__host__ __device__ __forceinline__ long long part_owner(long long f, long long T, long long W, bool s32) {
    if (s32) return (long long)(((uint32_t)(f + 1) * (uint32_t)W + (uint32_t)T - 1u) / (uint32_t)T) - 1;
    return ((f + 1) * W + T - 1) / T - 1;
}

// one warp's share of one matrix of a launch (two matrices split the warps in halves)
struct WarpRange {
    GemvMat M;
    int m;                 // matrix index within the launch
    long long T, Wm, wl, wbase;
    bool s32, idle;
    int f0, f1;            // block range [f0, f1)
};

__host__ __device__ __forceinline__ WarpRange warp_range(const GemvMat (&mat)[2], int nmat, long long wid, long long Wall) {
    WarpRange r;
    r.m = 0;
    r.Wm = Wall;
    r.wl = wid;
    r.wbase = 0;
    if (nmat == 2) {
        const long long W0 = Wall / 2;
        if (wid >= W0) { r.m = 1; r.wl = wid - W0; r.Wm = Wall - W0; r.wbase = W0; }
        else r.Wm = W0;
    }
    r.M = mat[r.m];
    r.T = (long long)r.M.NU * r.M.KT;
    // with fewer blocks than warps only the first T workers get (one-block) ranges, so that every
    // worker between the first and last contributor of a unit is a contributor
    if (r.Wm > r.T) r.Wm = r.T;
    r.idle = r.wl >= r.Wm;
    r.s32 = (unsigned long long)r.T * (unsigned long long)(r.Wm + 1) < (1ull << 32);
    r.f0 = r.idle ? 0 : (int)part_begin(r.wl, r.T, r.Wm, r.s32);
    r.f1 = r.idle ? 0 : (int)part_begin(r.wl + 1, r.T, r.Wm, r.s32);
    return r;
}

// ------------------------------------------------------------------------------------------
// A fragments of the weight tiles
// ------------------------------------------------------------------------------------------
struct QConst {            // W4 / W3 dequantization constants of a slab (fp16 pairs)
    uint32_t zg, zh;       // (1024 + z) pairs, rows g and g+8
    uint32_t f16h;         // -(64 + z), row g+8  (W4 high nibble)
    uint32_t f8g, f8h;     // -(128 + z)          (W3 fields 1, 4)
    uint32_t f64g, f64h;   // -(16 + z)           (W3 field 2)
};

__device__ __forceinline__ uint32_t h2bits(float v) {
    __half h = __float2half_rn(v);
    uint16_t b = *reinterpret_cast<uint16_t*>(&h);
    return (uint32_t)b | ((uint32_t)b << 16);
}

template <int FMT>
__device__ __forceinline__ void mma_step(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    if constexpr (!act_f16_for(FMT)) mma_bf16(d, a, b0, b1);
    else mma_f16(d, a, b0, b1);
}

// ------------------------------------------------------------------------------------------
// one block: acc[r][j] += scale * (slab r of the block) . (activation k-step, column tile j)
//   bv[st][j]: the lane's two 16-byte pieces of activation row 8j + g (columns 64 st + 16 t ..
//              64 st + 16 t + 15 of the k-step; zero for rows >= B)
//   sc[j][e]:  input scale of batch column 8j + 2t + e for this k-step
// ------------------------------------------------------------------------------------------
// The raw 32-bit words of one lane's share of a 16x64 tile, and the A fragments of k16 step s
// computed from them: bf16 as stored; W8, W4 and W3 the exact fp16 values q - z by the
// exponent-field trick (OR a code into the mantissa of 1024.0, subtract 1024 + z).
template <int FMT>
struct TileWords {
    static constexpr int n = FMT == FMT_BF16 ? 16 : FMT == FMT_W8 ? 8 : FMT == FMT_W4 ? 4 : 3;
    uint32_t w[n];
};

template <int FMT>
__device__ __forceinline__ void load_tile_words(const uint8_t* tile, int lane, TileWords<FMT>& tw) {
    if constexpr (FMT == FMT_BF16) {
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const uint4 v = *reinterpret_cast<const uint4*>(tile + (s * 32 + lane) * 16);
            tw.w[4 * s] = v.x; tw.w[4 * s + 1] = v.y; tw.w[4 * s + 2] = v.z; tw.w[4 * s + 3] = v.w;
        }
    } else if constexpr (FMT == FMT_W8) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const uint4 v = *reinterpret_cast<const uint4*>(tile + (c * 32 + lane) * 16);
            tw.w[4 * c] = v.x; tw.w[4 * c + 1] = v.y; tw.w[4 * c + 2] = v.z; tw.w[4 * c + 3] = v.w;
        }
    } else if constexpr (FMT == FMT_W4) {
        const uint4 v = *reinterpret_cast<const uint4*>(tile + lane * 16);
        tw.w[0] = v.x; tw.w[1] = v.y; tw.w[2] = v.z; tw.w[3] = v.w;
    } else {
        const uint2 v01 = *reinterpret_cast<const uint2*>(tile + lane * 8);
        tw.w[0] = v01.x; tw.w[1] = v01.y;
        tw.w[2] = *reinterpret_cast<const uint32_t*>(tile + 256 + lane * 4);
    }
}

template <int FMT>
__device__ __forceinline__ void step_frags(const TileWords<FMT>& tw, int s, const QConst& qc, uint32_t (&a)[4]) {
    const uint32_t M = 0x64006400u;
    if constexpr (FMT == FMT_BF16) {
        a[0] = tw.w[4 * s]; a[1] = tw.w[4 * s + 1]; a[2] = tw.w[4 * s + 2]; a[3] = tw.w[4 * s + 3];
    } else if constexpr (FMT == FMT_W8) {
        const uint32_t K1152 = 0x64806480u;   // 1024 + 128 as an fp16 pair
        const uint32_t M8 = 0x64646464u;      // prmt source of the 0x64 exponent byte
        const int c = s >> 1, h = s & 1;
        const uint32_t A = tw.w[4 * c + 2 * h], B = tw.w[4 * c + 2 * h + 1];
        a[0] = hsub2_u32(prmt(A, M8, 0x4240), K1152);
        a[1] = hsub2_u32(prmt(B, M8, 0x4240), K1152);
        a[2] = hsub2_u32(prmt(A, M8, 0x4341), K1152);
        a[3] = hsub2_u32(prmt(B, M8, 0x4341), K1152);
    } else if constexpr (FMT == FMT_W4) {
        // row g: the low nibble, 1024 + q - (1024 + z); row g+8: the nibble above it, read as
        // 1024 + 16 q, times 1/16 minus (64 + z).  Both exact in fp16.
        const uint32_t R16 = h2bits(1.0f / 16.0f);
        const uint32_t x = tw.w[s], y = tw.w[s] >> 8;
        a[0] = hsub2_u32(and_or(x, 0x000F000Fu, M), qc.zg);
        a[1] = hfma2_u32(and_or(x, 0x00F000F0u, M), R16, qc.f16h);
        a[2] = hsub2_u32(and_or(y, 0x000F000Fu, M), qc.zg);
        a[3] = hfma2_u32(and_or(y, 0x00F000F0u, M), R16, qc.f16h);
    } else {  // W3: pair p = 4s + reg
        const uint32_t R8 = h2bits(1.0f / 8.0f), R64 = h2bits(1.0f / 64.0f);
#pragma unroll
        for (int reg = 0; reg < 4; ++reg) {
            const int p = 4 * s + reg;
            const bool hi = reg & 1;
            const uint32_t z = hi ? qc.zh : qc.zg, f8 = hi ? qc.f8h : qc.f8g, f64 = hi ? qc.f64h : qc.f64g;
            uint32_t r;
            if (p < 15) {
                const uint32_t x = tw.w[p / 5];
                const int i = p % 5;
                if (i == 0) r = hsub2_u32(and_or(x, 0x00070007u, M), z);
                else if (i == 1) r = hfma2_u32(and_or(x, 0x00380038u, M), R8, f8);
                else if (i == 2) r = hfma2_u32(and_or(x, 0x01C001C0u, M), R64, f64);
                else if (i == 3) r = hsub2_u32(and_or(x >> 9, 0x00070007u, M), z);
                else r = hfma2_u32(and_or(x >> 9, 0x00380038u, M), R8, f8);
            } else {
                const uint32_t c = ((tw.w[0] >> 15) & 0x00010001u) | ((tw.w[1] >> 14) & 0x00020002u) |
                                   ((tw.w[2] >> 13) & 0x00040004u);
                r = hsub2_u32(c | M, z);
            }
            a[reg] = r;
        }
    }
}

// W8 and W4 with the zero point deferred: the A fragments hold the codes read as fp16 1024 + code
// (W8: one prmt per register; W4: one lop3, the nibble of row g+8 read as 1024 + 16 q), so the
// products are sum (1024 + code) u; the group's activation sum U = sum u, produced by an MMA of
// the same activation fragments with an all-ones A, removes the offset once per group:
//   W8 (stored q + 128):  sum q u = c - 1152 U
//   W4 row g:             sum (q - z) u = c - (1024 + z) U
//   W4 row g+8:           sum (q - z) u = c / 16 - (64 + z) U
// Products of fp16 values are exact and summed in fp32; the offset sums are ~10^3 x the result
// at most, which leaves ~1e-4 relative error per group sum.  SYM (the vocabulary heads, whose
// greedy argmax must see equal rows as equal): both rows of a slab are read at scale 1 (two more
// shifts per word), so two rows holding the same codes give the same sums bit for bit.
template <int FMT>
__host__ __device__ constexpr bool deferred_zero() { return FMT == FMT_W8 || FMT == FMT_W4; }

template <int FMT, bool SYM>
__device__ __forceinline__ void step_frags_raw(const TileWords<FMT>& tw, int s, uint32_t (&a)[4]) {
    if constexpr (FMT == FMT_W8) {
        const uint32_t M8 = 0x64646464u;      // prmt source of the 0x64 exponent byte
        const int c = s >> 1, h = s & 1;
        const uint32_t A = tw.w[4 * c + 2 * h], B = tw.w[4 * c + 2 * h + 1];
        a[0] = prmt(A, M8, 0x4240);
        a[1] = prmt(B, M8, 0x4240);
        a[2] = prmt(A, M8, 0x4341);
        a[3] = prmt(B, M8, 0x4341);
    } else if constexpr (SYM) {
        const uint32_t M = 0x64006400u;
        const uint32_t x = tw.w[s];
        a[0] = and_or(x, 0x000F000Fu, M);
        a[1] = and_or(x >> 4, 0x000F000Fu, M);
        a[2] = and_or(x >> 8, 0x000F000Fu, M);
        a[3] = and_or(x >> 12, 0x000F000Fu, M);
    } else {
        const uint32_t M = 0x64006400u;
        const uint32_t x = tw.w[s], y = tw.w[s] >> 8;
        a[0] = and_or(x, 0x000F000Fu, M);
        a[1] = and_or(x, 0x00F000F0u, M);
        a[2] = and_or(y, 0x000F000Fu, M);
        a[3] = and_or(y, 0x00F000F0u, M);
    }
}

// exact float of a small non-negative integer n < 2^23 (bits OR-ed into 2^23, minus 2^23)
__device__ __forceinline__ float small_int_f(uint32_t n) { return __uint_as_float(0x4B000000u | n) - 8388608.0f; }

// one block: acc[r][j] += scale * (slab r of the block) . (activation k-step, column tile j)
//   bv[st][j]: the lane's two 16-byte pieces of activation row 8j + g (columns 64 st + 16 t ..
//              64 st + 16 t + 15 of the k-step; zero for rows >= B)
//   sc[j][e]:  input scale of batch column 8j + 2t + e for this k-step
//   col1:      the odd batch columns 2t + 1 are used (B > 1); when false their sums are not formed
// All tiles' words and slab metadata are loaded first; then each k16 step dequantizes one
// register quad per slab and issues the slabs' MMAs back to back, so the R accumulation chains
// interleave instead of running one after another.
template <int FMT, int GRP, int NT, bool SYM>
__device__ __forceinline__ void consume_block_dz(const uint8_t* blk, const uint4 (&bv)[layout_info(FMT, GRP).SUB][NT][2],
                                                 int lane, const float (&sc)[NT][2],
                                                 float (&acc)[layout_info(FMT, GRP).R][NT][4], bool col1) {
    constexpr LayoutInfo L = layout_info(FMT, GRP);
    constexpr int R = L.R, SUB = L.SUB;
    const int g = lane >> 2;
    TileWords<FMT> tw[R][SUB];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int st = 0; st < SUB; ++st) load_tile_words<FMT>(blk + (r * SUB + st) * L.tile_bytes, lane, tw[r][st]);
    float c[R][NT][4], cu[NT][4];
#pragma unroll
    for (int j = 0; j < NT; ++j) {
        cu[j][0] = cu[j][1] = cu[j][2] = cu[j][3] = 0.0f;
#pragma unroll
        for (int r = 0; r < R; ++r) c[r][j][0] = c[r][j][1] = c[r][j][2] = c[r][j][3] = 0.0f;
    }
    const uint32_t ones[4] = {0x3C003C00u, 0x3C003C00u, 0x3C003C00u, 0x3C003C00u};   // fp16 1.0 pairs
#pragma unroll
    for (int st = 0; st < SUB; ++st)
#pragma unroll
        for (int s = 0; s < 4; ++s) {
#pragma unroll
            for (int j = 0; j < NT; ++j) {
                const uint4& v = bv[st][j][s >> 1];
                mma_f16(cu[j], ones, (s & 1) ? v.z : v.x, (s & 1) ? v.w : v.y);
            }
#pragma unroll
            for (int r = 0; r < R; ++r) {
                uint32_t a[4];
                step_frags_raw<FMT, SYM>(tw[r][st], s, a);
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    const uint4& v = bv[st][j][s >> 1];
                    mma_f16(c[r][j], a, (s & 1) ? v.z : v.x, (s & 1) ? v.w : v.y);
                }
            }
        }
    // slab metadata (scales; W4 zeros) read after the products, so its registers are not live
    // across them
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const uint8_t* meta = blk + R * SUB * L.tile_bytes + r * L.meta_bytes;
        const __half2 sp = *reinterpret_cast<const __half2*>(meta + g * 4);
        const float s_lo = __low2float(sp), s_hi = __high2float(sp);
        float zl = 1152.0f, zh = 1152.0f;
        if constexpr (FMT == FMT_W4) {
            const uint32_t zb = meta[32 + g];
            zl = small_int_f(1024u + (zb & 15u));
            zh = small_int_f((SYM ? 1024u : 64u) + (zb >> 4));
        }
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            float v0, v2;
            if constexpr (FMT == FMT_W4 && SYM) {
                v0 = fmaf(-zl, cu[j][0], c[r][j][0]);
                v2 = fmaf(-zh, cu[j][0], c[r][j][2]);
            } else if constexpr (FMT == FMT_W4) {
                v0 = fmaf(-zl, cu[j][0], c[r][j][0]);
                v2 = fmaf(c[r][j][2], 0.0625f, -zh * cu[j][0]);
            } else {
                v0 = fmaf(-1152.0f, cu[j][0], c[r][j][0]);
                v2 = fmaf(-1152.0f, cu[j][0], c[r][j][2]);
            }
            acc[r][j][0] = fmaf(s_lo * sc[j][0], v0, acc[r][j][0]);
            acc[r][j][2] = fmaf(s_hi * sc[j][0], v2, acc[r][j][2]);
            if (NT > 1 || col1) {
                float v1, v3;
                if constexpr (FMT == FMT_W4 && SYM) {
                    v1 = fmaf(-zl, cu[j][1], c[r][j][1]);
                    v3 = fmaf(-zh, cu[j][1], c[r][j][3]);
                } else if constexpr (FMT == FMT_W4) {
                    v1 = fmaf(-zl, cu[j][1], c[r][j][1]);
                    v3 = fmaf(c[r][j][3], 0.0625f, -zh * cu[j][1]);
                } else {
                    v1 = fmaf(-1152.0f, cu[j][1], c[r][j][1]);
                    v3 = fmaf(-1152.0f, cu[j][1], c[r][j][3]);
                }
                acc[r][j][1] = fmaf(s_lo * sc[j][1], v1, acc[r][j][1]);
                acc[r][j][3] = fmaf(s_hi * sc[j][1], v3, acc[r][j][3]);
            }
        }
    }
}

template <int FMT, int GRP, int NT>
__device__ __forceinline__ void consume_block_bv(const uint8_t* blk, const uint4 (&bv)[layout_info(FMT, GRP).SUB][NT][2],
                                                 int lane, const float (&sc)[NT][2],
                                                 float (&acc)[layout_info(FMT, GRP).R][NT][4], bool col1 = true,
                                                 bool sym = false) {
    if constexpr (deferred_zero<FMT>()) {
        if (FMT == FMT_W4 && sym) consume_block_dz<FMT, GRP, NT, true>(blk, bv, lane, sc, acc, col1);
        else consume_block_dz<FMT, GRP, NT, false>(blk, bv, lane, sc, acc, col1);
        return;
    }
    constexpr LayoutInfo L = layout_info(FMT, GRP);
    constexpr int R = L.R, SUB = L.SUB;
    const int g = lane >> 2;
    TileWords<FMT> tw[R][SUB];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int st = 0; st < SUB; ++st) load_tile_words<FMT>(blk + (r * SUB + st) * L.tile_bytes, lane, tw[r][st]);
    QConst qc[R];
    float s_lo[R], s_hi[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        qc[r] = QConst{};
        s_lo[r] = s_hi[r] = 1.0f;
        if constexpr (FMT != FMT_BF16) {
            const uint8_t* meta = blk + R * SUB * L.tile_bytes + r * L.meta_bytes;
            const __half2 sp = *reinterpret_cast<const __half2*>(meta + g * 4);
            s_lo[r] = __low2float(sp);
            s_hi[r] = __high2float(sp);
            if constexpr (FMT == FMT_W4 || FMT == FMT_W3) {
                const uint32_t zb = meta[32 + g];
                const uint32_t zl = (zb & 15u) | 0x6400u, zh = (zb >> 4) | 0x6400u;
                qc[r].zg = zl | (zl << 16);
                qc[r].zh = zh | (zh << 16);
                qc[r].f16h = hsub2_u32(h2bits(960.0f), qc[r].zh);
                qc[r].f8g = hsub2_u32(h2bits(896.0f), qc[r].zg);
                qc[r].f8h = hsub2_u32(h2bits(896.0f), qc[r].zh);
                qc[r].f64g = hsub2_u32(h2bits(1008.0f), qc[r].zg);
                qc[r].f64h = hsub2_u32(h2bits(1008.0f), qc[r].zh);
            }
        }
    }
    float c[R][NT][4];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int j = 0; j < NT; ++j) c[r][j][0] = c[r][j][1] = c[r][j][2] = c[r][j][3] = 0.0f;
#pragma unroll
    for (int st = 0; st < SUB; ++st)
#pragma unroll
        for (int s = 0; s < 4; ++s)
#pragma unroll
            for (int r = 0; r < R; ++r) {
                uint32_t a[4];
                step_frags<FMT>(tw[r][st], s, qc[r], a);
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    const uint4& v = bv[st][j][s >> 1];
                    mma_step<FMT>(c[r][j], a, (s & 1) ? v.z : v.x, (s & 1) ? v.w : v.y);
                }
            }
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            acc[r][j][0] = fmaf(s_lo[r] * sc[j][0], c[r][j][0], acc[r][j][0]);
            acc[r][j][1] = fmaf(s_lo[r] * sc[j][1], c[r][j][1], acc[r][j][1]);
            acc[r][j][2] = fmaf(s_hi[r] * sc[j][0], c[r][j][2], acc[r][j][2]);
            acc[r][j][3] = fmaf(s_hi[r] * sc[j][1], c[r][j][3], acc[r][j][3]);
        }
}

//   arow(b): byte address of activation row b's 64-column slice st = 0 of this k-step
// Columns b >= B read row B-1 instead of zeros: their sums are computed and never stored (every
// epilogue checks b < B), and the loads need no branch.
template <int FMT, int GRP, int NT, bool SYM = false, typename ActRow>
__device__ __forceinline__ void consume_block(const uint8_t* blk, ActRow arow, int B, int lane, const float (&sc)[NT][2],
                                              float (&acc)[layout_info(FMT, GRP).R][NT][4]) {
    constexpr int SUB = layout_info(FMT, GRP).SUB;
    const int g = lane >> 2, t = lane & 3;
    uint4 bv[SUB][NT][2];
#pragma unroll
    for (int st = 0; st < SUB; ++st)
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            const int b = min(8 * j + g, B - 1);
            const uint8_t* p = arow(b) + (64 * st + 16 * t) * 2;
            bv[st][j][0] = *reinterpret_cast<const uint4*>(p);
            bv[st][j][1] = *reinterpret_cast<const uint4*>(p + 16);
        }
    consume_block_bv<FMT, GRP, NT>(blk, bv, lane, sc, acc, B > 1, SYM);
}

// the same with the k-step's activation staged as SUB boxes (box st at box0 + st * box_bytes) of
// B rows x 64 columns, 128 B per row with the 128-byte swizzle: 16-byte chunk c of row b sits at
// chunk c ^ (b & 7)
template <int FMT, int GRP, int NT, bool SYM = false>
__device__ __forceinline__ void consume_block_swz(const uint8_t* blk, const uint8_t* box0, int box_bytes, int B, int lane,
                                                  const float (&sc)[NT][2],
                                                  float (&acc)[layout_info(FMT, GRP).R][NT][4]) {
    constexpr int SUB = layout_info(FMT, GRP).SUB;
    const int g = lane >> 2, t = lane & 3;
    uint4 bv[SUB][NT][2];
#pragma unroll
    for (int st = 0; st < SUB; ++st)
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            const int b = min(8 * j + g, B - 1);
            const uint8_t* row = box0 + st * box_bytes + b * 128;
            bv[st][j][0] = *reinterpret_cast<const uint4*>(row + (((2 * t) ^ (b & 7)) << 4));
            bv[st][j][1] = *reinterpret_cast<const uint4*>(row + (((2 * t + 1) ^ (b & 7)) << 4));
        }
    consume_block_bv<FMT, GRP, NT>(blk, bv, lane, sc, acc, B > 1, SYM);
}

// ------------------------------------------------------------------------------------------
// epilogue of a finished unit u (values v) of matrix wr.m of the launch
// ------------------------------------------------------------------------------------------
template <int FMT, int GRP, int NT, int EPI>
__device__ __forceinline__ void unit_epilogue(const GemvArgs& args, const WarpRange& wr, int u,
                                              float (&v)[layout_info(FMT, GRP).R][NT][4],
                                              unsigned long long (&best)[NT][2], int lane) {
    constexpr int R = layout_info(FMT, GRP).R;
    const int g = lane >> 2, t = lane & 3;
    const int B = args.B;
    const GemvMat& M = wr.M;
    const int m = wr.m;
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
}

// ------------------------------------------------------------------------------------------
// a unit leaves this warp: finish it here or hand a partial to its last contributor
// ------------------------------------------------------------------------------------------
// ACCUM_ONLY: the launch always provides the accumulator area (the partials path is not compiled)
template <int FMT, int GRP, int NT, int EPI, bool ACCUM_ONLY = false>
__device__ __forceinline__ void unit_flush(const GemvArgs& args, const WarpRange& wr, int u,
                                           float (&acc)[layout_info(FMT, GRP).R][NT][4],
                                           unsigned long long (&best)[NT][2], int lane) {
    constexpr int R = layout_info(FMT, GRP).R;
    const long long lo = part_owner((long long)u * wr.M.KT, wr.T, wr.Wm, wr.s32),
                    hi = part_owner((long long)(u + 1) * wr.M.KT - 1, wr.T, wr.Wm, wr.s32);
    if (lo == hi) {
        unit_epilogue<FMT, GRP, NT, EPI>(args, wr, u, acc, best, lane);
        return;
    }
    const size_t ubase = (size_t)(wr.m ? args.mat[0].NU : 0) + u;
    int* cnt = args.counters + ubase;
    if (ACCUM_ONLY || args.accum) {
        float* au = args.accum + ubase * (R * NT * 128);
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int j = 0; j < NT; ++j)
                red_add_v4(au + ((r * NT + j) * 32 + lane) * 4, acc[r][j][0], acc[r][j][1], acc[r][j][2],
                           acc[r][j][3]);
        __threadfence();
        __syncwarp();
        int old = 0;
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
        unit_epilogue<FMT, GRP, NT, EPI>(args, wr, u, tot, best, lane);
        return;
    }
    if constexpr (ACCUM_ONLY) return;
    const long long first_u = wr.f0 / wr.M.KT;
    float* mine = args.partials + ((size_t)(wr.wbase + wr.wl) * 2 + (u == first_u ? 0 : 1)) * (R * NT * 128);
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int j = 0; j < NT; ++j)
            *reinterpret_cast<float4*>(mine + ((r * NT + j) * 32 + lane) * 4) =
                make_float4(acc[r][j][0], acc[r][j][1], acc[r][j][2], acc[r][j][3]);
    __threadfence();
    __syncwarp();
    int old = 0;
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
            const long long fu = part_begin(w2, wr.T, wr.Wm, wr.s32) / wr.M.KT;
            const float* p = args.partials + ((size_t)(wr.wbase + w2) * 2 + (u == fu ? 0 : 1)) * (R * NT * 128);
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
    unit_epilogue<FMT, GRP, NT, EPI>(args, wr, u, tot, best, lane);
}

// ------------------------------------------------------------------------------------------
// greedy heads: publish a warp's best keys; the last warp of all Wall emits the tokens and
// advances the sessions' frame counters
// ------------------------------------------------------------------------------------------
template <int NT>
__device__ __forceinline__ void argmax_publish(const GemvArgs& args, int m, const unsigned long long (&best)[NT][2],
                                               long long Wall, int lane) {
    const int g = lane >> 2, t = lane & 3;
    const int B = args.B;
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

}  // namespace vc
