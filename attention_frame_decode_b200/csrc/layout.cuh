// layout.cuh -- device storage layout of a linear weight W[N][K] for the streaming GEMV.
//
// The matrix is cut into units of 16*R rows and k-steps of KS = max(64, group) columns.
// A "block" (unit u, k-step kt) holds R*SUB tiles of 16 rows x 64 columns (SUB = KS/64)
// followed by one metadata record per 16-row slab (its fp16 scales and, for W4 and W3, its
// zeros in 4-bit fields, for this k-step's quantization group).  Blocks are stored
// unit-major, k-step-minor:
//       offset(u, kt) = (u * KT + kt) * block_bytes
// so any contiguous range of the flattened (u, kt) index is one contiguous byte range:
// a warp streams its share of the matrix with 1-D bulk copies and no gather.
//
// Inside a tile, lane (g = lane/4, t = lane%4) owns rows g and g+8, columns 16t..16t+15,
// i.e. exactly the mma.m16n8k16 A-fragment registers it needs for the four k16 steps of
// the tile (k-slot -> column map: step s, slot pair (2t,2t+1) -> columns 16t+4s+{0,1},
// slot pair (2t+8,2t+9) -> columns 16t+4s+{2,3}); the activation B-fragments use the same
// map, so the product is unchanged.  Per lane and step the four A registers are
//   reg0 = (row g,   c0 c1)  reg1 = (row g+8, c0 c1)  reg2 = (row g, c2 c3)  reg3 = (row g+8, c2 c3)
// with cX = 16t + 4s + X.  Formats:
//   BF16: 64 B / lane: [step s][lane][16 B] = the four registers as bf16 pairs.
//   W8  : 32 B / lane: [s/2][lane][16 B]; per step a word for row g and one for row g+8, bytes
//         (c0, c2, c1, c3), stored offset-binary (q + 128).  prmt + one fp16 subtract give q.
//   W4  : 16 B / lane: [lane][word s]; nibble (reg) holds the first column of register reg,
//         nibble (reg + 4) the second: two lop3 masks + the fp16 exponent trick give q - z.
//   W3  : 12 B / lane: [lane][w0 w1] then [lane][w2]; 16 register pairs p = 4s + reg; pair p < 15
//         lives in word p/5 field p%5 (3-bit fields at bits 3i and 16+3i), pair 15 in bits 15 and
//         31 of the three words (bit b of its codes in word b).
// Metadata per 16-row slab: scales as 8 fp16 pairs (s_g, s_g+8), then (W4/W3) 8 bytes of zero
// pairs (z_g | z_g+8 << 4).  Rows >= N and columns >= K are zero weights.
#pragma once
#include <stdint.h>

namespace vc {

enum Fmt : int { FMT_BF16 = 0, FMT_W8 = 1, FMT_W4 = 2, FMT_W3 = 3 };

struct LayoutInfo {
    int R, KS, SUB, lane_bytes, tile_bytes, meta_bytes, block_bytes, bps, bits;
};

__host__ __device__ constexpr int round_up(int a, int b) { return (a + b - 1) / b * b; }

__host__ __device__ constexpr LayoutInfo layout_info(int fmt, int group) {
    LayoutInfo L{};
    L.KS = fmt == FMT_BF16 ? 64 : (group > 64 ? group : 64);
    L.SUB = L.KS / 64;
    L.lane_bytes = fmt == FMT_BF16 ? 64 : fmt == FMT_W8 ? 32 : fmt == FMT_W4 ? 16 : 12;
    L.bits = fmt == FMT_BF16 ? 16 : fmt == FMT_W8 ? 8 : fmt == FMT_W4 ? 4 : 3;
    L.tile_bytes = 32 * L.lane_bytes;
    L.meta_bytes = fmt == FMT_BF16 ? 0 : fmt == FMT_W8 ? 32 : 40;
    // slabs per unit: keep a block near 4 KB (one stage of a warp's copy ring)
    L.R = (fmt == FMT_BF16 || (fmt == FMT_W8 && L.KS == 128)) ? 2 : 4;
    L.block_bytes = round_up(L.R * L.SUB * L.tile_bytes + L.R * L.meta_bytes, 16);
    L.bps = L.block_bytes * 2 <= 4608 ? 2 : 1;
    return L;
}

struct MatGeom {
    int N, K, NU, KT;
    long long bytes;
};

__host__ __device__ constexpr MatGeom mat_geom(int fmt, int group, int N, int K) {
    LayoutInfo L = layout_info(fmt, group);
    MatGeom g{};
    g.N = N;
    g.K = K;
    g.NU = (N + 16 * L.R - 1) / (16 * L.R);
    g.KT = (K + L.KS - 1) / L.KS;
    g.bytes = (long long)g.NU * g.KT * L.block_bytes;
    return g;
}

// byte offset of the code of element (n, k) and, for sub-byte formats, the bit position(s).
// W3 codes may be split (pair 15); this returns the word offsets and bit positions.
struct CodePos {
    long long off[3];   // byte offsets of the containing word(s) (W3 pair 15: one per code bit)
    int bit[3];         // bit position(s) within those 32-bit words
    int nparts;         // 1, or 3 for W3 pair 15
    long long meta;     // byte offset of the slab's metadata record
    int g, hi;          // row inside the slab: g + 8*hi
};

__host__ __device__ inline CodePos code_pos(int fmt, int group, int KT, int n, int k) {
    LayoutInfo L = layout_info(fmt, group);
    CodePos P{};
    int u = n / (16 * L.R), r = (n % (16 * L.R)) / 16, row16 = n % 16;
    int g = row16 % 8, hi = row16 / 8;
    int kt = k / L.KS, st = (k % L.KS) / 64, c64 = k % 64;
    int t = c64 / 16, s = (c64 % 16) / 4, x = c64 % 4;
    int lane = g * 4 + t;
    int reg = hi + 2 * (x / 2);
    long long blk = ((long long)u * KT + kt) * L.block_bytes;
    long long tile = blk + (long long)(r * L.SUB + st) * L.tile_bytes;
    P.meta = blk + (long long)L.R * L.SUB * L.tile_bytes + (long long)r * L.meta_bytes;
    P.g = g;
    P.hi = hi;
    P.nparts = 1;
    if (fmt == FMT_BF16) {
        P.off[0] = tile + (long long)(s * 32 + lane) * 16 + reg * 4 + (x % 2) * 2;
        P.bit[0] = 0;
    } else if (fmt == FMT_W8) {
        int wi = (s % 2) * 2 + hi;
        int byte = (x % 2) * 2 + x / 2;
        P.off[0] = tile + (long long)((s / 2) * 32 + lane) * 16 + wi * 4;
        P.bit[0] = byte * 8;
    } else if (fmt == FMT_W4) {
        P.off[0] = tile + (long long)lane * 16 + s * 4;
        P.bit[0] = (reg + 4 * (x % 2)) * 4;
    } else {
        int p = 4 * s + reg, half = x % 2;
        long long w_off[3] = {tile + (long long)lane * 8, tile + (long long)lane * 8 + 4, tile + 256 + (long long)lane * 4};
        if (p < 15) {
            int wi = p / 5, i = p % 5;
            P.off[0] = w_off[wi];
            P.bit[0] = 3 * i + 16 * half;
        } else {
            P.nparts = 3;
            for (int b = 0; b < 3; ++b) {
                P.off[b] = w_off[b];
                P.bit[b] = 15 + 16 * half;
            }
        }
    }
    return P;
}

}  // namespace vc
