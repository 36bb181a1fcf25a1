// Host-side check of the device weight layout of the streaming GEMV (csrc/layout.cuh), compiled
// with the host compiler: for each format and group size, every code of a padded matrix lies
// inside the matrix bytes, no two codes share a bit, the codes of a tile fill it exactly, and each
// slab's metadata record lies inside its block after the tiles.  Prints "ok" or the first fault.
#define __host__
#define __device__
#include "../../attention_frame_decode_b200/csrc/layout.cuh"

#include <cstdio>
#include <vector>

using namespace vc;

static int check(int fmt, int group, int N, int K) {
    const LayoutInfo L = layout_info(fmt, group);
    const MatGeom G = mat_geom(fmt, group, N, K);
    const long long nbits = G.bytes * 8;
    std::vector<unsigned char> used((size_t)nbits, 0);
    const int rows = G.NU * 16 * L.R, cols = G.KT * L.KS;
    const long long tiles_end_in_block = (long long)L.R * L.SUB * L.tile_bytes;
    long long code_bits = 0;
    for (int n = 0; n < rows; ++n) {
        for (int k = 0; k < cols; ++k) {
            const CodePos P = code_pos(fmt, group, G.KT, n, k);
            const long long blk = ((long long)(n / (16 * L.R)) * G.KT + k / L.KS) * L.block_bytes;
            const int width = P.nparts == 3 ? 1 : L.bits;
            for (int i = 0; i < P.nparts; ++i) {
                if (P.bit[i] < 0 || P.bit[i] + width > 32) {
                    printf("fmt %d g %d: (%d,%d) bit %d out of its word\n", fmt, group, n, k, P.bit[i]);
                    return 1;
                }
                const long long b0 = P.off[i] * 8 + P.bit[i];
                if (P.off[i] < blk || b0 + width > (blk + tiles_end_in_block) * 8) {
                    printf("fmt %d g %d: (%d,%d) outside its block's tiles\n", fmt, group, n, k);
                    return 1;
                }
                for (int j = 0; j < width; ++j) {
                    if (used[(size_t)(b0 + j)]) {
                        printf("fmt %d g %d: (%d,%d) shares bit %lld\n", fmt, group, n, k, b0 + j);
                        return 1;
                    }
                    used[(size_t)(b0 + j)] = 1;
                    code_bits++;
                }
            }
            const long long meta_lo = blk + tiles_end_in_block + (long long)((n % (16 * L.R)) / 16) * L.meta_bytes;
            if (P.meta != meta_lo || P.meta + L.meta_bytes > blk + L.block_bytes) {
                printf("fmt %d g %d: (%d,%d) metadata record misplaced\n", fmt, group, n, k);
                return 1;
            }
            if (P.g + 8 * P.hi != n % 16) {
                printf("fmt %d g %d: (%d,%d) slab row %d\n", fmt, group, n, k, P.g + 8 * P.hi);
                return 1;
            }
        }
    }
    // the tiles are packed: every bit of every tile area holds a code bit
    if (code_bits != (long long)G.NU * G.KT * tiles_end_in_block * 8) {
        printf("fmt %d g %d: %lld code bits for %lld tile bits\n", fmt, group, code_bits,
               (long long)G.NU * G.KT * tiles_end_in_block * 8);
        return 1;
    }
    if (L.block_bytes % 16 || L.block_bytes < tiles_end_in_block + L.R * L.meta_bytes) {
        printf("fmt %d g %d: block of %d bytes\n", fmt, group, L.block_bytes);
        return 1;
    }
    return 0;
}

int main() {
    const int shapes[][2] = {{64, 64}, {100, 200}, {16, 960}, {130, 320}};
    const int cases[][2] = {{FMT_BF16, 64}, {FMT_W8, 64}, {FMT_W8, 128}, {FMT_W4, 64},
                            {FMT_W4, 128}, {FMT_W3, 64}, {FMT_W3, 128}};
    for (auto& c : cases)
        for (auto& s : shapes)
            if (check(c[0], c[1], s[0], s[1])) return 1;
    // bits per stored weight of a full block, in 64ths of a bit (per format and group 64)
    for (auto& c : cases) {
        const LayoutInfo L = layout_info(c[0], c[1]);
        const long long w = (long long)L.R * 16 * L.KS;
        printf("fmt %d g %d: %lld/64 bits per weight\n", c[0], c[1], (long long)L.block_bytes * 8 * 64 / w);
    }
    printf("ok\n");
    return 0;
}
