// Host-side check of the streaming GEMV's stream-K partition (csrc/gemv_core.cuh: part_begin,
// part_owner, warp_range), compiled by nvcc and run on the host only (no kernel is launched, no
// CUDA call is made).  For every projection shape of the Nano and tiny stacks, every weight
// format and group size, and every grid the launches use (148 or 132 SMs x 1 or 2 CTAs of 8
// warps, and the no-allocation entry's 32 SMs), it checks what the kernel's sums depend on:
//   * the workers of a matrix own contiguous, disjoint, non-empty block ranges that cover it;
//   * the 32-bit quotients equal the 64-bit ones wherever the kernel takes them;
//   * for every row unit, the workers whose ranges touch it are exactly [lo, hi] as part_owner
//     names them (the last contributor counts hi - lo arrivals before it finishes the unit);
//   * a unit split between workers is the first or the last unit of each contributor's range
//     (the partial-sum slots hold two units per worker);
//   * the partial-sum and counter indices stay inside the scratch the launches are given.
// Prints one line per launch family and "ok", or the first violation.
#include "../../attention_frame_decode_b200/csrc/gemv_core.cuh"

#include <cstdio>
#include <vector>

using namespace vc;

static const long long kCounterInts = 2 * 65536;   // gemv_counter_ints()

static int check(const GemvMat (&mat)[2], int nmat, long long Wall, int num_sms, const char* what) {
    if (Wall > (long long)num_sms * kWarps) {
        printf("%s: %lld workers exceed the partial-sum scratch of %d SMs\n", what, Wall, num_sms);
        return 1;
    }
    std::vector<WarpRange> rs((size_t)Wall);
    for (long long wid = 0; wid < Wall; ++wid) rs[(size_t)wid] = warp_range(mat, nmat, wid, Wall);
    for (int m = 0; m < nmat; ++m) {
        const long long KT = mat[m].KT, NU = mat[m].NU, T = NU * KT;
        std::vector<const WarpRange*> ws;   // the matrix's workers in local order
        for (const WarpRange& r : rs)
            if (r.m == m) ws.push_back(&r);
        if (ws.empty()) { printf("%s: matrix %d has no workers\n", what, m); return 1; }
        const long long Wm = ws[0]->Wm;
        long long next = 0;
        for (size_t i = 0; i < ws.size(); ++i) {
            const WarpRange& r = *ws[i];
            if (r.wl != (long long)i || r.Wm != Wm || r.T != T) {
                printf("%s: matrix %d worker %zu: local index or totals inconsistent\n", what, m, i);
                return 1;
            }
            if (r.idle) {
                if (r.wl < Wm || r.f0 != r.f1) { printf("%s: idle worker %zu holds blocks\n", what, i); return 1; }
                continue;
            }
            if (r.f0 != next || r.f1 <= r.f0) {
                printf("%s: matrix %d worker %zu range [%d, %d) after %lld\n", what, m, i, r.f0, r.f1, next);
                return 1;
            }
            next = r.f1;
            if (r.s32 && (part_begin(r.wl, T, Wm, true) != part_begin(r.wl, T, Wm, false) ||
                          part_begin(r.wl + 1, T, Wm, true) != part_begin(r.wl + 1, T, Wm, false))) {
                printf("%s: matrix %d worker %zu: 32-bit and 64-bit ranges differ\n", what, m, i);
                return 1;
            }
            if ((r.wbase + r.wl) * 2 + 1 >= (long long)num_sms * kWarps * 2) {
                printf("%s: partial-sum slot out of the scratch\n", what);
                return 1;
            }
        }
        if (next != T) { printf("%s: matrix %d covered up to %lld of %lld blocks\n", what, m, next, T); return 1; }
        const bool s32 = ws[0]->s32;
        for (long long u = 0; u < NU; ++u) {
            const long long lo = part_owner(u * KT, T, Wm, s32), hi = part_owner((u + 1) * KT - 1, T, Wm, s32);
            if (s32 && (lo != part_owner(u * KT, T, Wm, false) || hi != part_owner((u + 1) * KT - 1, T, Wm, false))) {
                printf("%s: matrix %d unit %lld: 32-bit and 64-bit owners differ\n", what, m, u);
                return 1;
            }
            long long first = -1, last = -1;
            for (long long w = 0; w < Wm; ++w) {
                const WarpRange& r = *ws[(size_t)w];
                const bool touches = r.f0 < (u + 1) * KT && r.f1 > u * KT;
                if (touches) {
                    if (first < 0) first = w;
                    else if (w != last + 1) { printf("%s: unit %lld: contributors not contiguous\n", what, u); return 1; }
                    last = w;
                }
            }
            if (first != lo || last != hi) {
                printf("%s: matrix %d unit %lld: contributors [%lld, %lld], owners [%lld, %lld]\n", what, m, u, first,
                       last, lo, hi);
                return 1;
            }
            if (lo != hi) {
                for (long long w = lo; w <= hi; ++w) {
                    const WarpRange& r = *ws[(size_t)w];
                    const long long fu = r.f0 / KT, lu = (r.f1 - 1) / KT;
                    if (u != fu && u != lu) {
                        printf("%s: split unit %lld is inside worker %lld's range\n", what, u, w);
                        return 1;
                    }
                }
            }
            if ((m ? mat[0].NU : 0) + u >= kCounterInts) { printf("%s: counter index out of range\n", what); return 1; }
        }
    }
    return 0;
}

int main() {
    struct Proj { const char* name; int N, K, nmat; };
    const Proj nano[] = {{"in_proj", 22656, 4480, 1}, {"out_proj", 4480, 10240, 1}, {"qkv", 7168, 4480, 1},
                         {"o_proj", 4480, 5120, 1},   {"mlp_up", 15680, 4480, 1},  {"mlp_down", 4480, 15680, 1},
                         {"heads", 131072, 4480, 2}};
    const Proj tiny[] = {{"in_proj", 552, 256, 1}, {"out_proj", 256, 256, 1}, {"qkv", 512, 256, 1},
                         {"o_proj", 256, 256, 1},  {"mlp_up", 1024, 256, 1},  {"mlp_down", 256, 1024, 1},
                         {"heads", 1024, 256, 2}};
    const int fmts[][2] = {{0, 64}, {1, 64}, {1, 128}, {2, 64}, {2, 128}, {3, 64}, {3, 128}};
    // (SMs, CTAs per SM): two CTAs for up to 8 rows, one for 9..16 rows or launch shapes 1 and 2,
    // 32 SMs x 2 for the no-allocation entry
    const int grids[][2] = {{148, 2}, {148, 1}, {132, 2}, {132, 1}, {32, 2}};
    long long launches = 0;
    for (int set = 0; set < 2; ++set) {
        const Proj* ps = set ? tiny : nano;
        for (int p = 0; p < 7; ++p)
            for (const auto& f : fmts)
                for (const auto& g : grids) {
                    const MatGeom G = mat_geom(f[0], f[1], ps[p].N, ps[p].K);
                    GemvMat mat[2];
                    for (int m = 0; m < 2; ++m) mat[m] = GemvMat{nullptr, G.N, G.K, G.NU, G.KT};
                    char what[160];
                    snprintf(what, sizeof what, "%s %s fmt %d g %d, %d SMs x %d CTAs", set ? "tiny" : "nano",
                             ps[p].name, f[0], f[1], g[0], g[1]);
                    if (check(mat, ps[p].nmat, (long long)g[0] * g[1] * 8, g[0], what)) return 1;
                    ++launches;
                }
    }
    printf("%lld launch geometries\nok\n", launches);
    return 0;
}
