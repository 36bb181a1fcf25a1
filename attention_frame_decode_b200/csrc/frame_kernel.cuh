// frame_kernel.cuh -- the persistent frame kernel: one cooperative launch per decode frame.
//
// The per-frame LLM step is bound by memory bandwidth ("NemotronLabs VoiceChat 11B: GPTQ 3-bit
// LLM, MLX", introduction and measurement bullets): every weight byte of the 56 layers and both
// heads is read once per frame.  A chain of one kernel per projection drains the memory pipe at
// every kernel boundary (ramp, tail, launch gap); this kernel keeps it full for the whole frame:
//   * one CTA per SM (grid = SM count, co-resident by cooperative launch) runs the frame's ops in
//     order -- input, then per layer its projections and mixer, then the heads -- with a
//     grid-wide barrier between dependent ops;
//   * every warp owns one byte range of every projection of the frame (the split of
//     gemv_core.cuh) and streams the concatenation of its ranges through its own ring of shared
//     memory slots with 1-D bulk copies (TMA engine) completing on mbarriers.  The copies run
//     ahead of the consumer across op boundaries: while a warp waits at a barrier, or runs a
//     Mamba-2 step or attention, its ring keeps filling with the next projection's weights;
//   * activation fragments are read from L2 (they were written by the previous op on other SMs)
//     one block ahead of their use;
//   * the Mamba-2 step, decode attention and the input op are warp-level work items over the
//     whole grid, in registers (the ring holds the shared memory).
// Every wait is bounded: a barrier or copy that does not complete within its limit sets
// VC_DEV_TIMEOUT, raises the launch's abort flag and the launch winds down (all later waits
// return at once; copies in flight are waited for, again with a bound).
#pragma once
#include "frame.cuh"
#include "gemv_core.cuh"

namespace vc {

__host__ __device__ constexpr int fk_warps(int NT) { return NT == 1 ? 12 : 8; }
// the CTA's activation area (after the rings): one batch row of up to 16256 columns
static constexpr int kFkActBytes = 32 * 1024 + 256;

static constexpr long long kBarrierPolls = 1ll << 24;

VC_DEV unsigned ld_acquire_u32(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
VC_DEV int ld_relaxed_i32(const int* p) {
    int v;
    asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// grid-wide barrier number k (1-based) of this launch; false once the launch is aborting
VC_DEV bool fk_barrier(const FrameParams& fp, unsigned k, int* s_ok) {
    __syncthreads();
    if (threadIdx.x == 0) {
        int ok = ld_relaxed_i32(fp.abort) == 0;
        if (ok) {
            __threadfence();
            atomicAdd(fp.barrier, 1u);
            const unsigned target = k * gridDim.x;
            long long i = 0;
            while (ld_acquire_u32(fp.barrier) < target) {
                ++i;
                if ((i & 255) == 0 && ld_relaxed_i32(fp.abort)) { ok = 0; break; }
                if (i > kBarrierPolls) {
                    atomicOr(fp.status, VC_DEV_TIMEOUT);
                    atomicExch(fp.abort, 1);
                    ok = 0;
                    break;
                }
                if (i > 2048) __nanosleep(64);
            }
            __threadfence();
        }
        *s_ok = ok;
    }
    __syncthreads();
    return *s_ok != 0;
}

// ------------------------------------------------------------------------------------------
// the weight stream of one warp: its ranges of every projection of the frame, in op order,
// cut into chunks of whole blocks (one ring slot each)
// ------------------------------------------------------------------------------------------
struct FkStream {
    int op;          // op whose range is being issued (n_ops: none left)
    int f, f1;       // next block and end of this warp's range in that op
    int bb, bpc;     // block bytes and blocks per chunk of that op's format
    const uint8_t* w;
    int issued;      // chunks issued so far (chunk c lives in slot c mod slots)
};

template <int LF, int LG, int HF, int HG>
__device__ __forceinline__ void fk_chunking(int head, int slot_bytes, int& bb, int& bpc) {
    bb = head ? layout_info(HF, HG).block_bytes : layout_info(LF, LG).block_bytes;
    bpc = slot_bytes / bb;
    if (bpc < 1) bpc = 1;
}

template <int LF, int LG, int HF, int HG>
__device__ __forceinline__ void fk_next_range(const FrameProgram* P, int n_ops, long long gw, long long Wall,
                                              int slot_bytes, FkStream& s) {
    for (++s.op; s.op < n_ops; ++s.op) {
        const FkOp o = P->ops[s.op];
        if (o.kind != FK_GEMV) continue;
        const FkGemv* G = &P->gemv[o.idx];
        GemvMat mat[2] = {G->a.mat[0], G->a.mat[1]};
        const WarpRange r = warp_range(mat, G->a.nmat, gw, Wall);
        if (r.idle || r.f0 >= r.f1) continue;
        s.f = r.f0;
        s.f1 = r.f1;
        s.w = r.M.w;
        fk_chunking<LF, LG, HF, HG>(G->head, slot_bytes, s.bb, s.bpc);
        return;
    }
}

// lane 0: issue the stream's next chunk into ring slot `slot`
template <int LF, int LG, int HF, int HG>
__device__ __forceinline__ void fk_issue(const FrameProgram* P, int n_ops, long long gw, long long Wall, int slot_bytes,
                                         FkStream& s, uint8_t* ring, uint64_t* bar, int slot) {
    if (s.op >= n_ops) return;
    const int nb = min(s.bpc, s.f1 - s.f);
    const uint32_t bytes = (uint32_t)(nb * s.bb);
    mbar_arrive_expect_tx(&bar[slot], bytes);
    bulk_g2s(ring + (size_t)slot * slot_bytes, s.w + (size_t)s.f * s.bb, bytes, &bar[slot]);
    ++s.issued;
    s.f += nb;
    if (s.f >= s.f1) fk_next_range<LF, LG, HF, HG>(P, n_ops, gw, Wall, slot_bytes, s);
}

// ------------------------------------------------------------------------------------------
// op: step input (one warp per (row b, unit of d))
// ------------------------------------------------------------------------------------------
VC_DEV void fk_input(const InputArgs& a, const FrameParams& fp, long long gw, long long Wall, int lane) {
    const int items = a.B * a.n_units;
    for (long long it = gw; it < items; it += Wall) {
        const int b = (int)(it / a.n_units), u = (int)(it % a.n_units);
        const int slot = a.slots ? a.slots[b] : b;
        if (u == 0 && lane == 0) {
            const int okb = a.ctx_len[slot] < a.cap;
            a.ok[b] = okb;
            if (!okb) atomicOr(a.status, VC_DEV_CAPACITY);
        }
        const uint16_t* et = nullptr;
        const uint16_t* ef = nullptr;
        if (a.emb_t) {
            const int tt = fp.tok_t[b], tf = fp.tok_f[b];
            if (tt >= 0 && tt < a.Vt) et = a.emb_t + (size_t)tt * a.d;
            if (tf >= 0 && tf < a.Vf) ef = a.emb_f + (size_t)tf * a.d;
        }
        float ss = 0.0f;
        const int k1 = min(a.d, (u + 1) * a.unit_rows);
        for (int k = u * a.unit_rows + lane; k < k1; k += 32) {
            float v = bf16_bits_to_f(fp.x[(size_t)b * a.d + k]);
            if (a.emb_t) {
                if (et) v += bf16_bits_to_f(et[k]);
                if (ef) v += bf16_bits_to_f(ef[k]);
                v = bf16_bits_to_f(act_bits<false>(v));   // the fused input is a bf16 embedding
            }
            a.r[(size_t)b * a.d + k] = v;
            const float an = v * a.gamma[k];
            a.act[(size_t)b * a.act_ld + k] = a.act_f16 ? act_bits<true>(an) : act_bits<false>(an);
            if (a.tap) a.tap[(size_t)b * a.d + k] = v;
            ss += v * v;
        }
        ss = warp_sum(ss);
        if (lane == 0) a.parts[(size_t)b * a.n_units + u] = ss;
    }
}

// ------------------------------------------------------------------------------------------
// op: Mamba-2 step.  Work item = one state row (session b, head h, channel p): N fp32 values,
// lane l holding n = 4l..4l+3; a warp takes a contiguous range of rows, 32 at a time:
//   xc = silu(conv_b + sum_k conv_w[k] window[k]) over the ring of the last W pre-conv rows,
//   dt = softplus(dt_raw + dt_bias), a = exp(A dt), A = -exp(A_log),
//   S <- a S + dt x B,  y = C.S + D x,  v = y silu(z),  out_proj input bf16(v gamma_n);
//   the per-(head, half) sums of v^2 are accumulated (atomically) for the gated norm's RMS, which
//   the out_proj applies as its input scale.
// The op is bound by the latency of its loads, so they are issued wide: each lane computes the
// per-row scalars (conv of the x channel, dt, decay, gate) of one of the 32 rows at once, and the
// state rows are fetched four at a time, the next four in flight while these are updated.
// ------------------------------------------------------------------------------------------
static constexpr int kFkRows = 4;

// causal conv + SiLU of channel c for frame t: the W-1 ring rows before t and this frame's row,
// every load issued at once (W <= 8, checked at create)
VC_DEV float fk_conv(const MambaStepArgs& a, const uint16_t* ring, int t, int c, const uint16_t* xBC) {
    float wv[8], rv[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        wv[k] = 0.0f;
        rv[k] = 0.0f;
        if (k < a.W) {
            wv[k] = __ldg(a.conv_w + (size_t)c * a.W + k);
            if (k < a.W - 1) {
                const int rs = ((t - (a.W - 1) + k) % a.W + a.W) % a.W;
                rv[k] = bf16_bits_to_f(ring[(size_t)rs * a.Cx + c]);
            } else {
                rv[k] = bf16_bits_to_f(xBC[c]);
            }
        }
    }
    float acc = __ldg(a.conv_b + c);
#pragma unroll
    for (int k = 0; k < 8; ++k) acc = fmaf(wv[k], rv[k], acc);
    return silu_f(acc);
}

VC_DEV void fk_load_rows(const MambaStepArgs& a, long long base, long long r1, int n0, bool lane_on,
                         float4 (&S)[kFkRows]) {
#pragma unroll
    for (int i = 0; i < kFkRows; ++i) {
        S[i] = make_float4(0, 0, 0, 0);
        const long long row = base + i;
        if (row < r1 && lane_on) {
            const int b = (int)(row / (a.H * a.P));
            const int slot = a.slots ? a.slots[b] : b;
            const int hp = (int)(row % (a.H * a.P));
            S[i] = __ldcg(reinterpret_cast<const float4*>(a.ssm + ((size_t)slot * a.H * a.P + hp) * a.N + n0));
        }
    }
}

VC_DEV void fk_mamba(const MambaStepArgs& a, long long gw, long long Wall, int lane) {
    const long long rows = (long long)a.B * a.H * a.P;
    const long long r0 = gw * rows / Wall, r1 = (gw + 1) * rows / Wall;
    const int n0 = 4 * lane;
    const bool lane_on = n0 < a.N;
    const int hpg = a.H / a.G;
    int cb = -1, cg = -1;                 // session and group whose B, C the lane holds
    float Bv[4] = {0, 0, 0, 0}, Cv[4] = {0, 0, 0, 0};
    float4 S[kFkRows], Sn[kFkRows];
    if (r0 < r1) fk_load_rows(a, r0, r1, n0, lane_on, S);
    for (long long base = r0; base < r1; base += 32) {
        // ---- per-row scalars, lane l for row base + l ----
        const long long row = base + lane;
        const bool valid = row < r1;
        float xv = 0.0f, dx = 0.0f, decay = 0.0f, zs = 0.0f, Dd = 0.0f, gam = 0.0f;
        int b = 0, hp = 0, okb = 0;
        if (valid) {
            b = (int)(row / (a.H * a.P));
            hp = (int)(row % (a.H * a.P));
            const int h = hp / a.P;
            const int slot = a.slots ? a.slots[b] : b;
            okb = a.ok ? a.ok[b] != 0 : 1;
            const int t = a.ctx_len[slot];
            const uint16_t* zx = a.zx + (size_t)b * a.zx_ld;
            uint16_t* ring = a.conv + (size_t)slot * a.W * a.Cx;
            xv = fk_conv(a, ring, t, hp, zx + a.E);
            const float dt = softplus_f(bf16_bits_to_f(zx[a.E + a.Cx + h]) + a.dt_bias[h]);
            decay = expf(-expf(a.A_log[h]) * dt);
            dx = dt * xv;
            zs = silu_f(bf16_bits_to_f(zx[hp]));
            Dd = a.D[h];
            gam = a.gnorm[hp];
            if (okb) ring[(size_t)(t % a.W) * a.Cx + hp] = zx[a.E + hp];   // the ring row of frame t
        }
        const int nrow = (int)min((long long)32, r1 - base);
        float vsq = 0.0f;   // this lane's row's v^2
        for (int sb = 0; sb < nrow; sb += kFkRows) {
            // the next state rows in flight while these are updated
            const long long nb_ = base + sb + kFkRows;
            if (nb_ < r1) fk_load_rows(a, nb_, r1, n0, lane_on, Sn);
#pragma unroll
            for (int i = 0; i < kFkRows; ++i) {
                const int src = sb + i;
                if (src >= nrow) break;
                const int rb = __shfl_sync(0xffffffffu, b, src), rhp = __shfl_sync(0xffffffffu, hp, src);
                const int rok = __shfl_sync(0xffffffffu, okb, src);
                const float rdx = __shfl_sync(0xffffffffu, dx, src), rdec = __shfl_sync(0xffffffffu, decay, src);
                const int h = rhp / a.P, p = rhp % a.P;
                const int g = h / hpg;
                if (rb != cb || g != cg) {   // B and C of this group for the lane's n
                    cb = rb;
                    cg = g;
                    const int slot = a.slots ? a.slots[rb] : rb;
                    const int t = a.ctx_len[slot];
                    const uint16_t* xBC = a.zx + (size_t)rb * a.zx_ld + a.E;
                    const uint16_t* ring = a.conv + (size_t)slot * a.W * a.Cx;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        Bv[e] = lane_on ? fk_conv(a, ring, t, a.E + g * a.N + n0 + e, xBC) : 0.0f;
                        Cv[e] = lane_on ? fk_conv(a, ring, t, a.E + a.G * a.N + g * a.N + n0 + e, xBC) : 0.0f;
                    }
                }
                if (rok && lane_on && p == 0 && h % hpg == 0) {   // the group's B, C rows of the ring
                    const int slot = a.slots ? a.slots[rb] : rb;
                    const int t = a.ctx_len[slot];
                    const uint16_t* xBC = a.zx + (size_t)rb * a.zx_ld + a.E;
                    uint16_t* rw = a.conv + ((size_t)slot * a.W + t % a.W) * a.Cx;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int cB = a.E + g * a.N + n0 + e, cC = a.E + a.G * a.N + g * a.N + n0 + e;
                        rw[cB] = xBC[cB];
                        rw[cC] = xBC[cC];
                    }
                }
                float4 sn;
                sn.x = fmaf(rdec, S[i].x, rdx * Bv[0]);
                sn.y = fmaf(rdec, S[i].y, rdx * Bv[1]);
                sn.z = fmaf(rdec, S[i].z, rdx * Bv[2]);
                sn.w = fmaf(rdec, S[i].w, rdx * Bv[3]);
                float y = Cv[0] * sn.x + Cv[1] * sn.y + Cv[2] * sn.z + Cv[3] * sn.w;
                y = warp_sum(y);
                if (rok && lane_on) {
                    const int slot = a.slots ? a.slots[rb] : rb;
                    *reinterpret_cast<float4*>(a.ssm + ((size_t)slot * a.H * a.P + rhp) * a.N + n0) = sn;
                }
                if (lane == src) {   // the row's own lane finishes it
                    const float v = fmaf(Dd, xv, y) * zs;
                    vsq = v * v;
                    const float an = v * gam;
                    a.act[(size_t)b * a.act_ld + hp] = a.act_f16 ? act_bits<true>(an) : act_bits<false>(an);
                }
            }
#pragma unroll
            for (int i = 0; i < kFkRows; ++i) S[i] = Sn[i];
        }
        // sums of v^2 per (session, head half): the 32 rows span at most two halves of length P/2
        // when P/2 >= 32, in general a few; reduce lane groups of equal key
        const int key = valid ? b * 2 * a.H + 2 * (hp / a.P) + ((hp % a.P) >= a.P / 2) : -1;
        unsigned todo = __ballot_sync(0xffffffffu, valid);
        while (todo) {
            const int leader = __ffs(todo) - 1;
            const int k = __shfl_sync(0xffffffffu, key, leader);
            const unsigned same = __ballot_sync(0xffffffffu, key == k);
            const float sum = warp_sum(key == k ? vsq : 0.0f);
            if (lane == leader) atomicAdd(a.parts + k, sum);
            todo &= ~same;
        }
    }
}

// ------------------------------------------------------------------------------------------
// op: GQA decode attention, partial softmax over splits of 32 keys.  Work item = (session b,
// KV head j, split); lane l holds dims l*DPL .. l*DPL+DPL-1 of the GQ query heads sharing j.
// Writes per (item, head): unnormalised output, running max and sum (online softmax).
// ------------------------------------------------------------------------------------------
template <int GQ, int DPL>
__device__ void fk_attn_t(const AttnArgs& a, long long gw, long long Wall, int lane) {
    constexpr int Dh = 32 * DPL, KB = 4, DW = DPL / 2;   // keys per load batch, 32-bit words per key
    static_assert(kFkAttnSplit == 32, "one key per lane");
    const int MS = a.max_splits;
    const long long items = (long long)a.B * a.Hk * MS;
    const float scale = rsqrtf((float)Dh);
    for (long long it = gw; it < items; it += Wall) {
        const int b = (int)(it / ((long long)a.Hk * MS));
        const int j = (int)((it / MS) % a.Hk);
        const int sp = (int)(it % MS);
        const int slot = a.slots ? a.slots[b] : b;
        const int t = a.ctx_len[slot];
        const int k0 = sp * kFkAttnSplit;
        if (!a.ok[b] || k0 > t) continue;
        const int nk = min(t + 1, k0 + kFkAttnSplit) - k0;
        const size_t head_off = ((size_t)slot * a.Hk + j) * a.cap;
        const uint32_t* Kg = reinterpret_cast<const uint32_t*>(a.kcache + (head_off + k0) * Dh + lane * DPL);
        const uint32_t* Vg = reinterpret_cast<const uint32_t*>(a.vcache + (head_off + k0) * Dh + lane * DPL);
        float q[GQ][DPL];
#pragma unroll
        for (int i = 0; i < GQ; ++i)
#pragma unroll
            for (int d = 0; d < DPL; ++d)
                q[i][d] = bf16_bits_to_f(__ldcg(a.q + (size_t)b * a.q_ld + (size_t)(j * GQ + i) * Dh + lane * DPL + d)) *
                          scale;
        // 1. scores: lane l owns the dims l*DPL.., every key's dot product is a warp sum, and lane
        //    e keeps key e's scores
        float sm[GQ];
#pragma unroll
        for (int i = 0; i < GQ; ++i) sm[i] = -INFINITY;
        uint32_t kw[KB][DW], kn[KB][DW];
        auto loadk = [&](int k, uint32_t (&K)[KB][DW]) {
#pragma unroll
            for (int e = 0; e < KB; ++e)
#pragma unroll
                for (int w = 0; w < DW; ++w) K[e][w] = k + e < nk ? __ldcg(Kg + (size_t)(k + e) * (Dh / 2) + w) : 0u;
        };
        loadk(0, kw);
        for (int kb = 0; kb < nk; kb += KB) {
            if (kb + KB < nk) loadk(kb + KB, kn);
#pragma unroll
            for (int e = 0; e < KB; ++e) {
                float kf[DPL];
#pragma unroll
                for (int w = 0; w < DW; ++w) {
                    kf[2 * w] = __uint_as_float(kw[e][w] << 16);
                    kf[2 * w + 1] = __uint_as_float(kw[e][w] & 0xFFFF0000u);
                }
#pragma unroll
                for (int i = 0; i < GQ; ++i) {
                    float s = 0.0f;
#pragma unroll
                    for (int d = 0; d < DPL; ++d) s = fmaf(q[i][d], kf[d], s);
                    s = warp_sum(s);
                    if (lane == kb + e && kb + e < nk) sm[i] = s;
                }
            }
#pragma unroll
            for (int e = 0; e < KB; ++e)
#pragma unroll
                for (int w = 0; w < DW; ++w) kw[e][w] = kn[e][w];
        }
        // 2. softmax of the split: max and sum over the lanes' keys
        float mx[GQ], pe[GQ], ls[GQ];
#pragma unroll
        for (int i = 0; i < GQ; ++i) {
            mx[i] = warp_max(sm[i]);
            pe[i] = lane < nk ? __expf(sm[i] - mx[i]) : 0.0f;
            ls[i] = warp_sum(pe[i]);
        }
        // 3. unnormalised p . V: lane l owns the dims l*DPL.., key e's weights come from lane e
        float o[GQ][DPL];
#pragma unroll
        for (int i = 0; i < GQ; ++i)
#pragma unroll
            for (int d = 0; d < DPL; ++d) o[i][d] = 0.0f;
        uint32_t vw[KB][DW], vn[KB][DW];
        auto loadv = [&](int k, uint32_t (&V)[KB][DW]) {
#pragma unroll
            for (int e = 0; e < KB; ++e)
#pragma unroll
                for (int w = 0; w < DW; ++w) V[e][w] = k + e < nk ? __ldcg(Vg + (size_t)(k + e) * (Dh / 2) + w) : 0u;
        };
        loadv(0, vw);
        for (int kb = 0; kb < nk; kb += KB) {
            if (kb + KB < nk) loadv(kb + KB, vn);
#pragma unroll
            for (int e = 0; e < KB; ++e) {
                float vf[DPL];
#pragma unroll
                for (int w = 0; w < DW; ++w) {
                    vf[2 * w] = __uint_as_float(vw[e][w] << 16);
                    vf[2 * w + 1] = __uint_as_float(vw[e][w] & 0xFFFF0000u);
                }
#pragma unroll
                for (int i = 0; i < GQ; ++i) {
                    const float p = __shfl_sync(0xffffffffu, pe[i], (kb + e) & 31);
#pragma unroll
                    for (int d = 0; d < DPL; ++d) o[i][d] = fmaf(p, vf[d], o[i][d]);
                }
            }
#pragma unroll
            for (int e = 0; e < KB; ++e)
#pragma unroll
                for (int w = 0; w < DW; ++w) vw[e][w] = vn[e][w];
        }
        float* part = a.scratch + ((((size_t)b * a.Hk + j) * MS + sp) * GQ) * (Dh + 2);
#pragma unroll
        for (int i = 0; i < GQ; ++i) {
#pragma unroll
            for (int d = 0; d < DPL; ++d) part[i * (Dh + 2) + lane * DPL + d] = o[i][d];
            if (lane == 0) {
                part[i * (Dh + 2) + Dh] = mx[i];
                part[i * (Dh + 2) + Dh + 1] = ls[i];
            }
        }
    }
}

// the shapes instantiated (GQ query heads per KV head, head dim 64 or 128); frame_attn_supported
// names them for the host
#define VC_FK_ATTN_SHAPES(X) X(1, 2) X(2, 2) X(4, 2) X(5, 2) X(1, 4) X(2, 4) X(4, 4) X(5, 4)

VC_DEV void fk_attn(const AttnArgs& a, long long gw, long long Wall, int lane) {
    const int GQ = a.Hq / a.Hk, DPL = a.Dh / 32;
#define VC_FK_ATTN_CASE(G, D) \
    if (GQ == G && DPL == D) { fk_attn_t<G, D>(a, gw, Wall, lane); return; }
    VC_FK_ATTN_SHAPES(VC_FK_ATTN_CASE)
#undef VC_FK_ATTN_CASE
}

// merge of the splits: work item = (session b, query head i, 32 dims); lane = one dim
VC_DEV void fk_attn_merge(const AttnArgs& a, long long gw, long long Wall, int lane) {
    const int GQ = a.Hq / a.Hk, Dh = a.Dh, MS = a.max_splits;
    const int dch = Dh / 32;
    const long long items = (long long)a.B * a.Hq * dch;
    for (long long it = gw; it < items; it += Wall) {
        const int b = (int)(it / ((long long)a.Hq * dch));
        const int i = (int)((it / dch) % a.Hq);
        const int d = (int)(it % dch) * 32 + lane;
        if (!a.ok[b]) continue;
        const int slot = a.slots ? a.slots[b] : b;
        const int nsplit = a.ctx_len[slot] / kFkAttnSplit + 1;
        const int j = i / GQ, ii = i % GQ;
        const float* base = a.scratch + (((size_t)b * a.Hk + j) * MS * GQ + ii) * (Dh + 2);
        float M = -INFINITY, L = 0.0f, O = 0.0f;
        for (int s0 = 0; s0 < nsplit; s0 += 16) {   // sixteen splits' loads in flight together
            float ms[16], ls[16], os[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const float* p = base + (size_t)(s0 + e) * GQ * (Dh + 2);
                const bool in = s0 + e < nsplit;
                ms[e] = in ? __ldcg(p + Dh) : -INFINITY;
                ls[e] = in ? __ldcg(p + Dh + 1) : 0.0f;
                os[e] = in ? __ldcg(p + d) : 0.0f;
            }
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                if (s0 + e >= nsplit) break;
                const float mn = fmaxf(M, ms[e]);
                const float c0 = __expf(M - mn), c1 = __expf(ms[e] - mn);
                L = L * c0 + ls[e] * c1;
                O = O * c0 + os[e] * c1;
                M = mn;
            }
        }
        const float o = O / L;
        a.act[(size_t)b * a.act_ld + (size_t)i * Dh + d] = a.act_f16 ? act_bits<true>(o) : act_bits<false>(o);
    }
}

// ------------------------------------------------------------------------------------------
// op: one projection.  The warp consumes its range chunk by chunk from the ring (waiting on the
// slot's mbarrier), refills the freed slot with the stream's next chunk, and finishes units.
// ------------------------------------------------------------------------------------------
template <int FMT, int GRP, int NT, int EPI>
__device__ __forceinline__ void fk_flush(const GemvArgs& a, const WarpRange& wr, int u,
                                         float (&acc)[layout_info(FMT, GRP).R][NT][4],
                                         unsigned long long (&best)[NT][2], int lane) {
    unit_flush<FMT, GRP, NT, EPI, true>(a, wr, u, acc, best, lane);
}

template <int FMT, int GRP, int NT>
__device__ __forceinline__ void fk_flush_any(int epi, const GemvArgs& a, const WarpRange& wr, int u,
                                             float (&acc)[layout_info(FMT, GRP).R][NT][4],
                                             unsigned long long (&best)[NT][2], int lane) {
    switch (epi) {
        case EPI_STORE: fk_flush<FMT, GRP, NT, EPI_STORE>(a, wr, u, acc, best, lane); break;
        case EPI_RELU2: fk_flush<FMT, GRP, NT, EPI_RELU2>(a, wr, u, acc, best, lane); break;
        case EPI_RESID: fk_flush<FMT, GRP, NT, EPI_RESID>(a, wr, u, acc, best, lane); break;
        case EPI_QKV: fk_flush<FMT, GRP, NT, EPI_QKV>(a, wr, u, acc, best, lane); break;
        default: fk_flush<FMT, GRP, NT, EPI_ARGMAX>(a, wr, u, acc, best, lane); break;
    }
}

// The activation of a projection: staged whole in shared memory when it fits the CTA's
// activation area (every block's fragments are then a shared-memory load), else read from L2
// one block ahead of its use.
template <int FMT, int GRP, int NT, bool ACT_SMEM>
struct FkAct {
    static constexpr LayoutInfo L = layout_info(FMT, GRP);
    const uint4* row[NT];   // the lane's row 8j + g (rows past the batch read its last row: their
                            // sums are computed and never stored), at column 16t, in uint4
    __device__ __forceinline__ void load(int kt, uint4 (&bv)[L.SUB][NT][2]) const {
#pragma unroll
        for (int st = 0; st < L.SUB; ++st)
#pragma unroll
            for (int j = 0; j < NT; ++j) {
                const uint4* p = row[j] + kt * (L.KS / 8) + 8 * st;
                if constexpr (ACT_SMEM) {
                    bv[st][j][0] = p[0];
                    bv[st][j][1] = p[1];
                } else {
                    bv[st][j][0] = __ldcg(p);
                    bv[st][j][1] = __ldcg(p + 1);
                }
            }
    }
};

// the warp's share of one projection; false when the launch must wind down (a copy never arrived)
template <int LF, int LG, int HF, int HG, int FMT, int GRP, int NT, bool ACT_SMEM>
__device__ __forceinline__ bool fk_gemv_run(const FkGemv& G, const float* insc_tab, const FkAct<FMT, GRP, NT, ACT_SMEM>& act,
                                            const WarpRange& wr, const FrameParams& fp, long long gw, long long Wall,
                                            int lane, uint8_t* ring, uint64_t* bar, int n_ops, FkStream& ps, int& ccount,
                                            unsigned long long (&best)[NT][2]) {
    constexpr LayoutInfo L = layout_info(FMT, GRP);
    constexpr int R = L.R, KS = L.KS;
    const GemvArgs& a = G.a;
    const int B = a.B, t = lane & 3;
    const int KT = wr.M.KT;
    const int bpc = max(1, fp.slot_bytes / L.block_bytes);
    const int ng = a.insc.parts ? a.insc.n_groups : 1;
    float acc[R][NT][4];
    auto zero_acc = [&]() {
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int j = 0; j < NT; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[r][j][e] = 0.0f;
    };
    zero_acc();
    int cur_u = wr.f0 / KT, kt = wr.f0 % KT;
    bool pending = false;
    float sc[NT][2];
    int sc_next = kt;
    uint4 bv[L.SUB][NT][2];
    if constexpr (!ACT_SMEM) act.load(kt, bv);
    for (int f = wr.f0; f < wr.f1;) {
        const int nb = min(bpc, wr.f1 - f);
        const int slot = ccount % fp.slots;
        const uint32_t phase = (uint32_t)(ccount / fp.slots) & 1u;
        if (!mbar_wait(&bar[slot], phase, fp.status)) return false;
        const uint8_t* base = ring + (size_t)slot * fp.slot_bytes;
        for (int jb = 0; jb < nb; ++jb) {
            if (kt == sc_next) {
                const int qg = ng > 1 ? (kt * KS) / a.insc.group_cols : 0;
                sc_next = ng > 1 ? min(KT, ((qg + 1) * a.insc.group_cols) / KS) : KT;
#pragma unroll
                for (int j = 0; j < NT; ++j)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int b = 8 * j + 2 * t + e;
                        sc[j][e] = b < B ? insc_tab[b * ng + qg] : 0.0f;
                    }
            }
            if constexpr (ACT_SMEM) {
                act.load(kt, bv);
                consume_block_bv<FMT, GRP, NT>(base + jb * L.block_bytes, bv, lane, sc, acc, B > 1, G.epi == EPI_ARGMAX);
            } else {
                uint4 bn[L.SUB][NT][2];
                act.load(kt + 1 == KT ? 0 : kt + 1, bn);   // one block ahead
                consume_block_bv<FMT, GRP, NT>(base + jb * L.block_bytes, bv, lane, sc, acc, B > 1, G.epi == EPI_ARGMAX);
#pragma unroll
                for (int st = 0; st < L.SUB; ++st)
#pragma unroll
                    for (int j = 0; j < NT; ++j) { bv[st][j][0] = bn[st][j][0]; bv[st][j][1] = bn[st][j][1]; }
            }
            pending = true;
            if (++kt == KT) {
                fk_flush_any<FMT, GRP, NT>(G.epi, a, wr, cur_u, acc, best, lane);
                zero_acc();
                pending = false;
                kt = 0;
                ++cur_u;
                if (ng > 1) sc_next = 0;
            }
        }
        __syncwarp();
        if (lane == 0) {
            fence_proxy_async();
            fk_issue<LF, LG, HF, HG>(fp.prog, n_ops, gw, Wall, fp.slot_bytes, ps, ring, bar, slot);
        }
        ++ccount;
        f += nb;
    }
    if (pending) fk_flush_any<FMT, GRP, NT>(G.epi, a, wr, cur_u, acc, best, lane);
    return true;
}

// one projection: the CTA stages the activation (when it fits its activation area) and builds
// the input-scale table, then every warp runs its share
template <int LF, int LG, int HF, int HG, int FMT, int GRP, int NT, int WARPS>
__device__ bool fk_gemv(const FkGemv& G, float* insc_tab, uint4* act_s, int act_s_bytes, const FrameParams& fp,
                        long long gw, long long Wall, int warp, int lane, uint8_t* ring, uint64_t* bar, int n_ops,
                        FkStream& ps, int& ccount) {
    constexpr LayoutInfo L = layout_info(FMT, GRP);
    const GemvArgs& a = G.a;
    const int B = a.B, t = lane & 3;
    const WarpRange wr = warp_range(a.mat, a.nmat, gw, Wall);
    const bool busy = !wr.idle && wr.f0 < wr.f1;
    // activation rows of KT * KS columns, padded by 16 bytes against bank conflicts
    const int rowq = wr.M.KT * (L.KS / 8) + 1;
    const bool smem_act = B * rowq * 16 <= act_s_bytes;
    if (smem_act) {
        const uint4* src = reinterpret_cast<const uint4*>(a.act);
        const int ldq = a.act_ld / 8;
        for (int i = threadIdx.x; i < B * (rowq - 1); i += blockDim.x) {
            const int b = i / (rowq - 1), c = i - b * (rowq - 1);
            act_s[b * rowq + c] = __ldcg(src + (size_t)b * ldq + c);
        }
    }
    {
        const InScale& is = a.insc;
        const int ng = is.parts ? is.n_groups : 1;
        for (int idx = warp; idx < B * ng; idx += WARPS) {
            float v = 1.0f;
            if (is.parts) {
                const int b = idx / ng, q = idx % ng;
                const float* p = is.parts + ((size_t)b * ng + q) * is.per_group;
                float s = 0.0f;
                for (int i = lane; i < is.per_group; i += 32) s += __ldcg(p + i);
                s = warp_sum(s);
                v = rsqrtf(s * is.inv_width + is.eps);
            }
            if (lane == 0) insc_tab[idx] = v;
        }
        __syncthreads();
    }
    unsigned long long best[NT][2];
#pragma unroll
    for (int j = 0; j < NT; ++j) best[j][0] = best[j][1] = 0ull;
    bool alive = true;
    if (busy) {
        if (smem_act) {
            FkAct<FMT, GRP, NT, true> act;
#pragma unroll
            for (int j = 0; j < NT; ++j) act.row[j] = act_s + min(8 * j + (lane >> 2), B - 1) * rowq + 2 * t;
            alive = fk_gemv_run<LF, LG, HF, HG, FMT, GRP, NT, true>(G, insc_tab, act, wr, fp, gw, Wall, lane, ring, bar,
                                                                   n_ops, ps, ccount, best);
        } else {
            FkAct<FMT, GRP, NT, false> act;
#pragma unroll
            for (int j = 0; j < NT; ++j)
                act.row[j] = reinterpret_cast<const uint4*>(a.act + (size_t)min(8 * j + (lane >> 2), B - 1) * a.act_ld) +
                             2 * t;
            alive = fk_gemv_run<LF, LG, HF, HG, FMT, GRP, NT, false>(G, insc_tab, act, wr, fp, gw, Wall, lane, ring, bar,
                                                                    n_ops, ps, ccount, best);
        }
    }
    if (G.epi == EPI_ARGMAX && alive) argmax_publish<NT>(a, wr.m, best, Wall, lane);
    return alive;
}

// ------------------------------------------------------------------------------------------
// the kernel
// ------------------------------------------------------------------------------------------
template <int LF, int LG, int HF, int HG, int NT>
__global__ void __launch_bounds__(fk_warps(NT) * 32, 1) frame_kernel(const FrameParams fp) {
    constexpr int WARPS = fk_warps(NT);
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t bars[WARPS][kMaxSlots];
    __shared__ float insc_tab[kMaxB * 16];
    __shared__ __align__(16) FkGemv cur[2];   // this GEMV op's and the next one's arguments
    __shared__ int s_ok;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long Wall = (long long)gridDim.x * WARPS;
    const long long gw = (long long)blockIdx.x * WARPS + warp;
    const FrameProgram* P = fp.prog;
    const int n_ops = P->n_ops;
    uint8_t* ring = smem + (size_t)warp * fp.slots * fp.slot_bytes;
    uint64_t* bar = bars[warp];
    uint4* act_s = reinterpret_cast<uint4*>(smem + (size_t)WARPS * fp.slots * fp.slot_bytes);

    // the weight stream starts at once: the first slots fill while the input op runs
    FkStream ps{};
    ps.op = -1;
    if (lane == 0) {
        for (int s = 0; s < fp.slots; ++s) mbar_init(&bar[s], 1);
        fence_mbar_init();
        fk_next_range<LF, LG, HF, HG>(P, n_ops, gw, Wall, fp.slot_bytes, ps);
        for (int s = 0; s < fp.slots; ++s) fk_issue<LF, LG, HF, HG>(P, n_ops, gw, Wall, fp.slot_bytes, ps, ring, bar, s);
    }
    __syncwarp();
    int ccount = 0;   // chunks consumed by this warp
    unsigned nbar = 0;
    int gsel = 0;     // the buffer of cur holding the next GEMV op's arguments
    // a GEMV op's arguments are copied to shared memory before the barrier that precedes it
    auto stage_args = [&](int oi) {
        if (oi < n_ops && P->ops[oi].kind == FK_GEMV) {
            const int n4 = (int)(sizeof(FkGemv) / 16);
            const uint4* src = reinterpret_cast<const uint4*>(&P->gemv[P->ops[oi].idx]);
            uint4* dst = reinterpret_cast<uint4*>(&cur[gsel]);
            for (int i = threadIdx.x; i < n4; i += blockDim.x) dst[i] = src[i];
        }
    };
    stage_args(0);
    __syncthreads();
    bool ok = true;
    for (int oi = 0; oi < n_ops && ok; ++oi) {
        const FkOp op = P->ops[oi];
        if (op.kind == FK_GEMV) {
            FkGemv& G = cur[gsel];
            gsel ^= 1;
            if (threadIdx.x == 0 && G.epi == EPI_ARGMAX) {   // the heads' token outputs are the launch's
                G.a.tok[0] = fp.tok_t;
                G.a.tok[1] = fp.tok_f;
            }
            if (blockIdx.x == 0 && G.zero_buf)
                for (int i = threadIdx.x; i < G.zero_n; i += blockDim.x) G.zero_buf[i] = 0.0f;
            bool alive;
            if (G.head)
                alive = fk_gemv<LF, LG, HF, HG, HF, HG, NT, WARPS>(G, insc_tab, act_s, kFkActBytes, fp, gw, Wall, warp,
                                                                  lane, ring, bar, n_ops, ps, ccount);
            else
                alive = fk_gemv<LF, LG, HF, HG, LF, LG, NT, WARPS>(G, insc_tab, act_s, kFkActBytes, fp, gw, Wall, warp,
                                                                  lane, ring, bar, n_ops, ps, ccount);
            if (!alive && lane == 0) atomicExch(fp.abort, 1);
        } else if (op.kind == FK_MAMBA) {
            fk_mamba(P->mamba[op.idx], gw, Wall, lane);
        } else if (op.kind == FK_ATTN) {
            fk_attn(P->attn[op.idx], gw, Wall, lane);
        } else if (op.kind == FK_ATTN_MERGE) {
            fk_attn_merge(P->attn[op.idx], gw, Wall, lane);
        } else {
            fk_input(P->input, fp, gw, Wall, lane);
        }
        if (oi + 1 < n_ops) {
            stage_args(oi + 1);
            ok = fk_barrier(fp, ++nbar, &s_ok);
        }
    }
    // after an abort, chunks issued but not consumed may still be in flight: wait for them
    // (bounded) before the CTA's shared memory is released.  In a completed frame none are.
    if (lane == 0)
        for (int c = ccount; c < ps.issued; ++c)
            if (!mbar_wait(&bar[c % fp.slots], (uint32_t)(c / fp.slots) & 1u, nullptr)) break;
    __syncwarp();
    // the last CTA out returns the barrier, abort and exit words to zero for the next launch
    // (every CTA has passed its last barrier when it gets here)
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(fp.barrier + 2, 1u) == gridDim.x - 1) {
            fp.barrier[0] = 0u;
            atomicExch(fp.abort, 0);
            fp.barrier[2] = 0u;
            __threadfence();
        }
    }
}

// one launch: a cooperative grid of num_sms CTAs (co-resident, as the grid barriers require)
template <int LF, int LG, int HF, int HG, int NT>
cudaError_t frame_launch_t(const FrameParams& p, int num_sms, size_t smem, cudaStream_t s) {
    auto kern = frame_kernel<LF, LG, HF, HG, NT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, fk_warps(NT) * 32, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorNotSupported;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(num_sms);
    cfg.blockDim = dim3(fk_warps(NT) * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace vc
