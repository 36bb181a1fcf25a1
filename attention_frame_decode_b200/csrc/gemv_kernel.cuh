// gemv_kernel.cuh -- streaming weight GEMV for the per-frame decode step (B <= 16 sessions),
// one launch per projection.
//
// The per-frame LLM step is bound by memory bandwidth, and its time falls with the bits per
// weight (NemotronLabs VoiceChat 11B: GPTQ 3-bit LLM, MLX, the measurement bullets of the
// introduction), so the kernel is built to read every weight byte exactly once at full HBM rate:
//   * persistent grid (two 8-warp CTAs per SM for up to 8 batch rows, one for 9..16); each warp
//     is a worker that owns one contiguous byte range of the matrix (gemv_core.cuh, layout.cuh)
//     and streams it through its own ring of shared memory slots with 1-D bulk copies
//     (cp.async.bulk, TMA engine) completing on mbarriers;
//   * the weight copies of the first ring slots are issued before griddepcontrol.wait, so they
//     overlap the tail of the previous kernel (programmatic dependent launch);
//   * dequantization, tensor-core products and the fused epilogues are the shared per-warp
//     building blocks of gemv_core.cuh.
#pragma once
#include <atomic>

#include "gemv_core.cuh"
#include "tc.cuh"

namespace vc {

// warps per CTA: 8 for every batch size
__host__ __device__ constexpr int warps_for(int) { return 8; }
// CTAs per SM: two 8-warp CTAs for up to 8 rows (<= 128 registers, <= ~105 KB shared memory each),
// so that under programmatic dependent launch the next kernel's CTAs can become resident and
// start their weight copies while this kernel drains; one CTA for 9..16 rows
__host__ __device__ constexpr int ctas_per_sm(int NT) { return NT == 1 ? 2 : 1; }
static constexpr int kRingBudget = 210 * 1024; // dynamic shared memory for the rings of one CTA
static constexpr int kMaxDynSmem = 220 * 1024;  // dynamic shared memory of one CTA, at most

// ------------------------------------------------------------------------------------------
// the kernel
// ------------------------------------------------------------------------------------------
struct RingGeom {
    int slots;        // ring slots per warp
    int slot_bytes;   // weights (bps blocks) [+ activation slices when act_smem == 0]
    int act_row;      // bytes per staged activation row (KS*2 + 16), act_tma == 0
    int act_smem;     // 1: the whole activation [B][act_ld] is copied to shared memory once per CTA
    int act_stride;   // bytes per activation row in shared memory (act_ld*2 + 16)
    int act_tma;      // 1: each block's activation slice is one tensor copy per 64 columns (B rows x
                      // 128 B, 128-byte swizzle) into a 1 KB-aligned region of the slot
    int act_off;      // byte offset of the activation slices in a slot
    int act_box;      // bytes per 64-column box region (B x 128 rounded up to 1 KB)
};

template <int FMT, int GRP, int NT, int EPI>
__global__ void __launch_bounds__(warps_for(NT) * 32, ctas_per_sm(NT))
    gemv_kernel(const GemvArgs args, const RingGeom rg, const __grid_constant__ CUtensorMap act_map) {
    constexpr int WARPS = warps_for(NT);
    constexpr LayoutInfo L = layout_info(FMT, GRP);
    constexpr int R = L.R, KS = L.KS, SUB = L.SUB;
    extern __shared__ __align__(128) uint8_t smem_raw[];
    // 1 KB alignment: the swizzled activation boxes' pattern repeats every 1 KB
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t bars[WARPS][kMaxSlots];
    __shared__ uint64_t act_bar;   // the staged activation rows (act_smem)
    __shared__ float insc_tab[kMaxB * 16];

    pdl_trigger();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = lane & 3;
    const int B = args.B;
    // the ring geometry in registers (read once from the parameter space)
    const int rg_slots = rg.slots, rg_slot_bytes = rg.slot_bytes, rg_act_row = rg.act_row, rg_act_stride = rg.act_stride;
    const bool rg_act_smem = rg.act_smem != 0, rg_act_tma = rg.act_tma != 0;
    const int rg_act_off = rg.act_off, rg_act_box = rg.act_box;

    // ---- worker range -------------------------------------------------------------------
    const long long Wall = (long long)gridDim.x * WARPS;
    const WarpRange wr = warp_range(args.mat, args.nmat, (long long)blockIdx.x * WARPS + warp, Wall);
    const GemvMat& M = wr.M;
    const int f0 = wr.f0, f1 = wr.f1;
    const int bps = L.bps;
    const int nstages = (f1 - f0 + bps - 1) / bps;
    const int KT = M.KT;

    uint8_t* ring = smem + (size_t)warp * rg_slots * rg_slot_bytes;
    uint64_t* bar = bars[warp];
    const int act_rows = B;

    // stage i covers blocks [f0 + i*bps, min(f0 + (i+1)*bps, f1)) and lives in ring slot i mod slots
    auto issue_weights = [&](int i, int slot) {
        const int fb = f0 + i * bps;
        const int nb = min(bps, f1 - fb);
        const uint32_t wbytes = nb * L.block_bytes;
        const uint32_t abytes = rg_act_smem ? 0u : (uint32_t)(nb * act_rows * KS * 2);   // the same for both forms
        mbar_arrive_expect_tx(&bar[slot], wbytes + abytes);
        bulk_g2s(ring + (size_t)slot * rg_slot_bytes, M.w + (size_t)fb * L.block_bytes, wbytes, &bar[slot]);
    };
    int act_kt = f0 % KT;   // k-step of the next block whose activation slice is issued
    auto issue_act = [&](int i, int slot) {
        const int nb = min(bps, f1 - (f0 + i * bps));
        uint8_t* abase = ring + (size_t)slot * rg_slot_bytes + rg_act_off;
        for (int j = 0; j < nb; ++j) {
            if (rg_act_tma) {
                for (int st = 0; st < SUB; ++st)
                    tma_load_2d(abase + (j * SUB + st) * rg_act_box, &act_map, act_kt * KS + 64 * st, 0, &bar[slot]);
            } else {
                for (int b = 0; b < act_rows; ++b)
                    bulk_g2s(abase + (j * act_rows + b) * rg_act_row,
                             args.act + (size_t)b * args.act_ld + (size_t)act_kt * KS, KS * 2, &bar[slot]);
            }
            if (++act_kt == KT) act_kt = 0;
        }
    };

    if (lane == 0) {
        for (int s = 0; s < rg_slots; ++s) mbar_init(&bar[s], 1);
        if (warp == 0) mbar_init(&act_bar, 1);
        fence_mbar_init();
        for (int i = 0; i < nstages && i < rg_slots; ++i) issue_weights(i, i);
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
    // the activation rows to shared memory (rows padded by 16 bytes): up to 32 KB by the threads'
    // own loads (they overlap the weight copies already queued on the copy engine); beyond that
    // one bulk copy per row
    uint8_t* act_s = smem + (size_t)WARPS * rg_slots * rg_slot_bytes;
    const bool act_bulk = rg_act_smem && B * args.act_ld * 2 > 32 * 1024;
    __syncthreads();   // act_bar initialised
    if (act_bulk && threadIdx.x == 0) {
        mbar_arrive_expect_tx(&act_bar, (uint32_t)(B * args.act_ld * 2));
        for (int b = 0; b < B; ++b)
            bulk_g2s(act_s + (size_t)b * rg_act_stride, args.act + (size_t)b * args.act_ld, (uint32_t)(args.act_ld * 2),
                     &act_bar);
    } else if (rg_act_smem) {
        const int row16 = args.act_ld / 8;   // 16-byte chunks per row
        for (int idx = threadIdx.x; idx < B * row16; idx += WARPS * 32) {
            const int b = idx / row16, c = idx % row16;
            *reinterpret_cast<uint4*>(act_s + (size_t)b * rg_act_stride + c * 16) =
                *reinterpret_cast<const uint4*>(args.act + (size_t)b * args.act_ld + (size_t)c * 8);
        }
    }
    bool act_ok = true;
    if (act_bulk) act_ok = mbar_wait(&act_bar, 0, args.status);
    __syncthreads();

    if (lane == 0 && !rg_act_smem)
        for (int i = 0; i < nstages && i < rg_slots; ++i) issue_act(i, i);

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

    zero_acc();
    bool alive = act_ok;
    int cur_u = f0 / KT, kt = f0 % KT;   // unit and k-step of the next block to consume
    bool pending = false;                 // acc holds contributions of cur_u not yet flushed
    int slot = 0;
    uint32_t phase = 0;
    float sc[NT][2];
    int sc_next = kt;   // first k-step at which sc must be (re)loaded
    for (int i = 0; i < nstages; ++i) {
        if (!mbar_wait(&bar[slot], phase, args.status)) { alive = false; break; }
        const uint8_t* base = ring + (size_t)slot * rg_slot_bytes;
        const int nb = min(bps, f1 - (f0 + i * bps));
        for (int jb = 0; jb < nb; ++jb) {
            const uint8_t* blk = base + jb * L.block_bytes;
            const uint8_t* arow0 = base + rg_act_off + (size_t)jb * (rg_act_tma ? SUB * rg_act_box : act_rows * rg_act_row);
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
            if (rg_act_smem) {
                const uint8_t* abase = act_s + (size_t)kt * KS * 2;
                consume_block<FMT, GRP, NT, EPI == EPI_ARGMAX>(blk, [&](int b) { return abase + (size_t)b * rg_act_stride; }, B,
                                                              lane, sc, acc);
            } else if (rg_act_tma) {
                consume_block_swz<FMT, GRP, NT, EPI == EPI_ARGMAX>(blk, arow0, rg_act_box, B, lane, sc, acc);
            } else {
                consume_block<FMT, GRP, NT, EPI == EPI_ARGMAX>(blk, [&](int b) { return arow0 + b * rg_act_row; }, B, lane,
                                                              sc, acc);
            }
            pending = true;
            if (++kt == KT) {   // the unit's last k-step: finish it (or hand over the partial)
                unit_flush<FMT, GRP, NT, EPI>(args, wr, cur_u, acc, best, lane);
                zero_acc();
                pending = false;
                kt = 0;
                ++cur_u;
                if (ng > 1) sc_next = 0;
            }
        }
        __syncwarp();
        if (lane == 0 && i + rg_slots < nstages) {
            fence_proxy_async();
            issue_weights(i + rg_slots, slot);
            if (!rg_act_smem) issue_act(i + rg_slots, slot);
        }
        if (++slot == rg_slots) { slot = 0; phase ^= 1u; }
    }
    if (alive && pending) unit_flush<FMT, GRP, NT, EPI>(args, wr, cur_u, acc, best, lane);

    if constexpr (EPI == EPI_ARGMAX) argmax_publish<NT>(args, wr.m, best, Wall, lane);
}

template <int FMT, int GRP, int NT, int EPI>
cudaError_t launch_t(const GemvLaunch& Lh, const GemvArgs& a, cudaStream_t s) {
    constexpr LayoutInfo L = layout_info(FMT, GRP);
    RingGeom rg{};
    CUtensorMap act_map;
    memset(&act_map, 0, sizeof(act_map));
    rg.act_row = L.KS * 2 + 16;
    rg.act_stride = a.act_ld * 2 + 16;
    const int act_total = a.B * rg.act_stride;
    const int wbytes = L.bps * L.block_bytes;
    constexpr int WARPS = warps_for(NT);
    // the whole activation goes to shared memory once per CTA when it fits beside rings of two
    // weight-only slots per warp (one CTA per SM for 9..16 rows leaves room for ~140 KB of
    // activations: 16 rows of K = 4480); otherwise each block's activation slice rides in the ring
    const int act_room = NT == 1 ? 32 * 1024 : kMaxDynSmem - WARPS * 2 * round_up(wbytes, 128);
    rg.act_smem = act_total <= act_room;
    // otherwise, for 9..16 rows (one CTA per SM, room for 1 KB-aligned slices), each block's slice
    // is one tensor copy per 64 columns instead of a copy per row (rows keep the per-row copies,
    // as does any shape whose tensor map cannot be made)
    rg.act_tma = NT == 2 && !rg.act_smem &&
                 tma_map_2d(&act_map, a.act, a.B, a.act_ld, a.act_ld, 64, a.B, act_f16_for(FMT), CU_TENSOR_MAP_SWIZZLE_128B);
    if (rg.act_tma) {
        rg.act_box = round_up(a.B * 128, 1024);
        rg.act_off = round_up(wbytes, 1024);
        rg.slot_bytes = round_up(rg.act_off + L.bps * L.SUB * rg.act_box, 1024);
    } else {
        rg.act_off = wbytes;
        rg.slot_bytes = round_up(wbytes + (rg.act_smem ? 0 : L.bps * a.B * rg.act_row), 128);
    }
    // CTAs per SM and the ring budget of each (GemvLaunch::shape, up to 8 rows): two CTAs with
    // half the budget each; one CTA with half the budget, leaving room for a CTA of the next
    // launch; one CTA with the whole budget
    const int shape = NT == 1 ? Lh.shape : 0;
    const int cps = shape ? 1 : ctas_per_sm(NT);
    const int share = shape == 2 ? 1 : ctas_per_sm(NT);
    // as many 4 KB-class slots per warp as the budget allows: the bytes in flight per SM
    // (warps x (slots - 1) x slot) must cover HBM latency x per-SM bandwidth (~60-100 KB)
    const int budget = kRingBudget / share - 4096;   // `share` CTAs must fit one SM
    rg.slots = (budget - (rg.act_smem ? act_total : 0)) / (WARPS * rg.slot_bytes);
    if (rg.slots > kMaxSlots) rg.slots = kMaxSlots;
    if (rg.slots < 2) rg.slots = 2;
    const size_t smem = (size_t)WARPS * rg.slots * rg.slot_bytes + (rg.act_smem ? act_total : 0) + 1024;   // + alignment
    if (smem > kMaxDynSmem + 1024) return cudaErrorInvalidValue;
    auto kern = gemv_kernel<FMT, GRP, NT, EPI>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    // shape 1: the largest shared-memory carveout, so that a CTA of the next launch can fit beside
    // this one; the preference stays with the kernel, so once shape 1 has been used in the process
    // the other shapes set it back to the default preference (untouched otherwise)
    static std::atomic<bool> carveout_set{false};
    if (shape == 1) carveout_set.store(true);
    if (e == cudaSuccess && carveout_set.load())
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 shape == 1 ? 100 : (int)cudaSharedmemCarveoutDefault);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(Lh.num_sms * cps);
    cfg.blockDim = dim3(WARPS * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = Lh.pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a, rg, act_map);
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
