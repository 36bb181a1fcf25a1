// gemm_tc.cu -- tcgen05 GEMM for the prefill projections (dense contraction over the frames).
//
// C[M][N] = A[M][K] . W[N][K]^T, 16-bit x 16-bit -> fp32 in tensor memory (TMEM).
// Persistent: one CTA per SM walks the 128 x 256 output tiles (M-tile fastest, so the CTAs
// resident together share a few W column tiles, each streamed from HBM once, while the
// activation rows stay in L2).  Per CTA:
//   warp 0 (one thread): TMA producer over a 4-stage ring of 64-wide k-blocks (128-byte swizzle,
//           each CTA loads its own tiles), across tile boundaries;
//   warp 1: allocates 512 TMEM columns = two 128 x 256 fp32 accumulators; one thread issues
//           tcgen05.mma (M=128, N=256, K=16, 4 per k-block) into accumulator (tile & 1),
//           commits each stage back to the producer and each finished tile to the epilogue;
//   warps 2-5: epilogue; each reads its 32 TMEM lanes (rows) with tcgen05.ld, applies the fused
//           epilogue (row scale of the pre-RMSNorm, squared ReLU, residual add, q/k/v split into
//           the KV cache), stores, and hands the accumulator back -- while the MMAs of the next
//           tile already run into the other accumulator.
// Every mbarrier wait is bounded; a timeout sets the status word and the CTA still frees TMEM.
#include <cuda.h>

#include "common.cuh"
#include "gemm_tc.cuh"
#include "tc.cuh"

namespace vc {

static constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
static constexpr int A_BYTES = BM * BK * 2, B_BYTES = BN * BK * 2, STAGE_BYTES = A_BYTES + B_BYTES;
static constexpr int GEMM_THREADS = 192;
static constexpr int TMEM_COLS = 512;   // two accumulators of BN fp32 columns

template <bool F16>
VC_DEV constexpr uint32_t idesc() {
    return umma_idesc(!F16, false, BM, BN);
}

template <int EPI, bool F16>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW, const GemmArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t full[STAGES], empty[STAGES], acc_full[2], acc_empty[2];
    __shared__ uint32_t tmem_base;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int mt = (a.M + BM - 1) / BM;
    const int tiles = mt * ((a.N + BN - 1) / BN);
    const int KB = (a.K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 128);
        }
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base, TMEM_COLS);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;

    if (warp == 0) {
        if (lane == 0) {
            int it = 0;   // k-blocks issued by this CTA so far
            bool ok = true;
            for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
                const int n0 = (tile / mt) * BN, m0 = (tile % mt) * BM;
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const int s = it % STAGES;
                    if (it >= STAGES && !mbar_wait(&empty[s], (uint32_t)(((it / STAGES) - 1) & 1), a.status)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
                    tma_load_2d(smem + s * STAGE_BYTES, &tmA, kb * BK, m0, &full[s]);
                    tma_load_2d(smem + s * STAGE_BYTES + A_BYTES, &tmW, kb * BK, n0, &full[s]);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int it = 0, lt = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x, ++lt) {
                const int b = lt & 1;
                // the epilogue has drained this accumulator (its use two tiles ago)
                if (lt >= 2 && !mbar_wait(&acc_empty[b], (uint32_t)(((lt >> 1) - 1) & 1), a.status)) break;
                tc_fence_after();
                const uint32_t dacc = tmem + (uint32_t)(b * BN);
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const int s = it % STAGES;
                    if (!mbar_wait(&full[s], (uint32_t)((it / STAGES) & 1), a.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t abase = smem_u32(smem + s * STAGE_BYTES), bbase = abase + A_BYTES;
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        tc_mma(dacc, desc_sw128(abase + k * 32), desc_sw128(bbase + k * 32), idesc<F16>(),
                               (kb | k) != 0);
                    tc_commit(&empty[s]);
                }
                tc_commit(&acc_full[b]);   // arrives when every MMA of the tile has completed
            }
        }
    } else {
        // epilogue: warp w reads TMEM lanes 32*(w%4) .. +31 = tile rows
        const int quarter = warp & 3;
        int lt = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++lt) {
            const int b = lt & 1;
            const int n0 = (tile / mt) * BN, m0 = (tile % mt) * BM;
            const int row = m0 + quarter * 32 + lane;
            const bool ready = mbar_wait(&acc_full[b], (uint32_t)((lt >> 1) & 1), a.status);
            tc_fence_after();
            if (!ready) break;
            const float rs = (a.row_scale && row < a.M) ? a.row_scale[row] : 1.0f;
            for (int c0 = 0; c0 < BN; c0 += 32) {
                float v[32];
                tc_ld32(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(b * BN + c0), v);
                if (row >= a.M) continue;
                const int col0 = n0 + c0;
                if constexpr (EPI == GE_F32) {
                    float* dst = a.out_f32 + (size_t)row * a.ldo32 + col0;
                    if (col0 + 32 <= a.N && (((uintptr_t)dst) & 15) == 0) {
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            reinterpret_cast<float4*>(dst)[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                    } else {
                        for (int j = 0; j < 32; ++j)
                            if (col0 + j < a.N) dst[j] = v[j];
                    }
                } else if constexpr (EPI == GE_RESID) {
                    float* dst = a.out_f32 + (size_t)row * a.ldo32 + col0;
                    if (col0 + 32 <= a.N && (((uintptr_t)dst) & 15) == 0) {
                        float4 r4[8];
#pragma unroll
                        for (int q = 0; q < 8; ++q) r4[q] = reinterpret_cast<const float4*>(dst)[q];
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            reinterpret_cast<float4*>(dst)[q] = make_float4(r4[q].x + v[4 * q], r4[q].y + v[4 * q + 1],
                                                                           r4[q].z + v[4 * q + 2], r4[q].w + v[4 * q + 3]);
                    } else {
                        for (int j = 0; j < 32; ++j)
                            if (col0 + j < a.N) dst[j] += v[j];
                    }
                } else if constexpr (EPI == GE_QKV) {
                    const int qrows = a.Hq * a.Dh;
                    for (int j = 0; j < 32; ++j) {
                        const int col = col0 + j;
                        if (col >= a.N) break;
                        const uint16_t bits = act_bits<false>(v[j] * rs);
                        if (col < qrows) {
                            a.out[(size_t)row * a.ldo + col] = bits;
                        } else {
                            const int rr = col - qrows, kvsel = rr / (a.Hk * a.Dh);
                            const int jj = (rr % (a.Hk * a.Dh)) / a.Dh, d = rr % a.Dh;
                            uint16_t* cache = kvsel == 0 ? a.kcache : a.vcache;
                            cache[((size_t)jj * a.cap + a.t0 + row) * a.Dh + d] = bits;
                        }
                    }
                } else {
                    uint32_t packed[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        float x0 = v[2 * j] * rs, x1 = v[2 * j + 1] * rs;
                        if constexpr (EPI == GE_RELU2) {
                            x0 = fmaxf(x0, 0.0f); x0 *= x0;
                            x1 = fmaxf(x1, 0.0f); x1 *= x1;
                        }
                        packed[j] = (EPI == GE_RELU2 && a.out_f16)
                                        ? ((uint32_t)act_bits<true>(x0) | ((uint32_t)act_bits<true>(x1) << 16))
                                        : ((uint32_t)act_bits<false>(x0) | ((uint32_t)act_bits<false>(x1) << 16));
                    }
                    uint16_t* dst = a.out + (size_t)row * a.ldo + col0;
                    if (col0 + 32 <= a.N && (((uintptr_t)dst) & 15) == 0) {
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            reinterpret_cast<uint4*>(dst)[q] =
                                make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
                    } else {
                        for (int j = 0; j < 32 && col0 + j < a.N; ++j)
                            dst[j] = (uint16_t)(packed[j / 2] >> (16 * (j & 1)));
                    }
                }
            }
            // accumulator b may take the tile after next
            tc_fence_before();
            mbar_arrive(&acc_empty[b]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ------------------------------------------------------------------------------------------
// host: tensor maps and launch
// ------------------------------------------------------------------------------------------
// 2-D 16-bit tensor map over rows x cols (row stride ld elements), box 64 x box_rows, 128 B swizzle
static bool make_map(CUtensorMap* map, const void* base, int rows, int cols, int ld, int box_rows, bool f16) {
    return tma_map_2d(map, base, rows, cols, ld, BK, box_rows, f16, CU_TENSOR_MAP_SWIZZLE_128B);
}

template <int EPI, bool F16>
static cudaError_t launch_t(const CUtensorMap& ma, const CUtensorMap& mw, const GemmArgs& a, cudaStream_t s) {
    const size_t smem = (size_t)STAGES * STAGE_BYTES + 1024;
    auto kern = gemm_tc_kernel<EPI, F16>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
        if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    }
    const int tiles = ((a.N + BN - 1) / BN) * ((a.M + BM - 1) / BM);
    dim3 grid((unsigned)(tiles < sms ? tiles : sms));
    kern<<<grid, GEMM_THREADS, smem, s>>>(ma, mw, a);
    return cudaGetLastError();
}

cudaError_t launch_gemm_tc(int epi, const GemmArgs& a, cudaStream_t s) {
    // TMA: 16-byte aligned bases, row strides a multiple of 16 bytes, K a multiple of 8 elements
    if ((((uintptr_t)a.A) & 15) || (((uintptr_t)a.W) & 15) || (a.lda % 8) || (a.ldw % 8) || (a.K % 8) || a.M < 1 ||
        a.N < 1 || a.K < 1)
        return cudaErrorInvalidValue;
    CUtensorMap ma, mw;
    const bool f16 = a.f16 != 0;
    if (!make_map(&ma, a.A, a.M, a.K, a.lda, BM, f16) || !make_map(&mw, a.W, a.N, a.K, a.ldw, BN, f16))
        return cudaErrorInvalidValue;
    if (f16) {
        switch (epi) {
            case GE_F32: return launch_t<GE_F32, true>(ma, mw, a, s);
            case GE_ROWSCALE: return launch_t<GE_ROWSCALE, true>(ma, mw, a, s);
            case GE_RELU2: return launch_t<GE_RELU2, true>(ma, mw, a, s);
            case GE_RESID: return launch_t<GE_RESID, true>(ma, mw, a, s);
            case GE_QKV: return launch_t<GE_QKV, true>(ma, mw, a, s);
        }
    } else {
        switch (epi) {
            case GE_F32: return launch_t<GE_F32, false>(ma, mw, a, s);
            case GE_ROWSCALE: return launch_t<GE_ROWSCALE, false>(ma, mw, a, s);
            case GE_RELU2: return launch_t<GE_RELU2, false>(ma, mw, a, s);
            case GE_RESID: return launch_t<GE_RESID, false>(ma, mw, a, s);
            case GE_QKV: return launch_t<GE_QKV, false>(ma, mw, a, s);
        }
    }
    return cudaErrorInvalidValue;
}

}  // namespace vc
