// gemv.cu -- dispatch of the streaming GEMV (kernel in gemv_kernel.cuh, one translation unit
// per weight format) and the weight-preparation kernels (quantize / pack / dequantize).
#include "gemv_kernel.cuh"

namespace vc {

static constexpr int kMaxBDispatch = 16;

// ------------------------------------------------------------------------------------------
// host launch
// ------------------------------------------------------------------------------------------
size_t gemv_partials_bytes(int num_sms) { return (size_t)num_sms * kWarps * 2 * (4 * 2 * 128) * sizeof(float); }
size_t gemv_counter_ints() { return 2 * 65536; }

cudaError_t launch_gemv(const GemvLaunch& L, const GemvArgs& a, cudaStream_t s) {
    if (a.B < 1 || a.B > kMaxBDispatch) return cudaErrorInvalidValue;
    switch (L.fmt) {
        case FMT_BF16: return launch_gemv_bf16(L, a, s);
        case FMT_W8: return launch_gemv_w8(L, a, s);
        case FMT_W4: return launch_gemv_w4(L, a, s);
        case FMT_W3: return launch_gemv_w3(L, a, s);
    }
    return cudaErrorInvalidValue;
}

// ------------------------------------------------------------------------------------------
// weight preparation: RTN quantization / bf16 copy / canonical repack into the device layout.
// One thread owns rows (g, g+8) of one 16-row slab for one k-step, so it writes every byte of
// its lanes' words and its metadata record alone (no read-modify-write races).
// ------------------------------------------------------------------------------------------
template <int FMT, int GRP>
__device__ void put_code(uint8_t* out, int KT, int n, int k, uint32_t code) {
    CodePos P = code_pos(FMT, GRP, KT, n, k);
    if constexpr (FMT == FMT_BF16) {
        *reinterpret_cast<uint16_t*>(out + P.off[0]) = (uint16_t)code;
    } else if (P.nparts == 1) {
        uint32_t* w = reinterpret_cast<uint32_t*>(out + P.off[0]);
        *w |= code << P.bit[0];
    } else {
        for (int b = 0; b < 3; ++b) {
            uint32_t* w = reinterpret_cast<uint32_t*>(out + P.off[b]);
            *w |= ((code >> b) & 1u) << P.bit[b];
        }
    }
}

template <int FMT, int GRP>
__device__ uint32_t get_code(const uint8_t* in, int KT, int n, int k) {
    CodePos P = code_pos(FMT, GRP, KT, n, k);
    if constexpr (FMT == FMT_BF16) {
        return *reinterpret_cast<const uint16_t*>(in + P.off[0]);
    } else if (P.nparts == 1) {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(in + P.off[0]);
        constexpr uint32_t mask = (1u << layout_info(FMT, GRP).bits) - 1u;
        return (w >> P.bit[0]) & mask;
    } else {
        uint32_t c = 0;
        for (int b = 0; b < 3; ++b) c |= ((*reinterpret_cast<const uint32_t*>(in + P.off[b]) >> P.bit[b]) & 1u) << b;
        return c;
    }
}

// mode 0: quantize fp32 w; mode 1: bf16 copy; mode 2: canonical packed codes
template <int FMT, int GRP>
__global__ void prepare_kernel(int mode, int N, int K, int NU, int KT, const float* wf, const uint16_t* wb,
                               const uint32_t* cq, const uint16_t* cs, const uint32_t* cz, uint8_t* out) {
    constexpr LayoutInfo L = layout_info(FMT, GRP);
    const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long total = (long long)NU * L.R * 8 * KT;
    if (tid >= total) return;
    const int kt = (int)(tid % KT);
    const long long rest = tid / KT;
    const int g = (int)(rest % 8);
    const long long slab = rest / 8;               // u * R + r
    const int n0 = (int)(slab * 16 + g), n1 = n0 + 8;
    const int k0 = kt * L.KS, k1 = min(K, k0 + L.KS);
    const int Q = (1 << L.bits) - 1;
    const int ngrp = (K + GRP - 1) / GRP;
    uint16_t sbits[2] = {0x3C00, 0x3C00};   // 1.0
    uint32_t zero[2] = {0, 0};
    for (int h = 0; h < 2; ++h) {
        const int n = h ? n1 : n0;
        for (int k = k0; k < k0 + L.KS; ++k) {
            uint32_t code;
            if (FMT == FMT_BF16) {
                code = 0;
                if (n < N && k < K) {
                    if (mode == 1) code = wb[(size_t)n * K + k];
                    else {
                        __nv_bfloat16 bv = __float2bfloat16_rn(wf[(size_t)n * K + k]);
                        code = *reinterpret_cast<uint16_t*>(&bv);
                    }
                }
                put_code<FMT, GRP>(out, KT, n, k, code);
            }
        }
        if (FMT == FMT_BF16) continue;
        // quantization parameters of this row's group (k-step == group)
        float sf = 1.0f;
        uint32_t z = 0;
        if (n < N) {
            if (mode == 0) {
                const float* wr = wf + (size_t)n * K;
                if (FMT == FMT_W8) {
                    float amax = 0.0f;
                    for (int k = k0; k < k1; ++k) amax = fmaxf(amax, fabsf(wr[k]));
                    __half s16 = __float2half_rn(__fdiv_rn(amax, 127.0f));
                    if (__half2float(s16) == 0.0f) s16 = __float2half_rn(1.0f);
                    sbits[h] = *reinterpret_cast<uint16_t*>(&s16);
                    sf = __half2float(s16);
                } else {
                    float mx = wr[k0], mn = wr[k0];
                    for (int k = k0; k < k1; ++k) { mx = fmaxf(mx, wr[k]); mn = fminf(mn, wr[k]); }
                    __half s16 = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), (float)Q));
                    if (__half2float(s16) == 0.0f) s16 = __float2half_rn(1.0f);
                    sbits[h] = *reinterpret_cast<uint16_t*>(&s16);
                    sf = __half2float(s16);
                    int zi = __float2int_rn(__fdiv_rn(-mn, sf));
                    zero[h] = (uint32_t)min(max(zi, 0), Q);
                }
            } else {
                const int grp = k0 / GRP;
                sbits[h] = cs[(size_t)n * ngrp + grp];
                if (FMT != FMT_W8) {
                    const int zw = (ngrp * L.bits + 31) / 32;
                    const long long bo = (long long)grp * L.bits;
                    const uint32_t* zr = cz + (size_t)n * zw;
                    uint64_t v = zr[bo >> 5] >> (bo & 31);
                    if ((bo & 31) + L.bits > 32) v |= (uint64_t)zr[(bo >> 5) + 1] << (32 - (bo & 31));
                    zero[h] = (uint32_t)(v & Q);
                }
            }
        }
        for (int k = k0; k < k0 + L.KS; ++k) {
            uint32_t code;
            if (n >= N || k >= K) {
                code = FMT == FMT_W8 ? 128u : zero[h];   // zero weight
            } else if (mode == 0) {
                const float w = wf[(size_t)n * K + k];
                int c = __float2int_rn(__fdiv_rn(w, sf));
                if (FMT == FMT_W8) code = (uint32_t)(min(max(c, -127), 127) + 128);
                else code = (uint32_t)min(max(c + (int)zero[h], 0), Q);
            } else {
                const int cw = (K * L.bits + 31) / 32;
                const long long bo = (long long)k * L.bits;
                const uint32_t* qr = cq + (size_t)n * cw;
                uint64_t v = qr[bo >> 5] >> (bo & 31);
                if ((bo & 31) + L.bits > 32) v |= (uint64_t)qr[(bo >> 5) + 1] << (32 - (bo & 31));
                const uint32_t raw = (uint32_t)(v & Q);
                code = FMT == FMT_W8 ? ((raw + 128u) & 255u) : raw;   // int8 two's complement -> offset binary
            }
            put_code<FMT, GRP>(out, KT, n, k, code);
        }
    }
    if (FMT == FMT_BF16) return;
    // metadata record of the slab: scale pair g and zero pair g
    CodePos P = code_pos(FMT, GRP, KT, n0, k0);
    *reinterpret_cast<uint16_t*>(out + P.meta + g * 4) = sbits[0];
    *reinterpret_cast<uint16_t*>(out + P.meta + g * 4 + 2) = sbits[1];
    if (FMT == FMT_W4 || FMT == FMT_W3) out[P.meta + 32 + g] = (uint8_t)(zero[0] | (zero[1] << 4));
}

template <int FMT, int GRP>
__global__ void dequant_kernel(int N, int K, int KT, const uint8_t* in, float* out) {
    constexpr LayoutInfo L = layout_info(FMT, GRP);
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (long long)N * K) return;
    const int n = (int)(i / K), k = (int)(i % K);
    const uint32_t c = get_code<FMT, GRP>(in, KT, n, k);
    if (FMT == FMT_BF16) {
        out[i] = __uint_as_float(c << 16);
        return;
    }
    CodePos P = code_pos(FMT, GRP, KT, n, k);
    const float s = __half2float(*reinterpret_cast<const __half*>(in + P.meta + P.g * 4 + P.hi * 2));
    int q;
    if (FMT == FMT_W8) q = (int)c - 128;
    else {
        const uint32_t zb = in[P.meta + 32 + P.g];
        q = (int)c - (int)(P.hi ? (zb >> 4) : (zb & 15u));
    }
    out[i] = s * (float)q;   // exact: fp16 significand x small integer
    (void)L;
}

// dense 16-bit row-major copy out[n][k] (row stride ldo) of a weight in the device layout, for the
// tensor-core GEMMs of the prefill: bf16 weights are copied bit for bit; quantized weights become
// s*(q - z) rounded once to fp16 (f16 = 1, the value the decode GEMV's dequantization produces) or
// to bf16 (f16 = 0)
template <int FMT, int GRP>
__global__ void unpack_kernel(int N, int K, int KT, const uint8_t* in, uint16_t* out, int ldo, int f16) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (long long)N * K) return;
    const int n = (int)(i / K), k = (int)(i % K);
    const uint32_t c = get_code<FMT, GRP>(in, KT, n, k);
    uint16_t bits;
    if (FMT == FMT_BF16) {
        bits = (uint16_t)c;
    } else {
        CodePos P = code_pos(FMT, GRP, KT, n, k);
        const float s = __half2float(*reinterpret_cast<const __half*>(in + P.meta + P.g * 4 + P.hi * 2));
        int q;
        if (FMT == FMT_W8) q = (int)c - 128;
        else {
            const uint32_t zb = in[P.meta + 32 + P.g];
            q = (int)c - (int)(P.hi ? (zb >> 4) : (zb & 15u));
        }
        const float w = s * (float)q;   // exact in fp32
        bits = f16 ? __half_as_ushort(__float2half_rn(w)) : __bfloat16_as_ushort(__float2bfloat16_rn(w));
    }
    out[(size_t)n * ldo + k] = bits;
}

// bf16 weights: one warp per 16-row tile of a block.  Lane (g, t) holds, in its four 16-byte
// words (s = 0..3), rows g and g + 8 at columns 16 t + 4 s + {0..3} (words 0/2: row g, words 1/3:
// row g + 8), so it writes 16 consecutive columns of both rows with two 16-byte stores each.
__global__ void unpack_bf16_tiles_kernel(int N, int K, int KT, int tiles, const uint8_t* in, uint16_t* out, int ldo) {
    constexpr LayoutInfo L = layout_info(FMT_BF16, 64);
    const int warp = (int)((blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5), lane = threadIdx.x & 31;
    if (warp >= tiles) return;
    const int r = warp % L.R, blk = warp / L.R;
    const int u = blk / KT, kt = blk % KT;
    const uint8_t* tile = in + (size_t)blk * L.block_bytes + (size_t)r * L.tile_bytes;
    uint4 v[4];
#pragma unroll
    for (int s = 0; s < 4; ++s) v[s] = *reinterpret_cast<const uint4*>(tile + (s * 32 + lane) * 16);
    const int g = lane >> 2, t = lane & 3;
    const int col = kt * 64 + 16 * t;
    const int row0 = u * 16 * L.R + 16 * r + g;
    const uint4 lo0 = make_uint4(v[0].x, v[0].z, v[1].x, v[1].z), lo1 = make_uint4(v[2].x, v[2].z, v[3].x, v[3].z);
    const uint4 hi0 = make_uint4(v[0].y, v[0].w, v[1].y, v[1].w), hi1 = make_uint4(v[2].y, v[2].w, v[3].y, v[3].w);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int row = row0 + 8 * h;
        if (row >= N) continue;
        uint16_t* dst = out + (size_t)row * ldo + col;
        if (col < K) *reinterpret_cast<uint4*>(dst) = h ? hi0 : lo0;
        if (col + 8 < K) *reinterpret_cast<uint4*>(dst + 8) = h ? hi1 : lo1;
    }
}

template <int FMT, int GRP>
static cudaError_t unp_t(int N, int K, const uint8_t* w, uint16_t* out, int ldo, int f16, cudaStream_t s) {
    MatGeom G = mat_geom(FMT, GRP, N, K);
    const long long total = (long long)N * K;
    unpack_kernel<FMT, GRP><<<(unsigned)((total + 255) / 256), 256, 0, s>>>(N, K, G.KT, w, out, ldo, f16);
    return cudaGetLastError();
}

cudaError_t launch_unpack16(int fmt, int group, int N, int K, const uint8_t* w, uint16_t* out, int ldo, int f16,
                            cudaStream_t s) {
    if (fmt == FMT_BF16 && K % 8 == 0 && ldo % 8 == 0 && (((uintptr_t)out) & 15) == 0) {
        constexpr LayoutInfo L = layout_info(FMT_BF16, 64);
        const MatGeom G = mat_geom(FMT_BF16, 64, N, K);
        const int tiles = G.NU * G.KT * L.R;
        unpack_bf16_tiles_kernel<<<(unsigned)((tiles + 7) / 8), 256, 0, s>>>(N, K, G.KT, tiles, w, out, ldo);
        return cudaGetLastError();
    }
    switch (fmt) {
        case FMT_BF16: return unp_t<FMT_BF16, 64>(N, K, w, out, ldo, f16, s);
        case FMT_W8:
            return group == 128 ? unp_t<FMT_W8, 128>(N, K, w, out, ldo, f16, s)
                                : unp_t<FMT_W8, 64>(N, K, w, out, ldo, f16, s);
        case FMT_W4:
            return group == 128 ? unp_t<FMT_W4, 128>(N, K, w, out, ldo, f16, s)
                                : unp_t<FMT_W4, 64>(N, K, w, out, ldo, f16, s);
        case FMT_W3:
            return group == 128 ? unp_t<FMT_W3, 128>(N, K, w, out, ldo, f16, s)
                                : unp_t<FMT_W3, 64>(N, K, w, out, ldo, f16, s);
    }
    return cudaErrorInvalidValue;
}

template <int FMT, int GRP>
static cudaError_t prep_t(int mode, int N, int K, const float* wf, const uint16_t* wb, const uint32_t* cq,
                          const uint16_t* cs, const uint32_t* cz, uint8_t* out, cudaStream_t s) {
    constexpr LayoutInfo L = layout_info(FMT, GRP);
    MatGeom G = mat_geom(FMT, GRP, N, K);
    cudaError_t e = cudaMemsetAsync(out, 0, (size_t)G.bytes, s);
    if (e != cudaSuccess) return e;
    const long long total = (long long)G.NU * L.R * 8 * G.KT;
    const int tb = 128;
    prepare_kernel<FMT, GRP><<<(unsigned)((total + tb - 1) / tb), tb, 0, s>>>(mode, N, K, G.NU, G.KT, wf, wb, cq, cs, cz,
                                                                             out);
    return cudaGetLastError();
}

static cudaError_t prep(int fmt, int group, int mode, int N, int K, const float* wf, const uint16_t* wb,
                        const uint32_t* cq, const uint16_t* cs, const uint32_t* cz, uint8_t* out, cudaStream_t s) {
    switch (fmt) {
        case FMT_BF16: return prep_t<FMT_BF16, 64>(mode, N, K, wf, wb, cq, cs, cz, out, s);
        case FMT_W8:
            return group == 128 ? prep_t<FMT_W8, 128>(mode, N, K, wf, wb, cq, cs, cz, out, s)
                                : prep_t<FMT_W8, 64>(mode, N, K, wf, wb, cq, cs, cz, out, s);
        case FMT_W4:
            return group == 128 ? prep_t<FMT_W4, 128>(mode, N, K, wf, wb, cq, cs, cz, out, s)
                                : prep_t<FMT_W4, 64>(mode, N, K, wf, wb, cq, cs, cz, out, s);
        case FMT_W3:
            return group == 128 ? prep_t<FMT_W3, 128>(mode, N, K, wf, wb, cq, cs, cz, out, s)
                                : prep_t<FMT_W3, 64>(mode, N, K, wf, wb, cq, cs, cz, out, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_quantize(int fmt, int group, int N, int K, const float* w, uint8_t* out, cudaStream_t s) {
    return prep(fmt, group, 0, N, K, w, nullptr, nullptr, nullptr, nullptr, out, s);
}
cudaError_t launch_pack_bf16(int N, int K, const uint16_t* w, uint8_t* out, cudaStream_t s) {
    return prep(FMT_BF16, 64, 1, N, K, nullptr, w, nullptr, nullptr, nullptr, out, s);
}
cudaError_t launch_pack_canonical(int fmt, int group, int N, int K, const uint32_t* q, const uint16_t* scales,
                                  const uint32_t* zeros, uint8_t* out, cudaStream_t s) {
    return prep(fmt, group, 2, N, K, nullptr, nullptr, q, scales, zeros, out, s);
}

template <int FMT, int GRP>
static cudaError_t deq_t(int N, int K, const uint8_t* w, float* out, cudaStream_t s) {
    MatGeom G = mat_geom(FMT, GRP, N, K);
    const long long total = (long long)N * K;
    dequant_kernel<FMT, GRP><<<(unsigned)((total + 255) / 256), 256, 0, s>>>(N, K, G.KT, w, out);
    return cudaGetLastError();
}

cudaError_t launch_dequant(int fmt, int group, int N, int K, const uint8_t* w, float* out, cudaStream_t s) {
    switch (fmt) {
        case FMT_BF16: return deq_t<FMT_BF16, 64>(N, K, w, out, s);
        case FMT_W8: return group == 128 ? deq_t<FMT_W8, 128>(N, K, w, out, s) : deq_t<FMT_W8, 64>(N, K, w, out, s);
        case FMT_W4: return group == 128 ? deq_t<FMT_W4, 128>(N, K, w, out, s) : deq_t<FMT_W4, 64>(N, K, w, out, s);
        case FMT_W3: return group == 128 ? deq_t<FMT_W3, 128>(N, K, w, out, s) : deq_t<FMT_W3, 64>(N, K, w, out, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace vc
