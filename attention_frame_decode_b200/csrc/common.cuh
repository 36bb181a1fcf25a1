// common.cuh -- small device helpers shared by the sm_100a kernels of libvc.
//
// PTX wrappers: mbarrier, 1-D bulk copies (cp.async.bulk, the TMA engine's
// untiled form), programmatic dependent launch, warp MMA, half/bfloat
// conversions.  All waits are bounded: a wait that exceeds its iteration
// budget records an error in the caller's device status word and returns
// false instead of spinning forever.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define VC_DEV __device__ __forceinline__

// device status bits VC_DEV_* (OR-ed into the caller's status word) come from vc.h
#include "../../include/vc.h"

static constexpr long long kWaitLimit = 1ll << 22;   // try_wait polls before giving up

// ------------------------------------------------------------------------------------------
// programmatic dependent launch
// ------------------------------------------------------------------------------------------
VC_DEV void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
VC_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ------------------------------------------------------------------------------------------
// mbarrier + bulk copy
// ------------------------------------------------------------------------------------------
VC_DEV uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

VC_DEV void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
VC_DEV void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
VC_DEV void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

VC_DEV void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

VC_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

VC_DEV bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// bounded wait; returns false (and flags VC_DEV_TIMEOUT) if the phase never completes
VC_DEV bool mbar_wait(uint64_t* bar, uint32_t parity, int* status) {
    for (long long i = 0; i < kWaitLimit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    if (status) atomicOr(status, VC_DEV_TIMEOUT);
    return false;
}

// global -> shared bulk copy completing on an mbarrier (16-byte aligned, size % 16 == 0)
VC_DEV void bulk_g2s(void* dst_smem, const void* src_gmem, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst_smem)),
        "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// ------------------------------------------------------------------------------------------
// warp MMA m16n8k16, fp32 accumulate in place (d += a b).  The accumulator is a read-write operand
// and the asm has no side effects, so the compiler keeps d in place and schedules freely.
// ------------------------------------------------------------------------------------------
VC_DEV void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
VC_DEV void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// ------------------------------------------------------------------------------------------
// bit tricks
// ------------------------------------------------------------------------------------------
template <uint32_t LUT>
VC_DEV uint32_t lop3(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, %4;" : "=r"(d) : "r"(a), "r"(b), "r"(c), "n"(LUT));
    return d;
}
// (a & b) | c
VC_DEV uint32_t and_or(uint32_t a, uint32_t b, uint32_t c) { return lop3<(0xF0 & 0xCC) | 0xAA>(a, b, c); }

VC_DEV uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

VC_DEV uint32_t h2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
VC_DEV __half2 u32_as_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

VC_DEV uint32_t hsub2_u32(uint32_t a, uint32_t b) { return h2_as_u32(__hsub2(u32_as_h2(a), u32_as_h2(b))); }
VC_DEV uint32_t hfma2_u32(uint32_t a, uint32_t b, uint32_t c) {
    return h2_as_u32(__hfma2(u32_as_h2(a), u32_as_h2(b), u32_as_h2(c)));
}


// orderable key for float max with lowest-index tie-break: larger key <=> larger value, then smaller index
VC_DEV unsigned long long argmax_key(float v, int idx) {
    uint32_t u = __float_as_uint(v);
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ((unsigned long long)u << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)idx);
}
VC_DEV int argmax_key_index(unsigned long long k) { return (int)(0xFFFFFFFFu - (uint32_t)(k & 0xFFFFFFFFull)); }

VC_DEV float silu_f(float x) { return x / (1.0f + __expf(-x)); }
VC_DEV float softplus_f(float x) { return x > 20.0f ? x : log1pf(__expf(x)); }

// store an fp32 value in the activation type a consumer's MMA wants; the value is first rounded
// to bf16 (the storage point), then widened to fp16 when the consumer is a quantized matrix
// (exact for |v| in fp16's normal range)
template <bool F16>
VC_DEV uint16_t act_bits(float v) {
    __nv_bfloat16 b = __float2bfloat16_rn(v);
    if constexpr (F16) {
        __half h = __float2half_rn(__bfloat162float(b));
        return *reinterpret_cast<uint16_t*>(&h);
    } else {
        return *reinterpret_cast<uint16_t*>(&b);
    }
}

// fp32 vector reduction into global memory (performed at L2), no return value
VC_DEV void red_add_v4(float* p, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}

VC_DEV float bf16_bits_to_f(uint16_t u) { return __uint_as_float((uint32_t)u << 16); }

VC_DEV float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
VC_DEV float warp_max(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
