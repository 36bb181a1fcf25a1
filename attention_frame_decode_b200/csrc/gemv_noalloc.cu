// gemv_noalloc.cu -- the decode step's streaming GEMV with its scratch in a static device array.
//
// vc_debug_gemv needs a caller-provided scratch buffer (stream-K partial sums and per-unit
// arrival counters).  Some callers cannot call cudaMalloc to provide one: a per-frame real-time
// loop, where cudaMalloc / cudaFree can synchronize the device and stall the frame; and hosts
// whose device memory is owned by another allocator (a framework's caching pool) that hands out
// no raw buffers.  vc_debug_gemv_noalloc serves them: the same kernel, launched on at most
// kStaticSms SMs' worth of CTAs, with its scratch in g_gemv_scratch below, a fixed-size array in
// the module's device image.  Nothing here calls cudaMalloc, cudaFree or an allocating routine.
//
// What must start at zero: the counters and the status word (the ints after the partial sums).
// Static device memory is zero when the module loads, and every launch returns each counter it
// uses to zero (the last contributor to a unit resets it), so they stay zero between calls.  The
// partial sums are written before they are read and need no initial value.  The status word
// collects the launches' device-side conditions (VC_DEV_TIMEOUT when a bounded wait for a weight
// copy gave up); vc_gemv_noalloc_status reads it.  A launch that timed out leaves counters
// non-zero, so results of later calls are not valid until vc_gemv_noalloc_reset clears the
// counters and the status word (a device memset; nothing is allocated).
//
// One array serves every call in the process on a device: calls whose executions overlap (on
// different streams, or from different host threads without ordering) race on it and give wrong
// results.  Callers order them.
#include "../../include/vc.h"
#include "gemv.cuh"
#include "layout.cuh"

namespace vc {
vc_status record_cuda_failure(cudaError_t e, const char* where);
}

using namespace vc;

namespace {

constexpr int kStaticSms = 32;                             // grid cap of the no-alloc launches
constexpr size_t kPartialBytes = (size_t)4 << 20;          // 4 MiB of stream-K partial sums
constexpr int kCounterInts = 65536;                        // arrival counters: units of 16*R rows
constexpr size_t kStatusOffset = kPartialBytes + (size_t)kCounterInts * sizeof(int);
// partial sums, counters, the status word (padded to 256 bytes): 4.25 MiB + 256 B
constexpr size_t kScratchBytes = kStatusOffset + 256;

static __device__ __align__(256) unsigned char g_gemv_scratch[kScratchBytes];

// The device address of g_gemv_scratch on the current device.  It is looked up on every call
// (a cheap runtime query that allocates nothing), so a device reset that reloads the module
// does not leave a stale address behind.
vc_status scratch_for_current_device(void** out) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress((void**)&p, g_gemv_scratch);
    if (e != cudaSuccess || !p)
        return record_cuda_failure(e != cudaSuccess ? e : cudaErrorUnknown, "cudaGetSymbolAddress(g_gemv_scratch)");
    *out = p;
    return VC_OK;
}

}  // namespace

extern "C" size_t vc_gemv_noalloc_scratch_bytes(void) { return kScratchBytes; }

extern "C" vc_status vc_debug_gemv_noalloc(const vc_qmat* w, const void* act, int act_ld, int B, float* out,
                                           vc_stream_t stream) {
    if (!w || !w->data || !act || !out || ((uintptr_t)act & 15u)) return VC_ERR_INVALID_ARG;
    const bool fmt_ok = w->fmt == VC_W_BF16 || ((w->fmt >= 1 && w->fmt <= 3) && (w->group == 64 || w->group == 128));
    if (!fmt_ok || w->N <= 0 || w->K <= 0 || B < 1 || B > 16) return VC_ERR_INVALID_ARG;
    if (act_ld % 128 || act_ld < round_up(w->K, 128)) return VC_ERR_INVALID_ARG;
    const int group = w->fmt == VC_W_BF16 ? 64 : w->group;
    // sizes beyond the static scratch: more row units than counters
    if (mat_geom(w->fmt, group, w->N, w->K).NU > kCounterInts) return VC_ERR_CAPACITY;
    int dev = 0, sms = kStaticSms;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return record_cuda_failure(e, "cudaDeviceGetAttribute");
    const int grid_sms = sms < kStaticSms ? sms : kStaticSms;
    if (gemv_partials_bytes(grid_sms) > kPartialBytes) return VC_ERR_CAPACITY;
    void* scratch = nullptr;
    vc_status st = scratch_for_current_device(&scratch);
    if (st != VC_OK) return st;
    GemvArgs a{};
    a.nmat = 1;
    const MatGeom G = mat_geom(w->fmt, group, w->N, w->K);
    a.mat[0] = GemvMat{(const uint8_t*)w->data, w->N, w->K, G.NU, G.KT};
    a.act = (const uint16_t*)act;
    a.act_ld = act_ld;
    a.B = B;
    a.tap = out;
    a.tap_ld = w->N;
    a.partials = (float*)scratch;
    a.counters = (int*)((unsigned char*)scratch + kPartialBytes);
    a.status = (int*)((unsigned char*)scratch + kStatusOffset);
    GemvLaunch L{};
    L.fmt = w->fmt;
    L.group = group;
    L.epi = EPI_STORE;
    L.num_sms = grid_sms;
    L.pdl = 0;
    e = launch_gemv(L, a, (cudaStream_t)stream);
    if (e != cudaSuccess) return record_cuda_failure(e, "vc_debug_gemv_noalloc launch");
    return VC_OK;
}

extern "C" vc_status vc_gemv_noalloc_status(int32_t* status, vc_stream_t stream) {
    if (!status) return VC_ERR_INVALID_ARG;
    void* scratch = nullptr;
    vc_status st = scratch_for_current_device(&scratch);
    if (st != VC_OK) return st;
    cudaError_t e = cudaMemcpyAsync(status, (unsigned char*)scratch + kStatusOffset, sizeof(int32_t),
                                    cudaMemcpyDeviceToHost, (cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return record_cuda_failure(e, "vc_gemv_noalloc_status");
    return VC_OK;
}

extern "C" vc_status vc_gemv_noalloc_reset(vc_stream_t stream) {
    void* scratch = nullptr;
    vc_status st = scratch_for_current_device(&scratch);
    if (st != VC_OK) return st;
    const cudaError_t e = cudaMemsetAsync((unsigned char*)scratch + kPartialBytes, 0, kScratchBytes - kPartialBytes,
                                          (cudaStream_t)stream);
    if (e != cudaSuccess) return record_cuda_failure(e, "vc_gemv_noalloc_reset");
    return VC_OK;
}
