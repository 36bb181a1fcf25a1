/*
 * synth.c -- seeded, counter-based generators for synthetic inputs.
 *
 * This module produces the random weights, states and frame inputs that both
 * the CUDA library's tests/benchmark and the CPU oracle consume.  It holds
 * none of the model's arithmetic: only random numbers and their rounding to
 * the storage type a tensor is declared in (bf16 / fp32).
 *
 * Generator (published definitions, written out here):
 *   - SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
 *     generators", OOPSLA 2014): the output function
 *        z += 0x9e3779b97f4a7c15;
 *        z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9;
 *        z = (z ^ (z >> 27)) * 0x94d049bb133111eb;
 *        return z ^ (z >> 31);
 *     used in counter mode: word i of stream (seed, tensor_id) is the output
 *     function applied to key + (i + 1) * 0x9e3779b97f4a7c15, where the key is
 *     the finalizer applied to seed and tensor_id.  Any element can therefore
 *     be regenerated on its own, in any order, by any thread.
 *   - Uniform [0,1): the top 53 bits of a word times 2^-53.
 *   - Normal: Box-Muller (1958) on the pair (u1, u2) drawn from words 2p and
 *     2p+1; element 2p takes r*cos(2*pi*u2), element 2p+1 takes r*sin(...),
 *     r = sqrt(-2 ln(1 - u1)).
 *
 * All functions are deterministic for a given (seed, tensor_id) and fill
 * [0, n) in parallel with OpenMP.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define GOLDEN 0x9e3779b97f4a7c15ULL

static inline uint64_t fin64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
    z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
    return z ^ (z >> 31);
}

static inline uint64_t stream_key(uint64_t seed, uint64_t tensor_id) {
    return fin64(fin64(seed + GOLDEN) ^ (tensor_id * 0xd1b54a32d192ed03ULL + 0x8cb92ba72f3d8dd7ULL));
}

static inline uint64_t word_at(uint64_t key, uint64_t i) { return fin64(key + (i + 1) * GOLDEN); }

static inline double unif01(uint64_t w) { return (double)(w >> 11) * (1.0 / 9007199254740992.0); }

/* round-to-nearest-even fp32 -> bf16 bit pattern (finite inputs) */
static inline uint16_t f32_to_bf16_bits(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

void synth_uniform_u64(uint64_t seed, uint64_t tensor_id, uint64_t n, uint64_t* out) {
    uint64_t key = stream_key(seed, tensor_id);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i) out[i] = word_at(key, (uint64_t)i);
}

/* fills one Box-Muller pair at a time (elements 2p and 2p+1) */
#define NORMAL_FILL(STORE)                                                          \
    uint64_t key = stream_key(seed, tensor_id);                                     \
    _Pragma("omp parallel for schedule(static)")                                    \
    for (int64_t p = 0; p < (int64_t)((n + 1) / 2); ++p) {                          \
        double u1 = unif01(word_at(key, 2 * (uint64_t)p));                          \
        double u2 = unif01(word_at(key, 2 * (uint64_t)p + 1));                      \
        double r = sqrt(-2.0 * log(1.0 - u1));                                      \
        double t = 6.283185307179586476925286766559 * u2;                           \
        uint64_t i0 = 2 * (uint64_t)p;                                              \
        STORE(i0, mean + std * r * cos(t));                                         \
        if (i0 + 1 < n) STORE(i0 + 1, mean + std * r * sin(t));                     \
    }

void synth_normal_f32(uint64_t seed, uint64_t tensor_id, uint64_t n, double mean, double std, float* out) {
#define ST_F32(i, v) out[i] = (float)(v)
    NORMAL_FILL(ST_F32)
#undef ST_F32
}

void synth_normal_bf16(uint64_t seed, uint64_t tensor_id, uint64_t n, double mean, double std, uint16_t* out) {
#define ST_BF16(i, v) out[i] = f32_to_bf16_bits((float)(v))
    NORMAL_FILL(ST_BF16)
#undef ST_BF16
}

void synth_uniform_f32(uint64_t seed, uint64_t tensor_id, uint64_t n, double lo, double hi, float* out) {
    uint64_t key = stream_key(seed, tensor_id);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i)
        out[i] = (float)(lo + (hi - lo) * unif01(word_at(key, (uint64_t)i)));
}

/* integers uniform on [lo, hi] inclusive (modulo bias is < 2^-40 for the ranges used) */
void synth_uniform_i32(uint64_t seed, uint64_t tensor_id, uint64_t n, int32_t lo, int32_t hi, int32_t* out) {
    uint64_t key = stream_key(seed, tensor_id);
    uint64_t span = (uint64_t)((int64_t)hi - (int64_t)lo + 1);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i)
        out[i] = (int32_t)((int64_t)lo + (int64_t)(word_at(key, (uint64_t)i) % span));
}

/* fp32 -> bf16 (RNE) for buffers the harness builds itself */
void synth_f32_to_bf16(uint64_t n, const float* in, uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i) out[i] = f32_to_bf16_bits(in[i]);
}
