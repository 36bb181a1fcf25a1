/*
 * oracle.c -- plain, slow, obviously-correct CPU reference of the hybrid
 * Mamba-2 / attention backbone frame step and its prefill.
 *
 * TEST INFRASTRUCTURE ONLY: loaded by tests/, the smoke check and the
 * benchmark's CPU-baseline leg; never by the CUDA library.  See oracle.h for
 * the sources each part follows.  Parity status of every function is recorded
 * in its comment ("pinned by ...").
 *
 * Storage points (OR_MIRROR rounds to bf16 exactly here; OR_EXACT rounds
 * nowhere):
 *   P1 pre-RMSNorm:   a = bf16(r * gamma); the matvec input is a * inv_rms
 *   P2 Mamba in_proj output [z | xBC | dt_raw]
 *   P3 conv history (holds the P2 xBC values)
 *   P4 gated RMSNorm: a = bf16(v * gamma_n); the out_proj input is a * inv_rms_group
 *   P5 attention q, k, v (so the KV cache holds bf16 values)
 *   P6 attention output o
 *   P7 MLP hidden relu(y)^2
 *   P8 final norm before the heads (as P1)
 * The residual stream r, the SSM state, scores, softmax and logits are never
 * rounded.  (The GPU path keeps those in fp32.)
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* threads the parallel loops below run on (OpenMP's default team size here) */
int or_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* rounding helpers                                                         */
/* ------------------------------------------------------------------------ */

/* round v to a binary float with `sig` significant bits, round-half-to-even,
 * whose smallest quantum is 2^qmin (gradual underflow).  Pinned by ties to
 * even, an fp16 subnormal tie and numpy's float16 conversion. */
static double round_sig(double v, int sig, int qmin) {
    if (v == 0.0 || !isfinite(v)) return v;
    int e;
    frexp(v, &e);               /* |v| = m * 2^e, m in [0.5, 1) */
    int qe = e - sig;           /* quantum exponent for this binade */
    if (qe < qmin) qe = qmin;
    return ldexp(nearbyint(ldexp(v, -qe)), qe);
}

double or_round_bf16(double v) { return round_sig(v, 8, -133); }
double or_round_fp16(double v) { return round_sig(v, 11, -24); }

static double bf16_val(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static double fp16_val(uint16_t h) {
    int s = h >> 15, e = (h >> 10) & 31, m = h & 1023;
    double v;
    if (e == 0) v = ldexp((double)m, -24);
    else if (e == 31) v = m ? NAN : INFINITY;
    else v = ldexp((double)(m | 1024), e - 25);
    return s ? -v : v;
}

static uint16_t fp16_bits(double v) { /* v already an exact fp16 value, finite */
    uint16_t s = v < 0 ? 0x8000 : 0;
    v = fabs(v);
    if (v == 0.0) return s;
    int e;
    double m = frexp(v, &e); /* v = m 2^e */
    if (e - 1 < -14) return s | (uint16_t)(v * 16777216.0); /* subnormal: v / 2^-24 */
    return s | (uint16_t)(((e - 1 + 15) << 10) | ((int)(m * 2048.0) - 1024));
}

static double silu(double x) { return x / (1.0 + exp(-x)); }
static double softplus(double x) { return x > 30.0 ? x + log1p(exp(-x)) : log1p(exp(x)); }

/* ------------------------------------------------------------------------ */
/* group quantization (weight-only, GPTQ-style storage; RTN decisions)       */
/* ------------------------------------------------------------------------ */

static int fmt_bits(int fmt) { return fmt == OR_W8 ? 8 : fmt == OR_W4 ? 4 : fmt == OR_W3 ? 3 : 16; }
static int words_per_row(int nelem, int bits) { return (int)(((long)nelem * bits + 31) / 32); }
static int n_groups(const or_mat* W) { return (W->K + W->group - 1) / W->group; }

static void put_bits(uint32_t* row, long idx, int bits, uint32_t code) {
    long o = idx * bits;
    int w = (int)(o >> 5), sh = (int)(o & 31);
    row[w] |= code << sh;
    if (sh + bits > 32) row[w + 1] |= code >> (32 - sh);
}

static uint32_t get_bits(const uint32_t* row, long idx, int bits) {
    long o = idx * bits;
    int w = (int)(o >> 5), sh = (int)(o & 31);
    uint64_t v = row[w] >> sh;
    if (sh + bits > 32) v |= (uint64_t)row[w + 1] << (32 - sh);
    return (uint32_t)(v & ((1u << bits) - 1u));
}

/* Round-to-nearest group quantizer.  Every decision is taken in IEEE fp32:
 *   W8 (symmetric):  s = fp16(amax / 127), q = clamp(rne(w / s), -127, 127)
 *   Wb (asymmetric, Q = 2^b - 1): s = fp16((max - min) / Q),
 *                    z = clamp(rne(-min / s), 0, Q), q = clamp(rne(w / s) + z, 0, Q)
 * with s := 1 when the fp16 scale would be 0 (constant or all-zero group).
 * Dequantization is w^ = s * (q - z) (z = 0 for W8).  GPTQ's calibration
 * (error feedback from activations, "Recipe" on the GPTQ 3-bit MLX page) is not
 * reproduced: with synthetic weights there is no calibration data.
 * Pinned by: constructed weights s (q - z) quantize back to (q, s, z) exactly,
 * a hand-worked example (tests/golden/quant_example.txt), and the RTN error
 * bound (half a step, one step at a clamped group extreme).                 */
void or_quantize(int fmt, int group, int N, int K, const float* w, uint32_t* q, uint16_t* scales,
                 uint32_t* zeros) {
    const int bits = fmt_bits(fmt);
    const int ng = (K + group - 1) / group;
    const int qw = words_per_row(K, bits), zw = words_per_row(ng, bits);
    const int Q = (1 << bits) - 1;
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) {
        const float* wr = w + (long)n * K;
        uint32_t* qr = q + (long)n * qw;
        memset(qr, 0, sizeof(uint32_t) * qw);
        if (fmt != OR_W8) memset(zeros + (long)n * zw, 0, sizeof(uint32_t) * zw);
        for (int g = 0; g < ng; ++g) {
            int k0 = g * group, k1 = k0 + group < K ? k0 + group : K;
            float sf;
            if (fmt == OR_W8) {
                float amax = 0.0f;
                for (int k = k0; k < k1; ++k) amax = fabsf(wr[k]) > amax ? fabsf(wr[k]) : amax;
                float s32 = amax / 127.0f;
                double s16 = or_round_fp16((double)s32);
                if (s16 == 0.0) s16 = 1.0;
                sf = (float)s16;
                scales[(long)n * ng + g] = fp16_bits(s16);
                for (int k = k0; k < k1; ++k) {
                    float t = wr[k] / sf;
                    int c = (int)nearbyintf(t);
                    c = c < -127 ? -127 : c > 127 ? 127 : c;
                    put_bits(qr, k, 8, (uint32_t)(uint8_t)(int8_t)c);
                }
            } else {
                float mx = wr[k0], mn = wr[k0];
                for (int k = k0; k < k1; ++k) {
                    mx = wr[k] > mx ? wr[k] : mx;
                    mn = wr[k] < mn ? wr[k] : mn;
                }
                float range = mx - mn;
                float s32 = range / (float)Q;
                double s16 = or_round_fp16((double)s32);
                if (s16 == 0.0) s16 = 1.0;
                sf = (float)s16;
                scales[(long)n * ng + g] = fp16_bits(s16);
                int z = (int)nearbyintf(-mn / sf);
                z = z < 0 ? 0 : z > Q ? Q : z;
                put_bits(zeros + (long)n * zw, g, bits, (uint32_t)z);
                for (int k = k0; k < k1; ++k) {
                    int c = (int)nearbyintf(wr[k] / sf) + z;
                    c = c < 0 ? 0 : c > Q ? Q : c;
                    put_bits(qr, k, bits, (uint32_t)c);
                }
            }
        }
    }
}

/* integer codes, zero points and scales of row n (pinned by the pack/unpack
 * round-trip and by the exact dequantization tests) */
static void codes_row(const or_mat* W, int n, int32_t* codes, int32_t* zeros, double* scales) {
    const int bits = fmt_bits(W->fmt), ng = n_groups(W);
    const uint32_t* qr = (const uint32_t*)W->q + (long)n * words_per_row(W->K, bits);
    for (int k = 0; k < W->K; ++k) {
        uint32_t c = get_bits(qr, k, bits);
        codes[k] = W->fmt == OR_W8 ? (int32_t)(int8_t)(uint8_t)c : (int32_t)c;
    }
    for (int g = 0; g < ng; ++g) {
        scales[g] = fp16_val(W->scales[(long)n * ng + g]);
        zeros[g] = W->fmt == OR_W8 ? 0
                                   : (int32_t)get_bits(W->zeros + (long)n * words_per_row(ng, bits), g, bits);
    }
}

void or_codes(const or_mat* W, int32_t* codes, int32_t* zeros, double* scales) {
    const int ng = n_groups(W);
#pragma omp parallel for schedule(static)
    for (int n = 0; n < W->N; ++n)
        codes_row(W, n, codes + (long)n * W->K, zeros + (long)n * ng, scales + (long)n * ng);
}

/* row n of the dequantized weight, w^ = s * (q - z), exact in double (pinned
 * against the independently decoded codes times scales) */
static void deq_row(const or_mat* W, int n, double* row, int32_t* tmp_codes, int32_t* tmp_z, double* tmp_s) {
    if (W->fmt == OR_BF16) {
        const uint16_t* r = (const uint16_t*)W->q + (long)n * W->K;
        for (int k = 0; k < W->K; ++k) row[k] = bf16_val(r[k]);
        return;
    }
    codes_row(W, n, tmp_codes, tmp_z, tmp_s);
    for (int k = 0; k < W->K; ++k) {
        int g = k / W->group;
        row[k] = tmp_s[g] * (double)(tmp_codes[k] - tmp_z[g]);
    }
}

void or_dequant(const or_mat* W, double* out) {
    const int ng = W->fmt == OR_BF16 ? 1 : n_groups(W);
#pragma omp parallel
    {
        int32_t* c = malloc(sizeof(int32_t) * W->K);
        int32_t* z = malloc(sizeof(int32_t) * ng);
        double* s = malloc(sizeof(double) * ng);
#pragma omp for schedule(static)
        for (int n = 0; n < W->N; ++n) deq_row(W, n, out + (long)n * W->K, c, z, s);
        free(c); free(z); free(s);
    }
}

/* Y[b][n] = sum_k W^[n][k] U[b][k] for b < B (rows of U are inputs).  Pinned
 * by equality with a dense product on the dequantized matrix. */
static void matmul_rows(const or_mat* W, int B, const double* U, double* Y) {
    const int ng = W->fmt == OR_BF16 ? 1 : n_groups(W);
#pragma omp parallel
    {
        double* row = malloc(sizeof(double) * W->K);
        int32_t* c = malloc(sizeof(int32_t) * W->K);
        int32_t* z = malloc(sizeof(int32_t) * ng);
        double* s = malloc(sizeof(double) * ng);
#pragma omp for schedule(dynamic, 16)
        for (int n = 0; n < W->N; ++n) {
            deq_row(W, n, row, c, z, s);
            for (int b = 0; b < B; ++b) {
                const double* u = U + (long)b * W->K;
                double acc = 0.0;
                for (int k = 0; k < W->K; ++k) acc += row[k] * u[k];
                Y[(long)b * W->N + n] = acc;
            }
        }
        free(row); free(c); free(z); free(s);
    }
}

void or_matvec(const or_mat* W, const double* u, double* y) { matmul_rows(W, 1, u, y); }

/* ------------------------------------------------------------------------ */
/* model pieces                                                             */
/* ------------------------------------------------------------------------ */

typedef struct {
    int d, L, H, P, N, G, W, E, Cx, NG, Hq, Hk, Dh, F, Vt, Vf, nm, na;
    double eps;
} dims;

static dims get_dims(const or_config* c) {
    dims m;
    m.d = c->d_model;
    m.L = (int)strlen(c->pattern);
    m.H = c->ssm_heads; m.P = c->ssm_head_dim; m.N = c->ssm_state; m.G = c->ssm_groups;
    m.W = c->conv_width; m.E = m.H * m.P; m.Cx = m.E + 2 * m.G * m.N; m.NG = c->norm_groups;
    m.Hq = c->attn_q_heads; m.Hk = c->attn_kv_heads; m.Dh = c->attn_head_dim;
    m.F = c->mlp_hidden; m.Vt = c->vocab_text; m.Vf = c->vocab_func;
    m.nm = m.na = 0;
    for (int l = 0; l < m.L; ++l) {
        if (c->pattern[l] == 'M') m.nm++;
        if (c->pattern[l] == '*') m.na++;
    }
    m.eps = c->eps;
    return m;
}

/* pre-RMSNorm (P1/P8): u = r * gamma / sqrt(mean(r^2) + eps) for one row.
 * Pinned by: RMSNorm of a constant vector (closed form), and end to end by the
 * brute-force full-sequence check. */
static void prenorm_row(const double* r, const float* gamma, int d, double eps, int mode, double* u) {
    double ss = 0.0;
    for (int k = 0; k < d; ++k) ss += r[k] * r[k];
    double inv = 1.0 / sqrt(ss / d + eps);
    for (int k = 0; k < d; ++k) {
        double a = r[k] * (double)gamma[k];
        u[k] = (mode == OR_MIRROR ? or_round_bf16(a) : a) * inv;
    }
}

static double rnd(int mode, double v) { return mode == OR_MIRROR ? or_round_bf16(v) : v; }

/* Causal depthwise conv1d + SiLU of one frame over the history ring.
 * xc[c] = silu(b[c] + sum_{k<W-1} w[c][k] * hist[k][c] + w[c][W-1] * xBC[c]);
 * the history then drops its oldest row and appends xBC.  Pinned by the
 * brute-force full causal convolution over the zero-padded sequence, and by the
 * memoryless-limit and hand-worked scalar cases. */
static void conv_step(const dims* m, const or_layer* L, double* hist, const double* xBC, double* xc) {
    for (int c = 0; c < m->Cx; ++c) {
        double acc = (double)L->conv_b[c];
        for (int k = 0; k < m->W - 1; ++k) acc += (double)L->conv_w[c * m->W + k] * hist[(long)k * m->Cx + c];
        acc += (double)L->conv_w[c * m->W + m->W - 1] * xBC[c];
        xc[c] = silu(acc);
    }
    for (int k = 0; k + 1 < m->W - 1; ++k)
        memcpy(hist + (long)k * m->Cx, hist + (long)(k + 1) * m->Cx, sizeof(double) * m->Cx);
    if (m->W > 1) memcpy(hist + (long)(m->W - 2) * m->Cx, xBC, sizeof(double) * m->Cx);
}

/* One SSM recurrence step for all heads:
 *   dt = softplus(dt_raw + dt_bias); a = exp(A dt), A = -exp(A_log)
 *   S[h][p][n] <- a S + dt x[h,p] B[g(h),n];  y[h,p] = sum_n C[g(h),n] S + D[h] x[h,p]
 * with g(h) = floor(h G / H).  Pinned by the brute-force O(T^2) closed form. */
static void ssm_step(const dims* m, const or_layer* L, double* S, const double* xc, const double* dt_raw,
                     double* y) {
    const double* x = xc;
    const double* Bv = xc + m->E;
    const double* Cv = xc + m->E + m->G * m->N;
#pragma omp parallel for schedule(static)
    for (int h = 0; h < m->H; ++h) {
        int g = (int)((long)h * m->G / m->H);
        double dt = softplus(dt_raw[h] + (double)L->dt_bias[h]);
        double A = -exp((double)L->A_log[h]);
        double a = exp(A * dt);
        for (int p = 0; p < m->P; ++p) {
            double xv = x[h * m->P + p];
            double* Sr = S + ((long)h * m->P + p) * m->N;
            double acc = 0.0;
            for (int n = 0; n < m->N; ++n) {
                Sr[n] = a * Sr[n] + dt * xv * Bv[g * m->N + n];
                acc += Cv[g * m->N + n] * Sr[n];
            }
            y[h * m->P + p] = acc + (double)L->D[h] * xv;
        }
    }
}

/* Chunked SSD over T frames (Dao & Gu, "Transformers are SSMs", the SSD
 * algorithm): within a chunk of Q frames, with the inclusive cumulative
 * log-decay Lam_i = sum_{r<=i} A dt_r,
 *   Y_diag[i] = sum_{j<=i} (C_i . B_j) exp(Lam_i - Lam_j) dt_j x_j
 *   Y_off[i]  = exp(Lam_i) C_i . S_prev
 *   S_next    = exp(Lam_end) S_prev + sum_j exp(Lam_end - Lam_j) dt_j x_j (outer) B_j
 *   y_i = Y_diag + Y_off + D x_i
 * Pinned by: equality with the sequential recurrence (any Q, ragged T). */
static void ssd_chunked(const dims* m, const or_layer* L, int T, int Q, double* S, const double* xc_all,
                        const double* dtr_all, long xc_stride, long dt_stride, double* y_all) {
#pragma omp parallel
    {
        double* Lam = malloc(sizeof(double) * Q);
        double* dts = malloc(sizeof(double) * Q);
        double* Snew = malloc(sizeof(double) * m->P * m->N);
        double* wrow = malloc(sizeof(double) * Q);
#pragma omp for schedule(static)
        for (int h = 0; h < m->H; ++h) {
            int g = (int)((long)h * m->G / m->H);
            double A = -exp((double)L->A_log[h]);
            double* Sh = S + (long)h * m->P * m->N;
            for (int c0 = 0; c0 < T; c0 += Q) {
                int len = T - c0 < Q ? T - c0 : Q;
                double run = 0.0;
                for (int i = 0; i < len; ++i) {
                    dts[i] = softplus(dtr_all[(long)(c0 + i) * dt_stride + h] + (double)L->dt_bias[h]);
                    run += A * dts[i];
                    Lam[i] = run;
                }
                for (int i = 0; i < len; ++i) {
                    const double* xi = xc_all + (long)(c0 + i) * xc_stride;
                    const double* Ci = xi + m->E + m->G * m->N + g * m->N;
                    /* weights of the diagonal block row i: (C_i . B_j) exp(Lam_i - Lam_j) dt_j */
                    for (int j = 0; j <= i; ++j) {
                        const double* Bj = xc_all + (long)(c0 + j) * xc_stride + m->E + g * m->N;
                        double cb = 0.0;
                        for (int n = 0; n < m->N; ++n) cb += Ci[n] * Bj[n];
                        wrow[j] = cb * exp(Lam[i] - Lam[j]) * dts[j];
                    }
                    for (int p = 0; p < m->P; ++p) {
                        double yd = 0.0;
                        for (int j = 0; j <= i; ++j) yd += wrow[j] * xc_all[(long)(c0 + j) * xc_stride + h * m->P + p];
                        double yo = 0.0;
                        for (int n = 0; n < m->N; ++n) yo += Ci[n] * Sh[(long)p * m->N + n];
                        yo *= exp(Lam[i]);
                        y_all[(long)(c0 + i) * m->E + h * m->P + p] = yd + yo + (double)L->D[h] * xi[h * m->P + p];
                    }
                }
                double lend = Lam[len - 1];
                for (int p = 0; p < m->P; ++p)
                    for (int n = 0; n < m->N; ++n) {
                        double acc = exp(lend) * Sh[(long)p * m->N + n];
                        for (int j = 0; j < len; ++j) {
                            const double* xj = xc_all + (long)(c0 + j) * xc_stride;
                            acc += exp(lend - Lam[j]) * dts[j] * xj[h * m->P + p] * xj[m->E + g * m->N + n];
                        }
                        Snew[(long)p * m->N + n] = acc;
                    }
                memcpy(Sh, Snew, sizeof(double) * m->P * m->N);
            }
        }
        free(Lam); free(dts); free(Snew); free(wrow);
    }
}

void or_mamba_mixer(const or_config* cfg, const or_layer* L, int T, const double* zxbcdt, double* ssm,
                    double* conv, int ssd_chunk, double* y_out, double* v_out) {
    dims m = get_dims(cfg);
    const long R = m.E + m.Cx + m.H;
    double* xc_all = malloc(sizeof(double) * (long)T * m.Cx);
    for (int t = 0; t < T; ++t) conv_step(&m, L, conv, zxbcdt + t * R + m.E, xc_all + (long)t * m.Cx);
    if (ssd_chunk <= 0) {
        for (int t = 0; t < T; ++t)
            ssm_step(&m, L, ssm, xc_all + (long)t * m.Cx, zxbcdt + t * R + m.E + m.Cx, y_out + (long)t * m.E);
    } else {
        ssd_chunked(&m, L, T, ssd_chunk, ssm, xc_all, zxbcdt + m.E + m.Cx, m.Cx, R, y_out);
    }
    for (int t = 0; t < T; ++t)
        for (int c = 0; c < m.E; ++c) v_out[(long)t * m.E + c] = y_out[(long)t * m.E + c] * silu(zxbcdt[t * R + c]);
    free(xc_all);
}

/* gated RMSNorm (P4): groups of E/NG channels; returns the out_proj input.
 * Pinned end to end by the brute-force full-sequence check (one and two
 * groups). */
static void gated_norm_row(const dims* m, const or_layer* L, const double* v, int mode, double* u) {
    int gs = m->E / m->NG;
    for (int q = 0; q < m->NG; ++q) {
        double ss = 0.0;
        for (int c = q * gs; c < (q + 1) * gs; ++c) ss += v[c] * v[c];
        double inv = 1.0 / sqrt(ss / gs + m->eps);
        for (int c = q * gs; c < (q + 1) * gs; ++c) u[c] = rnd(mode, v[c] * (double)L->gnorm[c]) * inv;
    }
}

/* causal softmax attention of one query row set against cached keys 0..t
 * (GQA: query head i reads KV head floor(i Hk / Hq); scale 1/sqrt(Dh); no
 * positional encoding).  Pinned by equality with full masked-softmax
 * attention over the sequence (brute force). */
static void attend(const dims* m, const double* q, const double* Kc, const double* Vc, int cap, int t,
                   int mode, double* o) {
    double* s = malloc(sizeof(double) * (t + 1));
    for (int i = 0; i < m->Hq; ++i) {
        int j = (int)((long)i * m->Hk / m->Hq);
        const double* qi = q + (long)i * m->Dh;
        const double* Kj = Kc + (long)j * cap * m->Dh;
        const double* Vj = Vc + (long)j * cap * m->Dh;
        double mx = -INFINITY;
        for (int tau = 0; tau <= t; ++tau) {
            double acc = 0.0;
            for (int e = 0; e < m->Dh; ++e) acc += qi[e] * Kj[(long)tau * m->Dh + e];
            s[tau] = acc / sqrt((double)m->Dh);
            mx = s[tau] > mx ? s[tau] : mx;
        }
        double den = 0.0;
        for (int tau = 0; tau <= t; ++tau) { s[tau] = exp(s[tau] - mx); den += s[tau]; }
        for (int e = 0; e < m->Dh; ++e) {
            double acc = 0.0;
            for (int tau = 0; tau <= t; ++tau) acc += s[tau] * Vj[(long)tau * m->Dh + e];
            o[(long)i * m->Dh + e] = rnd(mode, acc / den);
        }
    }
    free(s);
}

static long ssm_slot_size(const dims* m) { return (long)m->H * m->P * m->N; }
static long conv_slot_size(const dims* m) { return (long)(m->W - 1) * m->Cx; }
static long kv_slot_size(const dims* m, int cap) { return (long)m->Hk * cap * m->Dh; }

/* ------------------------------------------------------------------------ */
/* decode step                                                              */
/* ------------------------------------------------------------------------ */

/* One layer of the decode step for nl live rows (residual r [nl][d] updated in place; U, Y, Y2
 * and xc are scratch).  sl[i] is row i's state slot; mi / ai index the layer among the Mamba-2 /
 * attention layers.  Storage points of mirror mode: P1 (u), P2 (in_proj output), P4 (gated-norm
 * output), P5 (q, k, v), P6 (attention output), P7 (MLP hidden). */
static void layer_forward(const dims* mp, const or_layer* L, char kind, int mi, int ai, or_state* st, int nl,
                          const int* sl, int mode, double* r, double* U, double* Y, double* Y2, double* xc) {
    const dims m = *mp;
    const int d = m.d, cap = st->kv_capacity;
    for (int i = 0; i < nl; ++i) prenorm_row(r + (long)i * d, L->norm, d, m.eps, mode, U + (long)i * d);
    if (kind == 'M') {
        const long R = m.E + m.Cx + m.H;
        matmul_rows(&L->in_proj, nl, U, Y);
        for (int i = 0; i < nl; ++i) {
            double* zx = Y + (long)i * R;
            for (long c = 0; c < R; ++c) zx[c] = rnd(mode, zx[c]); /* P2 */
            int s = sl[i];
            double* S = st->ssm + ((long)mi * st->n_slots + s) * ssm_slot_size(&m);
            double* hist = st->conv + ((long)mi * st->n_slots + s) * conv_slot_size(&m);
            conv_step(&m, L, hist, zx + m.E, xc);
            double* yv = Y2 + (long)i * m.E;
            ssm_step(&m, L, S, xc, zx + m.E + m.Cx, yv);
            for (int c = 0; c < m.E; ++c) yv[c] *= silu(zx[c]);
            gated_norm_row(&m, L, yv, mode, U + (long)i * m.E);
        }
        matmul_rows(&L->out_proj, nl, U, Y);
        for (long k = 0; k < (long)nl * d; ++k) r[k] += Y[k];
    } else if (kind == '*') {
        const long R = (long)(m.Hq + 2 * m.Hk) * m.Dh;
        matmul_rows(&L->qkv, nl, U, Y);
        for (int i = 0; i < nl; ++i) {
            double* qkv = Y + (long)i * R;
            for (long c = 0; c < R; ++c) qkv[c] = rnd(mode, qkv[c]); /* P5 */
            int s = sl[i];
            int t = st->ctx_len[s];
            double* Kc = st->k + ((long)ai * st->n_slots + s) * kv_slot_size(&m, cap);
            double* Vc = st->v + ((long)ai * st->n_slots + s) * kv_slot_size(&m, cap);
            for (int j = 0; j < m.Hk; ++j)
                for (int e = 0; e < m.Dh; ++e) {
                    Kc[((long)j * cap + t) * m.Dh + e] = qkv[(long)m.Hq * m.Dh + (long)j * m.Dh + e];
                    Vc[((long)j * cap + t) * m.Dh + e] = qkv[(long)(m.Hq + m.Hk) * m.Dh + (long)j * m.Dh + e];
                }
            attend(&m, qkv, Kc, Vc, cap, t, mode, U + (long)i * m.Hq * m.Dh); /* P6 */
        }
        matmul_rows(&L->o, nl, U, Y);
        for (long k = 0; k < (long)nl * d; ++k) r[k] += Y[k];
    } else {
        matmul_rows(&L->up, nl, U, Y);
        for (long k = 0; k < (long)nl * m.F; ++k) {
            double h = Y[k] > 0.0 ? Y[k] : 0.0;
            U[k] = rnd(mode, h * h); /* P7 */
        }
        matmul_rows(&L->down, nl, U, Y);
        for (long k = 0; k < (long)nl * d; ++k) r[k] += Y[k];
    }
}

/* final norm (P8), the text and function heads, greedy argmax (lowest index on ties) for nl live
 * rows; out_row[i] is the output row of live row i.  U is scratch [nl][d]. */
static void heads_forward(const dims* mp, const or_weights* w, int nl, const int* out_row, int B, int mode,
                          const double* r, double* U, int32_t* tok_text, int32_t* tok_func, double* logits) {
    const dims m = *mp;
    const int d = m.d;
    for (int i = 0; i < nl; ++i) prenorm_row(r + (long)i * d, w->final_norm, d, m.eps, mode, U + (long)i * d);
    for (int hsel = 0; hsel < 2; ++hsel) {
        const or_mat* Wh = hsel == 0 ? &w->head_text : &w->head_func;
        int V = Wh->N;
        double* lg = malloc(sizeof(double) * (long)nl * V);
        matmul_rows(Wh, nl, U, lg);
        for (int i = 0; i < nl; ++i) {
            const double* li = lg + (long)i * V;
            int best = 0;
            for (int v = 1; v < V; ++v)
                if (li[v] > li[best]) best = v;
            (hsel == 0 ? tok_text : tok_func)[out_row[i]] = best;
            if (logits) {
                int Vmax = m.Vt > m.Vf ? m.Vt : m.Vf;
                memcpy(logits + ((long)hsel * B + out_row[i]) * Vmax, li, sizeof(double) * V);
            }
        }
        free(lg);
    }
}

static long scratch_width(const dims* m) {
    long maxw = m->E + m->Cx + m->H;
    if ((long)(m->Hq + 2 * m->Hk) * m->Dh > maxw) maxw = (long)(m->Hq + 2 * m->Hk) * m->Dh;
    if (m->F > maxw) maxw = m->F;
    if (m->E > maxw) maxw = m->E;
    if (m->d > maxw) maxw = m->d;
    return maxw;
}

int or_step(const or_config* cfg, const or_weights* w, or_state* st, int B, const uint16_t* x,
            const int32_t* slots, int mode, int32_t* tok_text, int32_t* tok_func, double* hidden,
            double* logits) {
    dims m = get_dims(cfg);
    const int d = m.d, cap = st->kv_capacity;
    int ret = 0;
    int* live = malloc(sizeof(int) * B);
    int* slot = malloc(sizeof(int) * B);
    int* sl = malloc(sizeof(int) * B);
    int nl = 0;
    for (int b = 0; b < B; ++b) {
        slot[b] = slots ? slots[b] : b;
        if (st->ctx_len[slot[b]] >= cap) {  /* cache full: the session is skipped */
            ret = 1;
            tok_text[b] = tok_func[b] = -1;
        } else {
            sl[nl] = slot[b];
            live[nl++] = b;
        }
    }
    const long maxw = scratch_width(&m);
    double* r = calloc((long)nl * d, sizeof(double));
    double* U = malloc(sizeof(double) * nl * maxw);
    double* Y = malloc(sizeof(double) * nl * maxw);
    double* Y2 = malloc(sizeof(double) * nl * maxw);
    double* xc = malloc(sizeof(double) * m.Cx);

    for (int i = 0; i < nl; ++i)
        for (int k = 0; k < d; ++k) r[(long)i * d + k] = bf16_val(x[(long)live[i] * d + k]);
    if (hidden)
        for (int i = 0; i < nl; ++i) memcpy(hidden + (long)live[i] * d, r + (long)i * d, sizeof(double) * d);

    int mi = 0, ai = 0;
    for (int l = 0; l < m.L; ++l) {
        char kind = cfg->pattern[l];
        layer_forward(&m, &w->layers[l], kind, mi, ai, st, nl, sl, mode, r, U, Y, Y2, xc);
        if (kind == 'M') mi++;
        if (kind == '*') ai++;
        if (hidden)
            for (int i = 0; i < nl; ++i)
                memcpy(hidden + ((long)(l + 1) * B + live[i]) * d, r + (long)i * d, sizeof(double) * d);
    }
    heads_forward(&m, w, nl, live, B, mode, r, U, tok_text, tok_func, logits);
    for (int i = 0; i < nl; ++i) st->ctx_len[slot[live[i]]] += 1;
    free(r); free(U); free(Y); free(Y2); free(xc); free(live); free(slot); free(sl);
    return ret;
}

int or_layer_step(const or_config* cfg, const or_weights* w, or_state* st, int layer, int B,
                  const double* r_in, const int32_t* slots, int mode, double* r_out) {
    dims m = get_dims(cfg);
    if (layer < 0 || layer >= m.L || B < 1) return 2;
    const int d = m.d;
    int mi = 0, ai = 0;
    for (int l = 0; l < layer; ++l) {
        if (cfg->pattern[l] == 'M') mi++;
        if (cfg->pattern[l] == '*') ai++;
    }
    int* sl = malloc(sizeof(int) * B);
    for (int b = 0; b < B; ++b) sl[b] = slots ? slots[b] : b;
    for (int b = 0; b < B; ++b)
        if (cfg->pattern[layer] == '*' && st->ctx_len[sl[b]] >= st->kv_capacity) {
            free(sl);
            return 1;
        }
    const long maxw = scratch_width(&m);
    double* U = malloc(sizeof(double) * B * maxw);
    double* Y = malloc(sizeof(double) * B * maxw);
    double* Y2 = malloc(sizeof(double) * B * maxw);
    double* xc = malloc(sizeof(double) * m.Cx);
    memcpy(r_out, r_in, sizeof(double) * (long)B * d);
    layer_forward(&m, &w->layers[layer], cfg->pattern[layer], mi, ai, st, B, sl, mode, r_out, U, Y, Y2, xc);
    free(U); free(Y); free(Y2); free(xc); free(sl);
    return 0;
}

void or_heads(const or_config* cfg, const or_weights* w, int B, const double* r, int mode, int32_t* tok_text,
              int32_t* tok_func, double* logits) {
    dims m = get_dims(cfg);
    int* rows = malloc(sizeof(int) * B);
    for (int b = 0; b < B; ++b) rows[b] = b;
    double* U = malloc(sizeof(double) * (long)B * m.d);
    heads_forward(&m, w, B, rows, B, mode, r, U, tok_text, tok_func, logits);
    free(U); free(rows);
}

/* ------------------------------------------------------------------------ */
/* prefill (layer by layer over all T frames)                                */
/* ------------------------------------------------------------------------ */

/* One layer of the prefill over T frames of one slot whose first frame is frame t0 (residual r
 * [T][d] updated in place; U, Y, Y2, V2 are scratch).  Same storage points as the step. */
static void prefill_layer_forward(const dims* mp, const or_config* cfg, const or_layer* L, char kind, int mi,
                                  int ai, or_state* st, int slot, int t0, int T, int mode, int ssd_chunk,
                                  double* r, double* U, double* Y, double* Y2, double* V2) {
    const dims m = *mp;
    const int d = m.d, cap = st->kv_capacity;
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) prenorm_row(r + (long)t * d, L->norm, d, m.eps, mode, U + (long)t * d);
    if (kind == 'M') {
        const long R = m.E + m.Cx + m.H;
        matmul_rows(&L->in_proj, T, U, Y);
        for (long k = 0; k < (long)T * R; ++k) Y[k] = rnd(mode, Y[k]); /* P2 */
        double* S = st->ssm + ((long)mi * st->n_slots + slot) * ssm_slot_size(&m);
        double* hist = st->conv + ((long)mi * st->n_slots + slot) * conv_slot_size(&m);
        or_mamba_mixer(cfg, L, T, Y, S, hist, ssd_chunk, Y2, V2);
#pragma omp parallel for schedule(static)
        for (int t = 0; t < T; ++t) gated_norm_row(&m, L, V2 + (long)t * m.E, mode, U + (long)t * m.E);
        matmul_rows(&L->out_proj, T, U, Y);
        for (long k = 0; k < (long)T * d; ++k) r[k] += Y[k];
    } else if (kind == '*') {
        const long R = (long)(m.Hq + 2 * m.Hk) * m.Dh;
        matmul_rows(&L->qkv, T, U, Y);
        for (long k = 0; k < (long)T * R; ++k) Y[k] = rnd(mode, Y[k]); /* P5 */
        double* Kc = st->k + ((long)ai * st->n_slots + slot) * kv_slot_size(&m, cap);
        double* Vc = st->v + ((long)ai * st->n_slots + slot) * kv_slot_size(&m, cap);
        for (int t = 0; t < T; ++t)
            for (int j = 0; j < m.Hk; ++j)
                for (int e = 0; e < m.Dh; ++e) {
                    Kc[((long)j * cap + t0 + t) * m.Dh + e] = Y[(long)t * R + (long)m.Hq * m.Dh + (long)j * m.Dh + e];
                    Vc[((long)j * cap + t0 + t) * m.Dh + e] =
                        Y[(long)t * R + (long)(m.Hq + m.Hk) * m.Dh + (long)j * m.Dh + e];
                }
#pragma omp parallel for schedule(dynamic, 4)
        for (int t = 0; t < T; ++t)
            attend(&m, Y + (long)t * R, Kc, Vc, cap, t0 + t, mode, U + (long)t * m.Hq * m.Dh); /* P6 */
        matmul_rows(&L->o, T, U, Y);
        for (long k = 0; k < (long)T * d; ++k) r[k] += Y[k];
    } else {
        matmul_rows(&L->up, T, U, Y);
        for (long k = 0; k < (long)T * m.F; ++k) {
            double h = Y[k] > 0.0 ? Y[k] : 0.0;
            U[k] = rnd(mode, h * h); /* P7 */
        }
        matmul_rows(&L->down, T, U, Y);
        for (long k = 0; k < (long)T * d; ++k) r[k] += Y[k];
    }
}

int or_prefill(const or_config* cfg, const or_weights* w, or_state* st, int slot, int T,
               const uint16_t* x, int mode, int ssd_chunk, double* hidden) {
    dims m = get_dims(cfg);
    const int d = m.d, cap = st->kv_capacity;
    const int t0 = st->ctx_len[slot];
    if (t0 + T > cap) return 1;
    const long maxw = scratch_width(&m);
    double* r = malloc(sizeof(double) * (long)T * d);
    double* U = malloc(sizeof(double) * (long)T * maxw);
    double* Y = malloc(sizeof(double) * (long)T * maxw);
    double* Y2 = malloc(sizeof(double) * (long)T * m.E);
    double* V2 = malloc(sizeof(double) * (long)T * m.E);
    for (long k = 0; k < (long)T * d; ++k) r[k] = bf16_val(x[k]);
    if (hidden) memcpy(hidden, r, sizeof(double) * (long)T * d);
    int mi = 0, ai = 0;
    for (int l = 0; l < m.L; ++l) {
        char kind = cfg->pattern[l];
        prefill_layer_forward(&m, cfg, &w->layers[l], kind, mi, ai, st, slot, t0, T, mode, ssd_chunk, r, U, Y, Y2,
                              V2);
        if (kind == 'M') mi++;
        if (kind == '*') ai++;
        if (hidden) memcpy(hidden + (long)(l + 1) * T * d, r, sizeof(double) * (long)T * d);
    }
    st->ctx_len[slot] = t0 + T;
    free(r); free(U); free(Y); free(Y2); free(V2);
    return 0;
}

int or_prefill_layer(const or_config* cfg, const or_weights* w, or_state* st, int slot, int layer, int T,
                     const double* r_in, int mode, int ssd_chunk, double* r_out) {
    dims m = get_dims(cfg);
    if (layer < 0 || layer >= m.L || T < 1) return 2;
    const int t0 = st->ctx_len[slot];
    if (t0 + T > st->kv_capacity) return 1;
    int mi = 0, ai = 0;
    for (int l = 0; l < layer; ++l) {
        if (cfg->pattern[l] == 'M') mi++;
        if (cfg->pattern[l] == '*') ai++;
    }
    const long maxw = scratch_width(&m);
    double* U = malloc(sizeof(double) * (long)T * maxw);
    double* Y = malloc(sizeof(double) * (long)T * maxw);
    double* Y2 = malloc(sizeof(double) * (long)T * m.E);
    double* V2 = malloc(sizeof(double) * (long)T * m.E);
    memcpy(r_out, r_in, sizeof(double) * (long)T * m.d);
    prefill_layer_forward(&m, cfg, &w->layers[layer], cfg->pattern[layer], mi, ai, st, slot, t0, T, mode, ssd_chunk,
                          r_out, U, Y, Y2, V2);
    free(U); free(Y); free(Y2); free(V2);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* fused per-frame input (the previous frame's tokens fed back)             */
/* ------------------------------------------------------------------------ */

static uint16_t bf16_bits_of(double v) {
    /* v is already a bf16 value: its float image has 16 zero low bits */
    float f = (float)v;
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

void or_fuse_inputs(int B, int d, const uint16_t* speech, const uint16_t* emb_text, int Vt,
                    const uint16_t* emb_func, int Vf, const int32_t* tok_text, const int32_t* tok_func,
                    uint16_t* out) {
    for (int b = 0; b < B; ++b) {
        const int tt = tok_text[b], tf = tok_func[b];
        for (int k = 0; k < d; ++k) {
            double v = bf16_val(speech[(long)b * d + k]);
            if (tt >= 0 && tt < Vt) v += bf16_val(emb_text[(long)tt * d + k]);
            if (tf >= 0 && tf < Vf) v += bf16_val(emb_func[(long)tf * d + k]);
            out[(long)b * d + k] = bf16_bits_of(or_round_bf16(v));
        }
    }
}
