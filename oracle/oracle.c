/*
 * fp64 CPU oracle of the routed, block-quantised MoE FFN layer.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this code; the library's compute path never does.
 * It shares no code, header or table with the CUDA path.
 *
 * What it computes, per token t (the MoE layer that the "Qwen3.8-Flash-Next
 * UD-IQ2_XS (L4 fix) for Basalt" model card, section "What was changed",
 * describes as a device-planned tail of grouped kernels over routed experts in
 * IQ4_NL, NVFP4, Q5_1 or Q8_0; the model card "Qwen3.8-Flash-Next-Basalt" and
 * the "llms-full.txt" FAQ describe the model as a mixture of experts in which
 * each token uses only its selected experts):
 *
 *   1. router logits   l_e = sum_h Wr[e,h] x[h]                   (fp64, exact)
 *   2. top-k           S = the k largest l_e, ties to the lower e
 *   3. gates           g_e = exp(l_e - m) / sum_{j in S} exp(l_j - m), m = max l
 *                      (softmax over all experts renormalised over S; the
 *                      full denominator cancels)
 *   4. each e in S, plus the always-on shared expert when present:
 *                      a = G_e x, b = U_e x, h = a/(1+exp(-a)) * b, y_e = D_e h
 *   5. combine         out = sum_{e in S} g_e y_e + y_shared
 *
 * G, U, D are the dequantised expert weights, held exactly in fp64.  The block
 * decoders below are written from the format definitions:
 *   Q8_0   32 weights: fp16 d, 32 int8 q              w = d*q
 *   Q5_1   32 weights: fp16 d, fp16 m, 32 5-bit q     w = d*q + m
 *   Q5_0   32 weights: fp16 d, 32 5-bit q             w = d*(q - 16)  (5.5 bits
 *                      per weight, the size the model card gives; the centred
 *                      code is the plainest reading of a five-bit format with a
 *                      single scale)
 *   IQ4_NL 32 weights: fp16 d, 32 4-bit indices i     w = d*T[i], T a 16-entry
 *                                                     int8 table (an input)
 *   NVFP4  16 weights: E4M3 scale b, 16 E2M1 codes n, and one fp32 scale s per
 *                      matrix                          w = s*e4m3(b)*e2m1(n)
 * (IQ4_NL at 4.5 bits per weight and Q5_0 at 5.5 are the sizes the model card
 * states when it requantises one tensor; E4M3 and E2M1 follow the OCP
 * Microscaling Formats (MX) v1.0 / OCP 8-bit Floating Point specifications.)
 * Byte layout of each block (little endian):
 *   Q8_0   34 B: [0,2) d, [2,34) q[32]
 *   Q5_1   24 B: [0,2) d, [2,4) m, [4,8) qh (bit j = bit 4 of element j),
 *               [8,24) qs: element j<16 low nibble of qs[j], j>=16 high nibble of qs[j-16]
 *   Q5_0   22 B: [0,2) d, [2,6) qh, [6,22) qs, bits and nibbles as Q5_1
 *   IQ4_NL 18 B: [0,2) d, [2,18) qs, nibble order as Q5_1
 *   NVFP4   9 B: [0] E4M3 scale, [1,9) element 2i low / 2i+1 high nibble of byte i
 *
 * Activation quantisation (act_quant = 1) is the NVFP4 tensor-core prefill's
 * reading: x before gate/up and h before down are each rounded to NVFP4 with a
 * per-token fp32 scale s = amax/(6*448), block scales e4m3_rne_satfinite(
 * amax16/(6*s)) and codes e2m1_rne_satfinite(v/(s*scale)), every step in fp32
 * as the tensor-core path computes it; the matvecs then run in fp64 on the
 * rounded values.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#include "oracle.h"

/* ---- scalar decoders --------------------------------------------------- */

/* IEEE binary16 -> double, from the bit fields */
double oracle_fp16(uint16_t u)
{
    int s = (u >> 15) & 1, e = (u >> 10) & 31, m = u & 1023;
    double v;
    if (e == 0) v = ldexp((double)m, -24);                  /* subnormal: m * 2^-24 */
    else if (e == 31) v = m ? NAN : INFINITY;
    else v = ldexp(1.0 + m / 1024.0, e - 15);
    return s ? -v : v;
}

/* bfloat16 -> double: the upper half of an IEEE binary32 */
double oracle_bf16(uint16_t u)
{
    int s = (u >> 15) & 1, e = (u >> 7) & 255, m = u & 127;
    double v;
    if (e == 0) v = ldexp((double)m, -133);                 /* m/128 * 2^-126 */
    else if (e == 255) v = m ? NAN : INFINITY;
    else v = ldexp(1.0 + m / 128.0, e - 127);
    return s ? -v : v;
}

/* OCP FP8 E4M3 ("fn"): bias 7, no infinities, S.1111.111 is NaN */
double oracle_e4m3(int c)
{
    int s = (c >> 7) & 1, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp(m / 8.0, -6);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* OCP FP4 E2M1: bias 1, exponent 0 is subnormal (0 or 0.5) */
double oracle_e2m1(int c)
{
    int s = (c >> 3) & 1, e = (c >> 1) & 3, m = c & 1;
    double v = e == 0 ? 0.5 * m : ldexp(1.0 + m / 2.0, e - 1);
    return s ? -v : v;
}

static uint16_t rd16(const uint8_t *p) { return (uint16_t)(p[0] | (p[1] << 8)); }

static uint32_t rd32(const uint8_t *p)
{
    return (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
}

int64_t oracle_row_bytes(int fmt, int64_t cols)
{
    switch (fmt) {
    case ORACLE_Q8_0: return cols / 32 * 34;
    case ORACLE_Q5_1: return cols / 32 * 24;
    case ORACLE_Q5_0: return cols / 32 * 22;
    case ORACLE_IQ4_NL: return cols / 32 * 18;
    case ORACLE_NVFP4: return cols / 16 * 9;
    default: return -1;
    }
}

/* Dequantise one row of `cols` weights stored as consecutive blocks. */
int oracle_decode_row(int fmt, const uint8_t *row, int64_t cols, const int8_t *table,
                      double tensor_scale, double *out)
{
    if (fmt == ORACLE_NVFP4) {
        if (cols % 16) return -1;
        for (int64_t b = 0; b < cols / 16; ++b) {
            const uint8_t *blk = row + b * 9;
            double sc = tensor_scale * oracle_e4m3(blk[0]);
            for (int j = 0; j < 16; ++j) {
                int nib = (j & 1) ? (blk[1 + j / 2] >> 4) : (blk[1 + j / 2] & 15);
                out[b * 16 + j] = sc * oracle_e2m1(nib);
            }
        }
        return 0;
    }
    if (cols % 32) return -1;
    for (int64_t b = 0; b < cols / 32; ++b) {
        double *o = out + b * 32;
        switch (fmt) {
        case ORACLE_Q8_0: {
            const uint8_t *blk = row + b * 34;
            double d = oracle_fp16(rd16(blk));
            for (int j = 0; j < 32; ++j) o[j] = d * (double)(int8_t)blk[2 + j];
            break;
        }
        case ORACLE_Q5_1: {
            const uint8_t *blk = row + b * 24;
            double d = oracle_fp16(rd16(blk)), m = oracle_fp16(rd16(blk + 2));
            uint32_t qh = rd32(blk + 4);
            const uint8_t *qs = blk + 8;
            for (int j = 0; j < 32; ++j) {
                int lo = j < 16 ? (qs[j] & 15) : (qs[j - 16] >> 4);
                int q = lo | (int)(((qh >> j) & 1u) << 4);
                o[j] = d * q + m;
            }
            break;
        }
        case ORACLE_Q5_0: {
            const uint8_t *blk = row + b * 22;
            double d = oracle_fp16(rd16(blk));
            uint32_t qh = rd32(blk + 2);
            const uint8_t *qs = blk + 6;
            for (int j = 0; j < 32; ++j) {
                int lo = j < 16 ? (qs[j] & 15) : (qs[j - 16] >> 4);
                int q = lo | (int)(((qh >> j) & 1u) << 4);
                o[j] = d * (double)(q - 16);
            }
            break;
        }
        case ORACLE_IQ4_NL: {
            if (!table) return -2;
            const uint8_t *blk = row + b * 18;
            double d = oracle_fp16(rd16(blk));
            const uint8_t *qs = blk + 2;
            for (int j = 0; j < 32; ++j) {
                int i = j < 16 ? (qs[j] & 15) : (qs[j - 16] >> 4);
                o[j] = d * (double)table[i];
            }
            break;
        }
        default: return -3;
        }
    }
    return 0;
}

/* ---- routing ------------------------------------------------------------ */

/* Logits, top-k (descending logit, ties to the lower expert index) and the
 * renormalised gates of one token. */
void oracle_route_token(const double *x, const uint16_t *wr, int H, int E, int k, int32_t *idx,
                        double *gate, double *logits)
{
    double *l = logits ? logits : (double *)malloc(sizeof(double) * (size_t)E);
    for (int e = 0; e < E; ++e) {
        double s = 0.0;
        for (int h = 0; h < H; ++h) s += oracle_bf16(wr[(int64_t)e * H + h]) * x[h];
        l[e] = s;
    }
    /* selection: k passes of "largest remaining, lowest index on ties" */
    char *taken = (char *)calloc((size_t)E, 1);
    for (int j = 0; j < k; ++j) {
        int best = -1;
        for (int e = 0; e < E; ++e)
            if (!taken[e] && (best < 0 || l[e] > l[best])) best = e;
        taken[best] = 1;
        idx[j] = best;
    }
    double m = l[idx[0]], den = 0.0;
    for (int j = 0; j < k; ++j) den += exp(l[idx[j]] - m);
    for (int j = 0; j < k; ++j) gate[j] = exp(l[idx[j]] - m) / den;
    free(taken);
    if (!logits) free(l);
}

void oracle_route(const double *x, const uint16_t *wr, int T, int H, int E, int k, int32_t *idx,
                  double *gate, double *logits)
{
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int t = 0; t < T; ++t)
        oracle_route_token(x + (int64_t)t * H, wr, H, E, k, idx + (int64_t)t * k,
                           gate + (int64_t)t * k, logits ? logits + (int64_t)t * E : NULL);
}

/* ---- activation quantisation (NVFP4 prefill reading) ---------------------- */

static double e4m3_rne_satfinite_f32(float a) /* a >= 0 */
{
    if (!(a > 0.f)) return 0.0;
    if ((double)a >= 448.0) return 448.0;
    /* value grid: subnormals m/8*2^-6 (step 2^-9) below 2^-6, then step
     * 2^(e-10) in [2^(e-7), 2^(e-6)) */
    int ex;
    frexp((double)a, &ex); /* a = f * 2^ex, f in [0.5, 1) */
    int e = ex - 1;        /* a in [2^e, 2^(e+1)) */
    double step = e < -6 ? ldexp(1.0, -9) : ldexp(1.0, e - 3);
    double q = (double)a / step, r = floor(q), f = q - r;
    if (f > 0.5 || (f == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
    double v = r * step;
    return v > 448.0 ? 448.0 : v;
}

static double e2m1_rne_satfinite_f32(float v)
{
    float a = fabsf(v);
    double m = a <= 0.25f ? 0.0 : a < 0.75f ? 0.5 : a <= 1.25f ? 1.0 : a < 1.75f ? 1.5
             : a <= 2.5f ? 2.0 : a < 3.5f ? 3.0 : a <= 5.f ? 4.0 : 6.0;
    return v < 0.f ? -m : m;
}

/* Round one activation vector of n values (n a multiple of 16) to NVFP4 with
 * a per-vector fp32 scale; writes the dequantised values. */
void oracle_act_quant_nvfp4(const double *in, int64_t n, double *out)
{
    float amax = 0.f;
    for (int64_t i = 0; i < n; ++i) amax = fmaxf(amax, fabsf((float)in[i]));
    float s = amax / (6.f * 448.f);
    if (!(s > 0.f)) {
        for (int64_t i = 0; i < n; ++i) out[i] = 0.0;
        return;
    }
    for (int64_t b = 0; b < n / 16; ++b) {
        float bmax = 0.f;
        for (int j = 0; j < 16; ++j) bmax = fmaxf(bmax, fabsf((float)in[b * 16 + j]));
        double sb = e4m3_rne_satfinite_f32(bmax / (6.f * s));
        float denom = s * (float)sb;
        for (int j = 0; j < 16; ++j) {
            double c = sb > 0.0 ? e2m1_rne_satfinite_f32((float)in[b * 16 + j] / denom) : 0.0;
            out[b * 16 + j] = (double)s * sb * c;
        }
    }
}

/* ---- experts and the layer --------------------------------------------- */

/* Blocks of expert e (e = n_experts: the shared expert) of one projection. */
static const uint8_t *expert_ptr(const oracle_desc *d, int proj, int e)
{
    if (e < 0 || e > d->n_experts || (e == d->n_experts && !d->has_shared)) return NULL;
    if (proj == 0) return d->gate_up + (int64_t)e * oracle_row_bytes(d->fmt_gate_up, d->hidden) * 2 * d->inter;
    return d->down + (int64_t)e * oracle_row_bytes(d->fmt_down, d->inter) * d->hidden;
}

/* One expert's SwiGLU FFN on one token: y = D (silu(G x) * (U x)). */
int oracle_expert(const oracle_desc *d, int e, const double *x, double *y, int act_quant)
{
    int H = d->hidden, I = d->inter;
    const uint8_t *gu = expert_ptr(d, 0, e), *dn = expert_ptr(d, 1, e);
    if (!gu || !dn) return -4;
    double gts = d->gate_up_scale ? d->gate_up_scale[e] : 1.0;
    double dts = d->down_scale ? d->down_scale[e] : 1.0;
    int64_t gub = oracle_row_bytes(d->fmt_gate_up, H), dnb = oracle_row_bytes(d->fmt_down, I);
    double *row = (double *)malloc(sizeof(double) * (size_t)(H > I ? H : I));
    double *hv = (double *)malloc(sizeof(double) * (size_t)I);
    double *xq = NULL;
    int rc = 0;
    const double *xin = x;
    if (act_quant == 1) {
        xq = (double *)malloc(sizeof(double) * (size_t)H);
        oracle_act_quant_nvfp4(x, H, xq);
        xin = xq;
    }
    for (int i = 0; i < I && !rc; ++i) {
        double a = 0.0, b = 0.0;
        rc |= oracle_decode_row(d->fmt_gate_up, gu + (int64_t)i * gub, H, d->table, gts, row);
        for (int h = 0; h < H; ++h) a += row[h] * xin[h];
        rc |= oracle_decode_row(d->fmt_gate_up, gu + (int64_t)(I + i) * gub, H, d->table, gts, row);
        for (int h = 0; h < H; ++h) b += row[h] * xin[h];
        hv[i] = a / (1.0 + exp(-a)) * b;
    }
    if (act_quant == 1 && !rc) oracle_act_quant_nvfp4(hv, I, hv);
    for (int r = 0; r < H && !rc; ++r) {
        double s = 0.0;
        rc |= oracle_decode_row(d->fmt_down, dn + (int64_t)r * dnb, I, d->table, dts, row);
        for (int i = 0; i < I; ++i) s += row[i] * hv[i];
        y[r] = s;
    }
    free(row);
    free(hv);
    free(xq);
    return rc;
}

/* The whole layer on T tokens.  idx/gate (T*k each) may be NULL. */
int oracle_layer(const oracle_desc *d, const double *x, const uint16_t *wr, int T, int k,
                 double *out, int32_t *idx_out, double *gate_out, int act_quant)
{
    int H = d->hidden, E = d->n_experts;
    if (k < 1 || k > E) return -5;
    int rc_all = 0;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int t = 0; t < T; ++t) {
        int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (size_t)k);
        double *gate = (double *)malloc(sizeof(double) * (size_t)k);
        double *y = (double *)malloc(sizeof(double) * (size_t)H);
        const double *xt = x + (int64_t)t * H;
        double *o = out + (int64_t)t * H;
        int rc = 0;
        oracle_route_token(xt, wr, H, E, k, idx, gate, NULL);
        for (int h = 0; h < H; ++h) o[h] = 0.0;
        for (int j = 0; j < k && !rc; ++j) {
            rc = oracle_expert(d, idx[j], xt, y, act_quant);
            for (int h = 0; h < H; ++h) o[h] += gate[j] * y[h];
        }
        if (d->has_shared && !rc) {
            rc = oracle_expert(d, E, xt, y, act_quant);
            for (int h = 0; h < H; ++h) o[h] += y[h];
        }
        if (idx_out) memcpy(idx_out + (int64_t)t * k, idx, sizeof(int32_t) * (size_t)k);
        if (gate_out) memcpy(gate_out + (int64_t)t * k, gate, sizeof(double) * (size_t)k);
        if (rc) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            rc_all = rc;
        }
        free(idx);
        free(gate);
        free(y);
    }
    return rc_all;
}

int oracle_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads the layer uses from now on (n >= 1), for timing the oracle on one core. */
void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n >= 1) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
