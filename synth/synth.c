/*
 * Seeded synthetic inputs for the block-quantised routed MoE layer.
 *
 * This module draws the inputs that both the fp64 oracle and the CUDA path
 * consume: Gaussian numbers from a counter-based generator, rounded to the
 * storage types (bf16 / fp16 / fp32), and weight matrices encoded into the
 * canonical block formats.  It holds none of the layer's arithmetic: no
 * block decoding, no expert FFN, no routing output.  The one place it forms
 * router logits is rejection sampling of the token vectors, so that the gap
 * between the k-th and (k+1)-th logit is at least a stated margin (an input
 * constraint, computed here in fp64 on its own).
 *
 * Canonical block layouts (byte offsets inside one block, little endian):
 *   Q8_0   34 B per 32 weights : [0,2) fp16 d, [2,34) int8 q[32]          w = d*q
 *   Q5_1   24 B per 32 weights : [0,2) fp16 d, [2,4) fp16 m, [4,8) u32 qh,
 *                                [8,24) qs[16]; element j<16 is the low
 *                                nibble of qs[j], j>=16 the high nibble of
 *                                qs[j-16]; bit 4 of element j is bit j of qh
 *                                                                      w = d*q + m
 *   IQ4_NL 18 B per 32 weights : [0,2) fp16 d, [2,18) qs[16], nibble order
 *                                as Q5_1                               w = d*T[q]
 *   NVFP4   9 B per 16 weights : [0] E4M3 block scale, [1,9) nibbles, element
 *                                2i the low and 2i+1 the high nibble of byte i,
 *                                plus one fp32 scale per matrix     w = s*e4m3*e2m1
 *
 * Counter-based generator: SplitMix64 (Steele, Lea, Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014).  Sample i of the stream with
 * key K uses the 64-bit output of state K + (i/4 + 1)*golden; its four 16-bit
 * fields index a 65536-entry table of standard-normal quantiles
 * z_j = Phi^-1((j + 0.5) / 65536), so every value can be regenerated alone.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define GOLDEN 0x9E3779B97F4A7C15ULL

enum { FMT_Q8_0 = 1, FMT_Q5_1 = 2, FMT_IQ4_NL = 3, FMT_NVFP4 = 4, FMT_Q5_0 = 5 };
enum { DT_F32 = 1, DT_BF16 = 2 };

static uint64_t mix64(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint64_t synth_key(uint64_t seed, uint64_t a, uint64_t b, uint64_t c, uint64_t d)
{
    uint64_t k = mix64(seed + GOLDEN);
    k = mix64(k ^ (a + 1 * GOLDEN));
    k = mix64(k ^ (b + 2 * GOLDEN));
    k = mix64(k ^ (c + 3 * GOLDEN));
    k = mix64(k ^ (d + 4 * GOLDEN));
    return k;
}

/* ---- standard normal quantile table ----------------------------------- */
static float g_ztab[65536];
static pthread_once_t g_ztab_once = PTHREAD_ONCE_INIT;

static double norm_cdf(double z) { return 0.5 * erfc(-z / sqrt(2.0)); }

static void ztab_init(void)
{
    for (int j = 0; j < 32768; ++j) {
        double p = (j + 0.5) / 65536.0;
        double lo = -12.0, hi = 0.0;
        for (int it = 0; it < 80; ++it) {
            double mid = 0.5 * (lo + hi);
            if (norm_cdf(mid) < p) lo = mid; else hi = mid;
        }
        float z = (float)(0.5 * (lo + hi));
        g_ztab[j] = z;
        g_ztab[65535 - j] = -z;
    }
}

const float *synth_normal_table(void)
{
    pthread_once(&g_ztab_once, ztab_init);
    return g_ztab;
}

static inline float normal_at(uint64_t key, int64_t i)
{
    uint64_t h = mix64(key + (uint64_t)((i >> 2) + 1) * GOLDEN);
    return g_ztab[(h >> (16 * (i & 3))) & 0xFFFF];
}

void synth_normal_f32(uint64_t key, int64_t n, float sigma, float *out)
{
    pthread_once(&g_ztab_once, ztab_init);
    int64_t i = 0;
    for (; i + 4 <= n; i += 4) {
        uint64_t h = mix64(key + (uint64_t)((i >> 2) + 1) * GOLDEN);
        out[i] = sigma * g_ztab[h & 0xFFFF];
        out[i + 1] = sigma * g_ztab[(h >> 16) & 0xFFFF];
        out[i + 2] = sigma * g_ztab[(h >> 32) & 0xFFFF];
        out[i + 3] = sigma * g_ztab[h >> 48];
    }
    for (; i < n; ++i) out[i] = sigma * normal_at(key, i);
}

uint64_t synth_u64(uint64_t key, int64_t i) { return mix64(key + (uint64_t)(i + 1) * GOLDEN); }

/* ---- storage-type rounding --------------------------------------------- */
static inline uint16_t f32_to_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

static inline float bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

static inline uint16_t f32_to_f16_rne(float f)
{
    _Float16 h = (_Float16)f; /* IEEE round-to-nearest-even */
    uint16_t u;
    memcpy(&u, &h, 2);
    return u;
}

static inline float f16_to_f32(uint16_t u)
{
    _Float16 h;
    memcpy(&h, &u, 2);
    return (float)h;
}

void synth_round_bf16(const float *in, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = f32_to_bf16_rne(in[i]);
}


/* scalar helpers the compiler keeps inline (no libm calls, no NaNs here) */
static inline float fmin_(float a, float b) { return a < b ? a : b; }
static inline float fmax_(float a, float b) { return a > b ? a : b; }
static inline float fabs_(float a) { return a < 0.f ? -a : a; }
/* round half away from zero, exact for |x| < 2^31; branch-free because
 * Gaussian data makes the two tests unpredictable */
static inline float round_away(float x)
{
    float r = (float)(int32_t)x;
    float f = x - r; /* exact */
    return r + (float)(f >= 0.5f) - (float)(f <= -0.5f);
}

/* ---- block encoders ----------------------------------------------------- */
int64_t synth_row_bytes(int fmt, int64_t cols)
{
    switch (fmt) {
    case FMT_Q8_0: return cols / 32 * 34;
    case FMT_Q5_1: return cols / 32 * 24;
    case FMT_Q5_0: return cols / 32 * 22;
    case FMT_IQ4_NL: return cols / 32 * 18;
    case FMT_NVFP4: return cols / 16 * 9;
    default: return -1;
    }
}

static void put16(uint8_t *p, uint16_t v) { p[0] = (uint8_t)v; p[1] = (uint8_t)(v >> 8); }

static void enc_q8_0(const float *w, uint8_t *blk)
{
    float amax = 0.f;
    for (int j = 0; j < 32; ++j) amax = fmax_(amax, fabs_(w[j]));
    uint16_t dh = f32_to_f16_rne(amax / 127.f);
    float d = f16_to_f32(dh);
    put16(blk, dh);
    for (int j = 0; j < 32; ++j) {
        float q = d == 0.f ? 0.f : round_away(w[j] / d);
        q = fmin_(127.f, fmax_(-127.f, q));
        blk[2 + j] = (uint8_t)(int8_t)q;
    }
}

static void enc_q5_1(const float *w, uint8_t *blk)
{
    float mn = w[0], mx = w[0];
    for (int j = 1; j < 32; ++j) { mn = fmin_(mn, w[j]); mx = fmax_(mx, w[j]); }
    uint16_t dh = f32_to_f16_rne((mx - mn) / 31.f);
    uint16_t mh = f32_to_f16_rne(mn);
    float d = f16_to_f32(dh), m = f16_to_f32(mh);
    put16(blk, dh);
    put16(blk + 2, mh);
    uint32_t qh = 0;
    uint8_t *qs = blk + 8;
    memset(qs, 0, 16);
    for (int j = 0; j < 32; ++j) {
        float q = d == 0.f ? 0.f : round_away((w[j] - m) / d);
        int qi = (int)fmin_(31.f, fmax_(0.f, q));
        if (j < 16) qs[j] |= (uint8_t)(qi & 15);
        else qs[j - 16] |= (uint8_t)((qi & 15) << 4);
        qh |= (uint32_t)((qi >> 4) & 1) << j;
    }
    blk[4] = (uint8_t)qh; blk[5] = (uint8_t)(qh >> 8);
    blk[6] = (uint8_t)(qh >> 16); blk[7] = (uint8_t)(qh >> 24);
}

/* Q5_0: the element of largest magnitude v sets d = -v/16 (fp16), so it gets
 * code 0; the others q = round(w/d) + 16, clamped to [0, 31]. */
static void enc_q5_0(const float *w, uint8_t *blk)
{
    int jx = 0;
    for (int j = 1; j < 32; ++j) if (fabs_(w[j]) > fabs_(w[jx])) jx = j;
    uint16_t dh = f32_to_f16_rne(-w[jx] / 16.f);
    float d = f16_to_f32(dh);
    put16(blk, dh);
    uint32_t qh = 0;
    uint8_t *qs = blk + 6;
    memset(qs, 0, 16);
    for (int j = 0; j < 32; ++j) {
        float q = d == 0.f ? 16.f : round_away(w[j] / d) + 16.f;
        int qi = (int)fmin_(31.f, fmax_(0.f, q));
        if (j < 16) qs[j] |= (uint8_t)(qi & 15);
        else qs[j - 16] |= (uint8_t)((qi & 15) << 4);
        qh |= (uint32_t)((qi >> 4) & 1) << j;
    }
    blk[2] = (uint8_t)qh; blk[3] = (uint8_t)(qh >> 8);
    blk[4] = (uint8_t)(qh >> 16); blk[5] = (uint8_t)(qh >> 24);
}

/* nearest table entry, ties to the lower index.  The table is sorted by value
 * (equal values keep their lowest index); v falls above boundary i when it is
 * past the midpoint of sorted entries i and i+1, or on it and entry i+1 has the
 * lower index.  The count of boundaries passed is v's sorted position. */
typedef struct { float mid[16]; int up_on_tie[16]; int idx[16]; int n; } iq4_sorted;

static void iq4_prepare(const int8_t *T, iq4_sorted *s)
{
    int order[16];
    float v[16];
    for (int c = 0; c < 16; ++c) order[c] = c;
    for (int a = 1; a < 16; ++a) /* stable insertion sort by value */
        for (int b = a; b > 0 && T[order[b - 1]] > T[order[b]]; --b) {
            int t = order[b]; order[b] = order[b - 1]; order[b - 1] = t;
        }
    s->n = 0;
    for (int a = 0; a < 16; ++a) {
        if (s->n && v[s->n - 1] == (float)T[order[a]]) continue;
        v[s->n] = (float)T[order[a]];
        s->idx[s->n] = order[a];
        s->n++;
    }
    for (int i = 0; i < 15; ++i) {
        s->mid[i] = i + 1 < s->n ? 0.5f * (v[i] + v[i + 1]) : INFINITY;
        s->up_on_tie[i] = i + 1 < s->n && s->idx[i + 1] < s->idx[i];
    }
}

static int iq4_nearest(float v, const iq4_sorted *s)
{
    int pos = 0;
    for (int i = 0; i < 15; ++i) pos += (v > s->mid[i]) | ((v == s->mid[i]) & s->up_on_tie[i]);
    return s->idx[pos];
}

static void enc_iq4_nl(const float *w, uint8_t *blk, const int8_t *T, const iq4_sorted *s)
{
    int jx = 0;
    for (int j = 1; j < 32; ++j) if (fabs_(w[j]) > fabs_(w[jx])) jx = j;
    int cx = 0;
    for (int c = 1; c < 16; ++c) if (abs(T[c]) > abs(T[cx])) cx = c;
    /* the block's extreme element maps onto the table's extreme entry */
    uint16_t dh = f32_to_f16_rne(T[cx] == 0 ? 0.f : w[jx] / (float)T[cx]);
    float d = f16_to_f32(dh);
    put16(blk, dh);
    uint8_t *qs = blk + 2;
    memset(qs, 0, 16);
    for (int j = 0; j < 32; ++j) {
        int q = iq4_nearest(d == 0.f ? 0.f : w[j] / d, s);
        if (j < 16) qs[j] |= (uint8_t)q;
        else qs[j - 16] |= (uint8_t)(q << 4);
    }
}

static double e4m3_value(int c)
{
    int e = (c >> 3) & 15, m = c & 7;
    return e == 0 ? ldexp(m / 8.0, -6) : ldexp(1.0 + m / 8.0, e - 7);
}

/* E4M3 (OCP FP8 "fn") encode of a non-negative value: nearest, ties to the
 * code with an even mantissa, saturating at 448 (code 0x7E). */
static int e4m3_encode_rne_sat(double a)
{
    if (!(a > 0.0)) return 0;
    int lo = 0, hi = 126;
    if (a >= e4m3_value(126)) return 126;
    while (hi - lo > 1) { /* invariant: value(lo) <= a < value(hi) */
        int mid = (lo + hi) / 2;
        if (e4m3_value(mid) <= a) lo = mid; else hi = mid;
    }
    double dl = a - e4m3_value(lo), dh = e4m3_value(hi) - a;
    if (dl < dh) return lo;
    if (dh < dl) return hi;
    return (lo & 1) ? hi : lo;
}

/* E2M1 encode, round to nearest even, saturating at 6 */
static int e2m1_encode_rne_sat(float v)
{
    /* codes 0..7 are 0, .5, 1, 1.5, 2, 3, 4, 6; midpoints tie to the even code */
    float a = fabs_(v);
    int c = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) + (a >= 3.5f)
          + (a > 5.f);
    return c | (signbit(v) ? 8 : 0);
}

static void enc_nvfp4(const float *w, uint8_t *blk, float s_t)
{
    float amax = 0.f;
    for (int j = 0; j < 16; ++j) amax = fmax_(amax, fabs_(w[j]));
    int sb = e4m3_encode_rne_sat((double)(amax / (6.f * s_t)));
    float sbv = (float)e4m3_value(sb);
    blk[0] = (uint8_t)sb;
    for (int i = 0; i < 8; ++i) {
        int n0 = 0, n1 = 0;
        if (sbv > 0.f) {
            n0 = e2m1_encode_rne_sat(w[2 * i] / (s_t * sbv));
            n1 = e2m1_encode_rne_sat(w[2 * i + 1] / (s_t * sbv));
        }
        blk[1 + i] = (uint8_t)(n0 | (n1 << 4));
    }
}

/* Encode a rows x cols row-major fp32 matrix into canonical blocks laid out
 * row by row (blocks run along cols).  NVFP4 also writes the matrix scale
 * s = amax / (6 * 448) to *tensor_scale (1 for an all-zero matrix). */
int synth_encode(int fmt, const float *w, int64_t rows, int64_t cols, const int8_t *table,
                 uint8_t *blocks, float *tensor_scale)
{
    int64_t bw = fmt == FMT_NVFP4 ? 16 : 32;
    if (cols % bw) return -1;
    if (fmt == FMT_IQ4_NL && !table) return -2;
    int64_t rb = synth_row_bytes(fmt, cols);
    if (rb < 0) return -3;
    float s_t = 1.f;
    iq4_sorted srt;
    srt.n = 0;
    if (fmt == FMT_IQ4_NL) iq4_prepare(table, &srt);
    if (fmt == FMT_NVFP4) {
        float amax = 0.f;
        for (int64_t i = 0; i < rows * cols; ++i) amax = fmax_(amax, fabs_(w[i]));
        s_t = amax > 0.f ? amax / (6.f * 448.f) : 1.f;
        if (tensor_scale) *tensor_scale = s_t;
    }
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < cols / bw; ++b) {
            const float *src = w + r * cols + b * bw;
            uint8_t *dst = blocks + r * rb + b * (rb / (cols / bw));
            switch (fmt) {
            case FMT_Q8_0: enc_q8_0(src, dst); break;
            case FMT_Q5_1: enc_q5_1(src, dst); break;
            case FMT_Q5_0: enc_q5_0(src, dst); break;
            case FMT_IQ4_NL: enc_iq4_nl(src, dst, table, &srt); break;
            case FMT_NVFP4: enc_nvfp4(src, dst, s_t); break;
            }
        }
    }
    return 0;
}

/* ---- whole inputs ------------------------------------------------------- */
enum { TAG_X = 1, TAG_ROUTER = 2, TAG_GATE_UP = 3, TAG_DOWN = 4, TAG_RANK = 5, TAG_XBASE = 6 };

/* One expert's weights: gate/up stacked [2I x H] (rows 0..I-1 gate, I..2I-1
 * up) and down [H x I], each drawn N(0, sigma^2) and encoded. */
int synth_expert(uint64_t seed, int layer, int expert, int fmt_gu, int fmt_dn, int H, int I,
                 float sigma, const int8_t *table, uint8_t *gu_blocks, uint8_t *dn_blocks,
                 float *gu_ts, float *dn_ts, float *scratch /* >= 2*I*H floats, or NULL */)
{
    pthread_once(&g_ztab_once, ztab_init);
    float *w = scratch ? scratch : (float *)malloc(sizeof(float) * (size_t)2 * I * H);
    if (!w) return -10;
    int rc = 0;
    if (gu_blocks) {
        synth_normal_f32(synth_key(seed, (uint64_t)layer, TAG_GATE_UP, (uint64_t)expert, 0),
                         (int64_t)2 * I * H, sigma, w);
        rc = synth_encode(fmt_gu, w, 2 * I, H, table, gu_blocks, gu_ts);
    }
    if (!rc && dn_blocks) {
        synth_normal_f32(synth_key(seed, (uint64_t)layer, TAG_DOWN, (uint64_t)expert, 0),
                         (int64_t)H * I, sigma, w);
        rc = synth_encode(fmt_dn, w, H, I, table, dn_blocks, dn_ts);
    }
    if (!scratch) free(w);
    return rc;
}

/* Experts [e0, e0+n) of one layer, in parallel over experts.  Expert e lands
 * at gu_blocks + (e-e0)*gate_up_bytes (likewise down / scales). */
int synth_layer_experts(uint64_t seed, int layer, int e0, int n, int fmt_gu, int fmt_dn, int H,
                        int I, float sigma, const int8_t *table, uint8_t *gu_blocks,
                        uint8_t *dn_blocks, float *gu_ts, float *dn_ts, int nthreads)
{
    pthread_once(&g_ztab_once, ztab_init);
    int64_t gub = synth_row_bytes(fmt_gu, H) * 2 * I;
    int64_t dnb = synth_row_bytes(fmt_dn, I) * H;
    int rc_all = 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads)
#endif
    {
        float *w = (float *)malloc(sizeof(float) * (size_t)2 * I * H);
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (int i = 0; i < n; ++i) {
            int rc = w ? synth_expert(seed, layer, e0 + i, fmt_gu, fmt_dn, H, I, sigma, table,
                                      gu_blocks ? gu_blocks + i * gub : NULL,
                                      dn_blocks ? dn_blocks + i * dnb : NULL,
                                      gu_ts ? gu_ts + i : NULL, dn_ts ? dn_ts + i : NULL, w)
                       : -10;
            if (rc) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
                rc_all = rc;
            }
        }
        free(w);
    }
    return rc_all;
}

/* Router weights, bf16 [E x H], N(0, sigma^2).  With zipf_s > 0 the last
 * column becomes a popularity bias: Wr[e][H-1] = -beta*zipf_s*ln(rank(e)),
 * rank a seeded permutation of 1..E; the token vectors then carry a constant
 * 1 in coordinate H-1. */
void synth_router(uint64_t seed, int layer, int E, int H, float sigma, float zipf_s, float beta,
                  uint16_t *wr, int32_t *rank_out)
{
    pthread_once(&g_ztab_once, ztab_init);
    uint64_t key = synth_key(seed, (uint64_t)layer, TAG_ROUTER, 0, 0);
    for (int64_t i = 0; i < (int64_t)E * H; ++i) wr[i] = f32_to_bf16_rne(sigma * normal_at(key, i));
    if (zipf_s > 0.f) {
        int32_t *perm = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
        uint64_t rk = synth_key(seed, (uint64_t)layer, TAG_RANK, 0, 0);
        for (int e = 0; e < E; ++e) perm[e] = e;
        for (int e = E - 1; e > 0; --e) { /* Fisher-Yates */
            int j = (int)(synth_u64(rk, e) % (uint64_t)(e + 1));
            int t = perm[e]; perm[e] = perm[j]; perm[j] = t;
        }
        for (int r = 0; r < E; ++r) { /* expert perm[r] has popularity rank r+1 */
            int e = perm[r];
            wr[(int64_t)e * H + H - 1] = f32_to_bf16_rne(-beta * zipf_s * logf((float)(r + 1)));
            if (rank_out) rank_out[e] = r + 1;
        }
        free(perm);
    }
}

/* Gap between the k-th and (k+1)-th largest router logit of one token, in
 * fp64 (bf16 and fp32 inputs are exact there). */
static double topk_gap(const float *x, const uint16_t *wr, int E, int H, int k, double *buf)
{
    int m = k + 1;
    for (int i = 0; i < m; ++i) buf[i] = -INFINITY;
    for (int e = 0; e < E; ++e) {
        double s = 0.0;
        const uint16_t *row = wr + (int64_t)e * H;
        for (int h = 0; h < H; ++h) s += (double)bf16_to_f32(row[h]) * (double)x[h];
        if (s > buf[m - 1]) {
            int p = m - 1;
            while (p > 0 && buf[p - 1] < s) { buf[p] = buf[p - 1]; --p; }
            buf[p] = s;
        }
    }
    return buf[k - 1] - buf[k];
}

/* Token vectors for one (layer, step): T x H, fp32 (dtype 1) or bf16 bits
 * (dtype 2).  corr == 0: x = z; corr > 0: x = b + corr*z with one base
 * vector b per (layer, step).  bias_feature sets x[H-1] = 1.  When
 * 0 < k < E and margin > 0, each token is redrawn until its top-k logit gap
 * is at least margin.  Returns the number of redraws, or -1 if a token ran
 * out of attempts. */
int64_t synth_tokens(uint64_t seed, int layer, int step, int T, int H, int dtype, float corr,
                     int bias_feature, const uint16_t *wr, int E, int k, double margin,
                     void *out, int max_attempts)
{
    pthread_once(&g_ztab_once, ztab_init);
    float *base = NULL;
    if (corr > 0.f) {
        base = (float *)malloc(sizeof(float) * (size_t)H);
        synth_normal_f32(synth_key(seed, (uint64_t)layer, TAG_XBASE, (uint64_t)step, 0), H, 1.f, base);
    }
    int64_t redraws = 0;
    int failed = 0;
    int check = wr && k > 0 && k < E && margin > 0.0;
#ifdef _OPENMP
#pragma omp parallel reduction(+ : redraws)
#endif
    {
        float *x = (float *)malloc(sizeof(float) * (size_t)H);
        double *buf = (double *)malloc(sizeof(double) * (size_t)(k + 2));
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 8)
#endif
        for (int t = 0; t < T; ++t) {
            int ok = 0;
            for (int a = 0; a < max_attempts && !ok; ++a) {
                uint64_t key = synth_key(seed, (uint64_t)layer, TAG_X, (uint64_t)step,
                                         (uint64_t)t * 4096u + (uint64_t)a);
                for (int h = 0; h < H; ++h) {
                    float z = normal_at(key, h);
                    float v = base ? base[h] + corr * z : z;
                    if (dtype == DT_BF16) v = bf16_to_f32(f32_to_bf16_rne(v));
                    x[h] = v;
                }
                if (bias_feature) x[H - 1] = 1.f;
                ok = !check || topk_gap(x, wr, E, H, k, buf) >= margin;
                if (!ok) redraws++;
            }
            if (!ok) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
                failed = 1;
            }
            if (dtype == DT_BF16) {
                uint16_t *o = (uint16_t *)out + (int64_t)t * H;
                for (int h = 0; h < H; ++h) o[h] = f32_to_bf16_rne(x[h]);
            } else {
                memcpy((float *)out + (int64_t)t * H, x, sizeof(float) * (size_t)H);
            }
        }
        free(x);
        free(buf);
    }
    free(base);
    return failed ? -1 : redraws;
}
