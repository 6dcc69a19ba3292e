/*
 * hcl_oracle.c -- plain, slow, fp64 CPU oracle of the CSA / HCA hybrid-attention hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg may load this library.  It shares no code, header, table or constant
 * with the CUDA library: every format decoder and encoder below is written here from its
 * published definition.
 *
 * References (web write-ups of the DeepSeek-V4 technical report):
 *   [Tripbot]  "论文解读｜DeepSeek-V4：百万 token 上下文的效率革命", blog.tripbot.top
 *              §3.1 (CSA: 4:1 softmax-gated pooling with a learned position bias, lightning
 *              indexer, top-k), §3.2 (HCA: 128:1 pooling, dense attention), §3.3 (128-token
 *              sliding-window branch, learnable attention sink).
 *   [CSDN]     "从论文出发，逐层剖析 CSA / HCA 混合注意力、mHC 残差连接与 Muon 优化器",
 *              gitcode.csdn.net, §1.1 and its "工程细节" paragraph (overlapped compression:
 *              entry i pools the current m tokens C^a and the previous window's last m
 *              tokens C^b), §1.2 (HCA), §1.4 (BF16 RoPE dims / FP8 other dims; FP4 indexer
 *              QK product; index scores quantised from FP32 to BF16).
 *   [Austery]  DeepSeek-V4 talk notes, austery.github.io, infrastructure section (MXFP4
 *              quantisation of the indexer QK path).
 *   OCP Microscaling Formats (MX) v1.0: E2M1 element, E8M0 shared scale, block of 32,
 *              X = 2^(floor(log2(amax)) - emax_elem) with emax_elem = 2 for E2M1.
 *   OFP8 (E4M3 "fn"): bias 7, no infinities, max finite 448.
 *
 * Readings of the pages taken here where they are silent (each is listed in the design
 * notes): slots outside [0, L) are masked out of the pooling softmax; gate logits are
 * per token and channel, the bias is one scalar per slot; an entry is visible to a query
 * at position p once its last token is <= p; one compressed row is both key and value;
 * index scores carry no scale; top-k ties go to the lower index; window rows and
 * compressed entries are distinct items of one softmax; the softmax scale is 1/sqrt(d).
 *
 * Build: gcc -O2 -ffp-contract=off -fopenmp -shared -fPIC (no fast-math).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------------------ */
/* scalar formats                                                                         */

/* bf16: the top 16 bits of an IEEE binary32. */
double or_bf16_to_f64(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Round a double to the nearest bf16 (ties to even), returned as bf16 bits.
 * bf16 keeps 8 significant bits; normal exponents -126..127; subnormal quantum 2^-133. */
uint16_t or_f64_to_bf16(double x)
{
    if (isnan(x)) return 0x7FC0;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (isinf(a)) return sign | 0x7F80;
    if (a == 0.0) return sign;
    int e = ilogb(a);                          /* floor(log2 a) */
    int qexp = (e < -126) ? -133 : e - 7;      /* exponent of one unit in the last place */
    double r = nearbyint(ldexp(a, -qexp));     /* round to nearest, ties to even */
    double v = ldexp(r, qexp);
    if (v >= ldexp(1.0, 128)) return sign | 0x7F80;   /* overflow -> inf */
    float f = (float)v;                        /* exact: v is a bf16 value */
    uint32_t u;
    memcpy(&u, &f, 4);
    return sign | (uint16_t)((u >> 16) & 0x7FFF);
}

/* E4M3 ("fn") code -> value.  bias 7; exponent field 0 is subnormal (m/8 * 2^-6);
 * S.1111.111 is NaN. */
double or_e4m3_to_f64(uint8_t c)
{
    int s = c >> 7, ef = (c >> 3) & 15, mf = c & 7;
    double v;
    if (ef == 15 && mf == 7) return NAN;
    if (ef == 0) v = ldexp((double)mf, -9);
    else v = ldexp(1.0 + mf / 8.0, ef - 7);
    return s ? -v : v;
}

/* binary32 -> E4M3, round to nearest even, saturating to +-448 (satfinite). */
uint8_t or_f32_to_e4m3(float xf)
{
    double x = (double)xf;
    if (isnan(x)) return 0x7F;
    uint8_t s = signbit(x) ? 0x80 : 0;
    double a = fabs(x);
    if (a == 0.0) return s;
    int e = ilogb(a);
    if (isinf(a) || e > 8) return s | 0x7E;           /* >= 512: saturate to 448 */
    if (e < -6) {                                     /* subnormal range: quantum 2^-9 */
        double r = nearbyint(ldexp(a, 9));            /* 0..8 */
        if (r >= 8.0) return s | 0x08;                /* rounds up to the min normal 2^-6 */
        return s | (uint8_t)r;
    }
    double r = nearbyint((ldexp(a, -e) - 1.0) * 8.0); /* mantissa steps 0..8 */
    if (r >= 8.0) { r = 0.0; e += 1; }
    if (e > 8 || (e == 8 && r > 6.0)) return s | 0x7E; /* above 448 -> 448 */
    return s | (uint8_t)(((e + 7) << 3) | (int)r);
}

/* E2M1 magnitudes by code 0..7 (OCP MX v1.0): 0, 0.5, 1, 1.5, 2, 3, 4, 6. */
static double e2m1_mag(int code)
{
    int ef = (code >> 1) & 3, mf = code & 1;
    if (ef == 0) return mf * 0.5;                     /* subnormal: m * 2^-1 */
    return ldexp(1.0 + mf * 0.5, ef - 1);             /* bias 1 */
}

double or_e2m1_to_f64(uint8_t nib)
{
    double v = e2m1_mag(nib & 7);
    return (nib & 8) ? -v : v;
}

/* binary32 -> E2M1 nibble: nearest representable magnitude, ties to the even code,
 * saturating to 6; the sign bit follows the input (so -0.1 -> -0). */
uint8_t or_f32_to_e2m1(float xf)
{
    double x = (double)xf;
    uint8_t s = signbit(x) ? 8 : 0;
    double a = fabs(x);
    if (isnan(x)) return 7;
    int best = 0;
    double bestd = fabs(a - e2m1_mag(0));
    for (int c = 1; c < 8; c++) {
        double dlt = fabs(a - e2m1_mag(c));
        if (dlt < bestd || (dlt == bestd && (c & 1) == 0)) { best = c; bestd = dlt; }
    }
    if (a > 6.0) best = 7;
    return s | (uint8_t)best;
}

/* E8M0 shared scale: 2^(code - 127); code 255 is NaN. */
double or_e8m0_to_f64(uint8_t c)
{
    if (c == 255) return NAN;
    return ldexp(1.0, (int)c - 127);
}

/* ------------------------------------------------------------------------------------ */
/* storage formats of one KV row / one index vector                                       */

/* KV store descriptor: fmt 0 = bf16 rows of d values; fmt 2 = split row: d/2 E4M3 codes
 * (non-RoPE dims) times a per-row fp32 scale, then d/2 bf16 RoPE dims.  Row t of sequence
 * b lives at slot (b * cap + t % cap): cap == L stores every row, cap < L is a ring. */
typedef struct {
    int fmt;
    const void *data;
    const float *scale;
    const uint16_t *rope;
    long cap;
} or_kv;

static void kv_row(const or_kv *kv, int d, long b, long t, double *out)
{
    long slot = b * kv->cap + (t % kv->cap);
    if (kv->fmt == 0) {
        const uint16_t *r = (const uint16_t *)kv->data + slot * d;
        for (int c = 0; c < d; c++) out[c] = or_bf16_to_f64(r[c]);
    } else {
        int h = d / 2;
        const uint8_t *n = (const uint8_t *)kv->data + slot * h;
        double sc = (double)kv->scale[slot];
        const uint16_t *r = kv->rope + slot * h;
        for (int c = 0; c < h; c++) out[c] = or_e4m3_to_f64(n[c]) * sc;
        for (int c = 0; c < h; c++) out[h + c] = or_bf16_to_f64(r[c]);
    }
}

/* Index vectors: fmt 0 = bf16; fmt 3 = MXFP4 (dI/2 packed bytes, element 2j in the low
 * nibble of byte j, then one E8M0 scale per 32 elements). */
static void index_vec(int fmt, const void *data, const uint8_t *sf, long row, int dI, double *out)
{
    if (fmt == 0) {
        const uint16_t *r = (const uint16_t *)data + row * dI;
        for (int c = 0; c < dI; c++) out[c] = or_bf16_to_f64(r[c]);
    } else {
        const uint8_t *p = (const uint8_t *)data + row * (dI / 2);
        const uint8_t *s = sf + row * (dI / 32);
        for (int c = 0; c < dI; c++) {
            uint8_t nib = (c & 1) ? (p[c / 2] >> 4) : (p[c / 2] & 15);
            out[c] = or_e2m1_to_f64(nib) * or_e8m0_to_f64(s[c / 32]);
        }
    }
}

/* ------------------------------------------------------------------------------------ */
/* a1 / a2: softmax-gated pooling compressor                                             */

/* Entry i of a sequence pools `span` consecutive raw tokens starting at first(i):
 *   CSA (overlap = 1): span = 2m, first = m(i-1): the previous window's last m tokens
 *                      (C^b) then the current m tokens (C^a)          [CSDN §1.1 工程细节]
 *   HCA (overlap = 0): span = m,  first = m i                          [Tripbot §3.2]
 * With slot j holding token t_j = first + j (slots with t_j outside [0, L) are dropped),
 *   c_i[ch] = sum_j softmax_j( g[t_j, ch] + bias[j] ) * x[t_j, ch]      [Tripbot §3.1]
 * Output: entries e0..e1-1, fp64 [B, e1-e0, d]. */
void or_compress(const uint16_t *x, const uint16_t *g, const float *bias, int B, long L,
                 int d, int m, int overlap, long e0, long e1, double *out)
{
    int span = overlap ? 2 * m : m;
    long n = e1 - e0;
#pragma omp parallel for collapse(2) schedule(static)
    for (long b = 0; b < B; b++) {
        for (long i = e0; i < e1; i++) {
            long first = overlap ? (long)m * (i - 1) : (long)m * i;
            double *o = out + (b * n + (i - e0)) * d;
            for (int ch = 0; ch < d; ch++) {
                double zmax = -INFINITY;
                for (int j = 0; j < span; j++) {
                    long t = first + j;
                    if (t < 0 || t >= L) continue;
                    double z = or_bf16_to_f64(g[(b * L + t) * d + ch]) + (double)bias[j];
                    if (z > zmax) zmax = z;
                }
                double den = 0.0, num = 0.0;
                for (int j = 0; j < span; j++) {
                    long t = first + j;
                    if (t < 0 || t >= L) continue;
                    double z = or_bf16_to_f64(g[(b * L + t) * d + ch]) + (double)bias[j];
                    double e = exp(z - zmax);
                    den += e;
                    num += e * or_bf16_to_f64(x[(b * L + t) * d + ch]);
                }
                o[ch] = (den > 0.0) ? num / den : 0.0;
            }
        }
    }
}

/* ------------------------------------------------------------------------------------ */
/* visibility (causal at entry granularity)                                              */

/* Number of entries of ratio m visible to a query at position p: entry i is complete,
 * hence visible, when its last token m i + m - 1 <= p, i.e. i < floor((p + 1) / m). */
long or_num_visible(long p, int m, long n_entries)
{
    if (p < 0) return 0;
    long v = (p + 1) / m;
    return v < n_entries ? v : n_entries;
}

/* ------------------------------------------------------------------------------------ */
/* a4: lightning indexer                                                                   */

/* s[b,t,i] = sum_h w[b,t,h] * max(0, q_I[b,t,h,:] . k_I[b,i,:])  for visible i, else -inf.
 * A multi-head dot-product scorer over all compressed entries            [Tripbot §3.1];
 * operands bf16 or MXFP4 (fmt 0 / 3)                         [CSDN §1.4, Austery infra].
 * Output fp64 [B, Tq, Nc]. */
void or_index_scores(int fmt, const void *qI, const uint8_t *qI_sf, const float *w,
                     const void *kI, const uint8_t *kI_sf, int B, int Tq, int HI, int dI,
                     long Nc, const int *q_pos, int m, double *s)
{
#pragma omp parallel
    {
        double *q = (double *)malloc(sizeof(double) * HI * dI);
        double *k = (double *)malloc(sizeof(double) * dI);
#pragma omp for collapse(2) schedule(static)
        for (long b = 0; b < B; b++) {
            for (long t = 0; t < Tq; t++) {
                long row = b * Tq + t;
                for (int h = 0; h < HI; h++) index_vec(fmt, qI, qI_sf, row * HI + h, dI, q + h * dI);
                long nvis = or_num_visible(q_pos[row], m, Nc);
                double *srow = s + row * Nc;
                for (long i = 0; i < Nc; i++) {
                    if (i >= nvis) { srow[i] = -INFINITY; continue; }
                    index_vec(fmt, kI, kI_sf, b * Nc + i, dI, k);
                    double acc = 0.0;
                    for (int h = 0; h < HI; h++) {
                        double dot = 0.0;
                        for (int c = 0; c < dI; c++) dot += q[h * dI + c] * k[c];
                        acc += (double)w[row * HI + h] * (dot > 0.0 ? dot : 0.0);
                    }
                    srow[i] = acc;
                }
            }
        }
        free(q);
        free(k);
    }
}

/* Index scores quantised from fp32 to BF16 before selection       [CSDN §1.4]:
 * in place, each value replaced by its nearest bf16 (ties to even). */
void or_round_bf16(double *s, long n)
{
    for (long i = 0; i < n; i++) s[i] = or_bf16_to_f64(or_f64_to_bf16(s[i]));
}

/* ------------------------------------------------------------------------------------ */
/* a5: per-query top-k                                                                     */

typedef struct { double s; long i; } scored;

static int by_score_desc(const void *pa, const void *pb)
{
    const scored *a = (const scored *)pa, *b = (const scored *)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->i < b->i) ? -1 : (a->i > b->i);     /* equal scores: lower index first */
}

static int by_index(const void *pa, const void *pb)
{
    long a = *(const int *)pa, b = *(const int *)pb;
    return (a > b) - (a < b);
}

/* The k highest-scoring visible entries of each query row             [Tripbot §3.1];
 * ties go to the lower index; returned in ascending index order, padded with -1 when
 * fewer than k entries are visible.  idx: int32 [B, Tq, k]. */
void or_topk(const double *s, int B, int Tq, long Nc, const int *q_pos, int m, int k, int *idx)
{
#pragma omp parallel
    {
        scored *buf = (scored *)malloc(sizeof(scored) * (Nc > 0 ? Nc : 1));
#pragma omp for schedule(dynamic)
        for (long row = 0; row < (long)B * Tq; row++) {
            long nvis = or_num_visible(q_pos[row], m, Nc);
            for (long i = 0; i < nvis; i++) { buf[i].s = s[row * Nc + i]; buf[i].i = i; }
            qsort(buf, nvis, sizeof(scored), by_score_desc);
            long take = nvis < k ? nvis : k;
            int *out = idx + row * k;
            for (long j = 0; j < take; j++) out[j] = (int)buf[j].i;
            qsort(out, take, sizeof(int), by_index);
            for (long j = take; j < k; j++) out[j] = -1;
        }
        free(buf);
    }
}

/* ------------------------------------------------------------------------------------ */
/* a6 / a7: attention over compressed entries plus the raw sliding window                 */

/* Joint softmax of one query head over n rows (each row is key and value), two passes:
 *   z_j = scale * q . v_j;  o = sum_j exp(z_j - M) v_j / D;  lse = M + log D
 * with D = sum_j exp(z_j - M) (+ exp(sink - M) when a sink logit is given: the sink takes
 * probability mass but contributes no value, so the weights may sum to less than 1
 * [Tripbot §3.3]).  No rows and no sink: o = 0, lse = -inf. */
static void attend(const double *q, int d, double *const *rows, long n, double scale,
                   int has_sink, double sink, double *z, double *o, double *lse)
{
    double zmax = has_sink ? sink : -INFINITY;
    for (long j = 0; j < n; j++) {
        double dot = 0.0;
        for (int c = 0; c < d; c++) dot += q[c] * rows[j][c];
        z[j] = scale * dot;
        if (z[j] > zmax) zmax = z[j];
    }
    for (int c = 0; c < d; c++) o[c] = 0.0;
    if (n == 0 && !has_sink) { *lse = -INFINITY; return; }
    double den = has_sink ? exp(sink - zmax) : 0.0;
    for (long j = 0; j < n; j++) den += exp(z[j] - zmax);
    for (long j = 0; j < n; j++) {
        double p = exp(z[j] - zmax) / den;
        for (int c = 0; c < d; c++) o[c] += p * rows[j][c];
    }
    *lse = zmax + log(den);
}

/* Window rows of a query at position p: raw tokens max(0, p - W + 1) .. p   [Tripbot §3.3] */
static long window_rows(const or_kv *raw, int d, long b, long p, int W, double *store, double **rows)
{
    long lo = p - W + 1;
    if (lo < 0) lo = 0;
    long n = 0;
    for (long t = lo; t <= p; t++, n++) {
        kv_row(raw, d, b, t, store + n * d);
        rows[n] = store + n * d;
    }
    return n;
}

/* CSA attention (a6): for query (b, t) at position p, the rows are the selected compressed
 * entries idx[b,t,:] (entries -1 skipped) followed by the window rows; one joint softmax per
 * head, scale applied to q.v                              [Tripbot §3.1 step 2, §3.3].
 * q: bf16 [B, Tq, H, d]; o: fp64 [B, Tq, H, d]; lse: fp64 [B, Tq, H]. */
void or_csa_attn(const uint16_t *q, int B, int Tq, int H, int d,
                 int kvc_fmt, const void *kvc, const float *kvc_scale, const uint16_t *kvc_rope,
                 long kvc_cap, const int *idx, int k,
                 int raw_fmt, const void *raw, const float *raw_scale, const uint16_t *raw_rope,
                 long raw_cap, int W, const int *q_pos, double scale, const float *sink,
                 double *o, double *lse)
{
    or_kv C = {kvc_fmt, kvc, kvc_scale, kvc_rope, kvc_cap};
    or_kv R = {raw_fmt, raw, raw_scale, raw_rope, raw_cap};
    long maxn = (long)k + (W > 0 ? W : 0);
#pragma omp parallel
    {
        double *store = (double *)malloc(sizeof(double) * (maxn + 1) * d);
        double **rows = (double **)malloc(sizeof(double *) * (maxn + 1));
        double *z = (double *)malloc(sizeof(double) * (maxn + 1));
        double *qh = (double *)malloc(sizeof(double) * d);
#pragma omp for collapse(2) schedule(dynamic)
        for (long b = 0; b < B; b++) {
            for (long t = 0; t < Tq; t++) {
                long row = b * Tq + t, n = 0;
                for (int j = 0; j < k; j++) {
                    int e = idx[row * k + j];
                    if (e < 0) continue;
                    kv_row(&C, d, b, e, store + n * d);
                    rows[n] = store + n * d;
                    n++;
                }
                n += window_rows(&R, d, b, q_pos[row], W, store + n * d, rows + n);
                for (int h = 0; h < H; h++) {
                    for (int c = 0; c < d; c++) qh[c] = or_bf16_to_f64(q[(row * H + h) * d + c]);
                    attend(qh, d, rows, n, scale, sink != NULL, sink ? (double)sink[h] : 0.0, z,
                           o + (row * H + h) * d, lse + row * H + h);
                }
            }
        }
        free(store); free(rows); free(z); free(qh);
    }
}

/* HCA attention (a7): rows are every HCA entry visible to the query (entry i of ratio m'
 * once its last token m'(i+1)-1 <= p), then the window rows; dense, no selection
 * [Tripbot §3.2, §3.3; CSDN §1.2]. */
void or_hca_attn(const uint16_t *q, int B, int Tq, int H, int d,
                 int kvh_fmt, const void *kvh, const float *kvh_scale, const uint16_t *kvh_rope,
                 long kvh_cap, long Nh, int mh,
                 int raw_fmt, const void *raw, const float *raw_scale, const uint16_t *raw_rope,
                 long raw_cap, int W, const int *q_pos, double scale, const float *sink,
                 double *o, double *lse)
{
    or_kv C = {kvh_fmt, kvh, kvh_scale, kvh_rope, kvh_cap};
    or_kv R = {raw_fmt, raw, raw_scale, raw_rope, raw_cap};
    long maxn = Nh + (W > 0 ? W : 0);
#pragma omp parallel
    {
        double *store = (double *)malloc(sizeof(double) * (maxn + 1) * d);
        double **rows = (double **)malloc(sizeof(double *) * (maxn + 1));
        double *z = (double *)malloc(sizeof(double) * (maxn + 1));
        double *qh = (double *)malloc(sizeof(double) * d);
#pragma omp for collapse(2) schedule(dynamic)
        for (long b = 0; b < B; b++) {
            for (long t = 0; t < Tq; t++) {
                long row = b * Tq + t, n = 0;
                long nvis = or_num_visible(q_pos[row], mh, Nh);
                for (long i = 0; i < nvis; i++, n++) {
                    kv_row(&C, d, b, i, store + n * d);
                    rows[n] = store + n * d;
                }
                n += window_rows(&R, d, b, q_pos[row], W, store + n * d, rows + n);
                for (int h = 0; h < H; h++) {
                    for (int c = 0; c < d; c++) qh[c] = or_bf16_to_f64(q[(row * H + h) * d + c]);
                    attend(qh, d, rows, n, scale, sink != NULL, sink ? (double)sink[h] : 0.0, z,
                           o + (row * H + h) * d, lse + row * H + h);
                }
            }
        }
        free(store); free(rows); free(z); free(qh);
    }
}

/* ------------------------------------------------------------------------------------ */
/* RMSNorm of queries and compressed entries                                              */

/* The attention normalises its queries and its KV entries with RMSNorm, which is why no
 * separate QK-Norm is needed                                            [Tripbot §5].
 * Per row of d values: out_c = x_c / sqrt(mean_c(x_c^2) + eps) * gamma_c (gamma NULL: 1).
 * x, out: fp64 [rows, d] (out may alias x). */
void or_rmsnorm(const double *x, long rows, int d, const float *gamma, double eps, double *out)
{
#pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; r++) {
        const double *xr = x + r * d;
        double ss = 0.0;
        for (int c = 0; c < d; c++) ss += xr[c] * xr[c];
        double inv = 1.0 / sqrt(ss / d + eps);
        double *o = out + r * d;
        for (int c = 0; c < d; c++) o[c] = xr[c] * inv * (gamma ? (double)gamma[c] : 1.0);
    }
}

/* ------------------------------------------------------------------------------------ */
/* a3: cache quantisers                                                                   */

/* Split KV row: RoPE dims (the last d/2) stay bf16; the other d/2 dims are stored as E4M3
 * with one fp32 scale per row                                               [CSDN §1.4].
 * scale = amax / 448 in fp32 (1 when amax = 0); code = E4M3_rne_sat(x / scale) with the
 * quotient rounded to fp32.  kv: bf16 [rows, d]. */
void or_quant_kv_fp8(const uint16_t *kv, long rows, int d, uint8_t *nope, float *scale, uint16_t *rope)
{
    int h = d / 2;
#pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; r++) {
        const uint16_t *x = kv + r * d;
        float amax = 0.0f;
        for (int c = 0; c < h; c++) {
            float v = fabsf((float)or_bf16_to_f64(x[c]));
            if (v > amax) amax = v;
        }
        float sc = (amax > 0.0f) ? amax / 448.0f : 1.0f;
        scale[r] = sc;
        for (int c = 0; c < h; c++) {
            float v = (float)or_bf16_to_f64(x[c]);
            float qv = v / sc;
            nope[r * h + c] = or_f32_to_e4m3(qv);
        }
        for (int c = 0; c < h; c++) rope[r * h + c] = x[h + c];
    }
}

/* MXFP4 (OCP MX v1.0, block 32): per block, X = 2^(floor(log2 amax) - 2) stored as E8M0
 * (biased by 127, clamped to 0..254; amax = 0 stores 127); element = E2M1_rne_sat(x / X).
 * Indexer QK path in FP4 [CSDN §1.4; Austery infra].  x: bf16 [rows, cols], cols % 32 == 0;
 * packed: [rows, cols/2] (element 2j in the low nibble); sf: [rows, cols/32]. */
void or_quant_mxfp4(const uint16_t *x, long rows, int cols, uint8_t *packed, uint8_t *sf)
{
    int nb = cols / 32;
#pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; r++) {
        for (int blk = 0; blk < nb; blk++) {
            const uint16_t *v = x + r * cols + blk * 32;
            double amax = 0.0;
            for (int c = 0; c < 32; c++) {
                double a = fabs(or_bf16_to_f64(v[c]));
                if (a > amax) amax = a;
            }
            int e = (amax > 0.0) ? ilogb(amax) - 2 : 0;
            int code = e + 127;
            if (code < 0) code = 0;
            if (code > 254) code = 254;
            sf[r * nb + blk] = (uint8_t)code;
            double X = ldexp(1.0, code - 127);
            for (int c = 0; c < 32; c += 2) {
                uint8_t lo = or_f32_to_e2m1((float)(or_bf16_to_f64(v[c]) / X));
                uint8_t hi = or_f32_to_e2m1((float)(or_bf16_to_f64(v[c + 1]) / X));
                packed[r * (cols / 2) + blk * 16 + c / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
}
