/*
 * dualqk_oracle.c -- plain, slow, fp64 CPU oracle of the Dual-QK decode path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file: only the tests, the package smoke check and the CPU
 * baseline leg of the benchmark use it.  It shares no source with the CUDA
 * library (no headers, helpers, tables or constants) and knows nothing of the
 * paged cache layout: it works on plain per-token arrays.
 *
 * What it computes, step by step, in the order of the method:
 *
 *  (1) key transform    k' = T_K k            "partial key whitening"
 *  (2) INT2 quantizer   per token, per group of 32 channels, asymmetric
 *                       (scale, min) in fp16, round-half-to-even codes 0..3;
 *                       key channel 0 kept in BF16 ("channel-0 protection")
 *  (3) query transform  q' = T_Q q, T_Q = T_K^{-T}, so q'.k' = q.k
 *  (4) channel pruning  keep channel 0 plus the largest-|q'| channels
 *                       (ties toward the lower index), 40 % sparsity
 *  (5) attention        softmax(q'.k^'/sqrt(d)) over the dequantized cache,
 *                       times the dequantized values
 *
 * Sources (page title, section):
 *  - "How does Dual-QK compress KV caches to 2-bit while keeping accuracy at
 *    128K context?", sections "Why the cache becomes a bottleneck" (rotation
 *    must preserve query-key dot products; query-channel pruning cuts key
 *    reads), "Paired transforms instead of shared rotation" (partial key
 *    whitening, query-aligned basis, non-orthogonal pair, channel-0
 *    protection), "Throughput on SGLang" (2 bits per stored value, 40 % of
 *    key channels removed from reads).
 *  - "Dual-QK: Sharp Queries and Flat Keys for Prunable 2-bit KV Caches",
 *    abstract (same facts, INT2, 40 % query-channel sparsity).
 * The pages give no formulas.  Where they are silent the oracle takes the
 * fixed readings of the build specification, each marked READING below.
 *
 * Arithmetic contract shared with any implementation that wants bit-exact
 * codes (READING): transform outputs are fp32 values obtained by summing the
 * exact fp64 products T[c][i]*x[i] sequentially in ascending i in fp64 and
 * rounding once; all quantizer arithmetic is fp64 with single roundings to
 * fp16/bf16 written out below from the IEEE 754 formats.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_GROUP 32

/* ------------------------------------------------------------------------- */
/* IEEE 754 binary16 and bfloat16 rounding, written from the format          */
/* definitions: p significant bits, minimum normal exponent emin, subnormal  */
/* spacing 2^(emin-p+1); round to nearest, ties to even (nearbyint in the    */
/* default rounding mode).                                                   */
/* ------------------------------------------------------------------------- */

/* binary16: 11 significant bits, emin = -14, max finite 65504.
 * READING: values beyond the finite range saturate to +-65504 (the method
 * needs finite scales). NaN maps to the canonical quiet NaN. */
uint16_t oracle_f64_to_f16(double x)
{
    if (isnan(x)) return 0x7E00u;
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    double a = fabs(x);
    if (a >= 65504.0) return (uint16_t)(sign | 0x7BFFu);
    if (a == 0.0) return sign;
    int e;
    (void)frexp(a, &e);             /* a = m 2^e, m in [0.5, 1) */
    int E = e - 1;                  /* 2^E <= a < 2^(E+1)        */
    if (E < -14) {                  /* subnormal: spacing 2^-24   */
        double r = nearbyint(ldexp(a, 24));
        return (uint16_t)(sign | (uint16_t)r);   /* r == 1024 is the min normal */
    }
    double r = nearbyint(ldexp(a, 10 - E));       /* in [1024, 2048] */
    int biased = E + 15;
    if (r == 2048.0) { r = 1024.0; biased += 1; }
    if (biased >= 31) return (uint16_t)(sign | 0x7BFFu);
    return (uint16_t)(sign | (uint16_t)(biased << 10) | (uint16_t)((int)r - 1024));
}

double oracle_f16_to_f64(uint16_t h)
{
    int E = (h >> 10) & 31, M = h & 1023;
    double s = (h & 0x8000u) ? -1.0 : 1.0;
    if (E == 0) return s * ldexp((double)M, -24);
    if (E == 31) return M ? NAN : s * INFINITY;
    return s * ldexp((double)(1024 + M), E - 25);
}

/* bfloat16: 8 significant bits, emin = -126; the value is stored as the top
 * half of the binary32 encoding of the rounded number. */
uint16_t oracle_f32_to_bf16(float xf)
{
    double x = (double)xf;
    if (isnan(x)) return 0x7FC0u;
    double a = fabs(x), r;
    if (a == 0.0 || isinf(a)) {
        r = a;
    } else {
        int e;
        (void)frexp(a, &e);
        int E = e - 1;
        if (E < -126) r = ldexp(nearbyint(ldexp(a, 133)), -133);
        else r = ldexp(nearbyint(ldexp(a, 7 - E)), E - 7);
    }
    float rf = (float)(signbit(x) ? -r : r);      /* exact: r has <= 8 bits */
    uint32_t bits;
    memcpy(&bits, &rf, 4);
    return (uint16_t)(bits >> 16);
}

double oracle_bf16_to_f64(uint16_t b)
{
    uint32_t bits = (uint32_t)b << 16;
    float f;
    memcpy(&f, &bits, 4);
    return (double)f;
}

/* ------------------------------------------------------------------------- */
/* (1)/(3) transforms                                                         */
/* ------------------------------------------------------------------------- */

/* y[c] = fp32( sum_{i=0}^{d-1} T[c][i] * x[i] ), fp64 running sum in
 * ascending i.  Products of two fp32 values are exact in fp64, so this is one
 * well-defined number per channel (READING: the contract above). */
void oracle_transform_f32(int d, const float *T, const float *x, float *y)
{
    for (int c = 0; c < d; ++c) {
        double s = 0.0;
        for (int i = 0; i < d; ++i) s += (double)T[(size_t)c * d + i] * (double)x[i];
        y[c] = (float)s;
    }
}

/* Same map kept in fp64 end to end (quantization-off mode). */
void oracle_transform_f64(int d, const double *T, const double *x, double *y)
{
    for (int c = 0; c < d; ++c) {
        double s = 0.0;
        for (int i = 0; i < d; ++i) s += T[(size_t)c * d + i] * x[i];
        y[c] = s;
    }
}

/* ------------------------------------------------------------------------- */
/* (2) INT2 quantizer of one token vector                                     */
/* ------------------------------------------------------------------------- */

/* x: d fp32 values (already transformed for keys).  protect_ch0: channel 0
 * is stored in BF16, left out of group 0's min/max, and its code slot is 0.
 * Per group g (channels gs*g .. gs*g + gs-1; gs = 32, or d for one group per
 * token):
 *   mn, mx      = min / max over the group (fp32 values; a zero is +0)
 *   scale_h     = fp16( (mx - mn) / 3 )          (fp64 arithmetic)
 *   min_h       = fp16( mn )
 *   code_c      = 0 if scale_h == 0, else clamp(rne((x_c - min_h)/scale_h), 0, 3)
 * READING: fixed groups aligned at channel 0; fp16 for scale and min; round
 * half to even; a zero scale gives code 0 (dequantizes to min). */
void oracle_quantize_vec_g(int d, int gs, const float *x, int protect_ch0,
                           uint8_t *codes, uint16_t *scale, uint16_t *minv, uint16_t *ch0)
{
    int ng = d / gs;
    for (int g = 0; g < ng; ++g) {
        int lo = g * gs, hi = lo + gs;
        int first = (g == 0 && protect_ch0) ? 1 : 0;
        double mn = INFINITY, mx = -INFINITY;
        for (int c = lo + first; c < hi; ++c) {
            double v = (double)x[c] + 0.0;      /* READING: -0 and +0 are the value 0 */
            if (v < mn) mn = v;
            if (v > mx) mx = v;
        }
        uint16_t sh = oracle_f64_to_f16((mx - mn) / 3.0);
        uint16_t mh = oracle_f64_to_f16(mn);
        scale[g] = sh;
        minv[g] = mh;
        double s = oracle_f16_to_f64(sh), m = oracle_f16_to_f64(mh);
        for (int c = lo; c < hi; ++c) {
            int code = 0;
            if (!(c == 0 && protect_ch0) && s != 0.0) {
                double r = nearbyint(((double)x[c] - m) / s);
                code = r < 0.0 ? 0 : (r > 3.0 ? 3 : (int)r);
            }
            codes[c] = (uint8_t)code;
        }
    }
    if (ch0) *ch0 = protect_ch0 ? oracle_f32_to_bf16(x[0]) : 0;
}

void oracle_quantize_vec(int d, const float *x, int protect_ch0,
                         uint8_t *codes, uint16_t *scale, uint16_t *minv, uint16_t *ch0)
{
    oracle_quantize_vec_g(d, OR_GROUP, x, protect_ch0, codes, scale, minv, ch0);
}

/* Dequantized channel value (fp64, exact from the stored fields). */
static double dequant(int c, int gs, int protect_ch0, const uint8_t *codes, const uint16_t *scale,
                      const uint16_t *minv, uint16_t ch0)
{
    if (c == 0 && protect_ch0) return oracle_bf16_to_f64(ch0);
    int g = c / gs;
    return oracle_f16_to_f64(minv[g]) + (double)codes[c] * oracle_f16_to_f64(scale[g]);
}

/* ------------------------------------------------------------------------- */
/* append: transform + quantize rows                                          */
/* ------------------------------------------------------------------------- */

/* k, v: [n][hkv][d] fp32 (model values, RoPE applied by the caller).
 * t_k: [hkv][d][d].  Outputs (plain arrays, token-major):
 *   kcodes/vcodes [n][hkv][d], kscale/kmin/vscale/vmin [n][hkv][d/32],
 *   kch0/vch0 [n][hkv]  (vch0 only meaningful when v_ch0 != 0).
 * Keys: channel 0 always protected.  Values: no transform; channel 0
 * protected only when v_ch0 != 0 (READING: the pages name channel-0
 * protection beside the key-side RoPE, so keys by default). */
int oracle_append_g(int d, int gs, int hkv, int v_ch0, const float *t_k,
                    const float *k, const float *v, long long n,
                    uint8_t *kcodes, uint16_t *kscale, uint16_t *kmin, uint16_t *kch0,
                    uint8_t *vcodes, uint16_t *vscale, uint16_t *vmin, uint16_t *vch0)
{
    if (gs <= 0 || d % gs || d <= 0 || hkv <= 0 || n < 0) return 1;
    int ng = d / gs;
    float *kp = (float *)malloc(sizeof(float) * (size_t)d);
    if (!kp) return 2;
    for (long long t = 0; t < n; ++t) {
        for (int j = 0; j < hkv; ++j) {
            size_t row = (size_t)(t * hkv + j);
            oracle_transform_f32(d, t_k + (size_t)j * d * d, k + row * d, kp);
            oracle_quantize_vec_g(d, gs, kp, 1, kcodes + row * d, kscale + row * ng, kmin + row * ng,
                                  kch0 + row);
            oracle_quantize_vec_g(d, gs, v + row * d, v_ch0, vcodes + row * d, vscale + row * ng,
                                  vmin + row * ng, vch0 + row);
        }
    }
    free(kp);
    return 0;
}

int oracle_append(int d, int hkv, int v_ch0, const float *t_k,
                  const float *k, const float *v, long long n,
                  uint8_t *kcodes, uint16_t *kscale, uint16_t *kmin, uint16_t *kch0,
                  uint8_t *vcodes, uint16_t *vscale, uint16_t *vmin, uint16_t *vch0)
{
    return oracle_append_g(d, OR_GROUP, hkv, v_ch0, t_k, k, v, n, kcodes, kscale, kmin, kch0, vcodes, vscale,
                           vmin, vch0);
}

/* ------------------------------------------------------------------------- */
/* (4) channel selection                                                      */
/* ------------------------------------------------------------------------- */

/* Number of kept channels, channel 0 included (READING: floor of the pruned
 * count, channel 0 always kept and counted). */
int oracle_n_keep(int d, int pct)
{
    return d - (pct * d) / 100;
}

/* Keep channel 0 and the (n_keep-1) channels of 1..d-1 with the largest
 * |q'_c|; equal magnitudes are ordered by ascending channel index.  Plain
 * insertion sort on (-|q'|, c); result written in ascending channel order. */
void oracle_select(int d, const double *absq, int n_keep, int16_t *sel)
{
    int *ord = (int *)malloc(sizeof(int) * (size_t)d);
    int m = 0;
    for (int c = 1; c < d; ++c) {
        int pos = m;
        while (pos > 0) {
            int o = ord[pos - 1];
            int before = absq[o] > absq[c] || (absq[o] == absq[c] && o < c);
            if (before) break;
            ord[pos] = ord[pos - 1];
            --pos;
        }
        ord[pos] = c;
        ++m;
    }
    char *keep = (char *)calloc((size_t)d, 1);
    keep[0] = 1;
    for (int r = 0; r < n_keep - 1 && r < m; ++r) keep[ord[r]] = 1;
    int w = 0;
    for (int c = 0; c < d; ++c)
        if (keep[c]) sel[w++] = (int16_t)c;
    free(keep);
    free(ord);
}

/* q' (fp32 contract) and the selected channels of one query head. */
void oracle_qprep(int d, const float *t_q_head, const float *q, int pct, float *qp, int16_t *sel)
{
    oracle_transform_f32(d, t_q_head, q, qp);
    double *a = (double *)malloc(sizeof(double) * (size_t)d);
    for (int c = 0; c < d; ++c) a[c] = fabs((double)qp[c]);
    oracle_select(d, a, oracle_n_keep(d, pct), sel);
    free(a);
}

/* ------------------------------------------------------------------------- */
/* (5) attention over the quantized cache of one sequence                      */
/* ------------------------------------------------------------------------- */

typedef struct {
    int d, gs, hq, hkv, v_ch0, pct, L;
    const uint8_t *kcodes; const uint16_t *kscale, *kmin, *kch0;
    const uint8_t *vcodes; const uint16_t *vscale, *vmin, *vch0;
    const float *q, *t_q;
    double *out; int16_t *sel; float *qprime;
    int next;                      /* next kv head to take (guarded by mu) */
    pthread_mutex_t mu;
} seq_job;

/* One query head h: s_t = (1/sqrt d) sum_{c in S} q'_c k^'_{t,c};
 * p = softmax(s) (max-subtracted, fp64, one pass over all L tokens);
 * o = sum_t p_t v^_t. */
static void decode_head(seq_job *J, int h, double *s, double *qd, char *in_s, int16_t *sel)
{
    int d = J->d, gs = J->gs, ng = d / gs, G = J->hq / J->hkv, j = h / G, L = J->L;
    int nk = oracle_n_keep(d, J->pct);
    float *qp = (float *)malloc(sizeof(float) * (size_t)d);
    oracle_qprep(d, J->t_q + (size_t)j * d * d, J->q + (size_t)h * d, J->pct, qp, sel);
    memset(in_s, 0, (size_t)d);
    for (int r = 0; r < nk; ++r) in_s[sel[r]] = 1;
    for (int c = 0; c < d; ++c) qd[c] = (double)qp[c];
    double inv_sqrt_d = 1.0 / sqrt((double)d), mx = -INFINITY;
    for (int t = 0; t < L; ++t) {
        size_t row = (size_t)t * J->hkv + j;
        double acc = 0.0;
        for (int c = 0; c < d; ++c) {
            if (!in_s[c]) continue;
            acc += qd[c] * dequant(c, gs, 1, J->kcodes + row * d, J->kscale + row * ng,
                                   J->kmin + row * ng, J->kch0[row]);
        }
        s[t] = acc * inv_sqrt_d;
        if (s[t] > mx) mx = s[t];
    }
    double den = 0.0;
    for (int t = 0; t < L; ++t) { s[t] = exp(s[t] - mx); den += s[t]; }
    double *o = J->out + (size_t)h * d;
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    for (int t = 0; t < L; ++t) {
        size_t row = (size_t)t * J->hkv + j;
        double p = s[t] / den;
        for (int c = 0; c < d; ++c)
            o[c] += p * dequant(c, gs, J->v_ch0, J->vcodes + row * d, J->vscale + row * ng,
                                J->vmin + row * ng, J->vch0[row]);
    }
    if (L == 0)
        for (int c = 0; c < d; ++c) o[c] = 0.0;       /* READING: empty context -> 0 */
    if (J->qprime) memcpy(J->qprime + (size_t)h * d, qp, sizeof(float) * (size_t)d);
    free(qp);
}

static void *seq_worker(void *arg)
{
    seq_job *J = (seq_job *)arg;
    int d = J->d, G = J->hq / J->hkv, nk = oracle_n_keep(d, J->pct);
    double *s = (double *)malloc(sizeof(double) * (size_t)(J->L > 0 ? J->L : 1));
    double *qd = (double *)malloc(sizeof(double) * (size_t)d);
    char *in_s = (char *)malloc((size_t)d);
    int16_t *tmp = (int16_t *)malloc(sizeof(int16_t) * (size_t)d);
    for (;;) {
        pthread_mutex_lock(&J->mu);
        int j = J->next++;
        pthread_mutex_unlock(&J->mu);
        if (j >= J->hkv) break;
        for (int h = j * G; h < (j + 1) * G; ++h) {
            decode_head(J, h, s, qd, in_s, tmp);
            if (J->sel) memcpy(J->sel + (size_t)h * nk, tmp, sizeof(int16_t) * (size_t)nk);
        }
    }
    free(s); free(qd); free(in_s); free(tmp);
    return NULL;
}

/* Decode one sequence of L tokens (plain arrays from oracle_append) for all
 * hq query heads; query head h reads kv head h / (hq/hkv).
 * out [hq][d] fp64; sel [hq][n_keep] (nullable); qprime [hq][d] (nullable).
 * Work is spread over up to `threads` POSIX threads, one kv head at a time. */
int oracle_decode_seq_g(int d, int gs, int hq, int hkv, int v_ch0, int pct, int L,
                        const uint8_t *kcodes, const uint16_t *kscale, const uint16_t *kmin,
                        const uint16_t *kch0, const uint8_t *vcodes, const uint16_t *vscale,
                        const uint16_t *vmin, const uint16_t *vch0,
                        const float *q, const float *t_q, double *out, int16_t *sel,
                        float *qprime, int threads)
{
    if (gs <= 0 || d % gs || hkv <= 0 || hq % hkv || pct < 0 || pct > 99 || L < 0) return 1;
    seq_job J = {d, gs, hq, hkv, v_ch0, pct, L, kcodes, kscale, kmin, kch0, vcodes, vscale, vmin,
                 vch0, q, t_q, out, sel, qprime, 0, PTHREAD_MUTEX_INITIALIZER};
    if (threads < 1) threads = 1;
    if (threads > hkv) threads = hkv;
    pthread_t *tid = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)threads);
    int started = 0;
    for (int i = 1; i < threads; ++i)
        if (pthread_create(&tid[started], NULL, seq_worker, &J) == 0) ++started;
    seq_worker(&J);
    for (int i = 0; i < started; ++i) pthread_join(tid[i], NULL);
    free(tid);
    pthread_mutex_destroy(&J.mu);
    return 0;
}

int oracle_decode_seq(int d, int hq, int hkv, int v_ch0, int pct, int L,
                      const uint8_t *kcodes, const uint16_t *kscale, const uint16_t *kmin,
                      const uint16_t *kch0, const uint8_t *vcodes, const uint16_t *vscale,
                      const uint16_t *vmin, const uint16_t *vch0,
                      const float *q, const float *t_q, double *out, int16_t *sel,
                      float *qprime, int threads)
{
    return oracle_decode_seq_g(d, OR_GROUP, hq, hkv, v_ch0, pct, L, kcodes, kscale, kmin, kch0, vcodes, vscale,
                               vmin, vch0, q, t_q, out, sel, qprime, threads);
}

/* ------------------------------------------------------------------------- */
/* quantization-off mode: everything fp64, no rounding anywhere              */
/* ------------------------------------------------------------------------- */

/* k, v: [L][hkv][d] fp64; q: [hq][d]; t_k, t_q: [hkv][d][d] fp64.
 * k' = T_K k and q' = T_Q q kept in fp64, channels selected by |q'| with the
 * same rule, s = q'.k'/sqrt(d) over the kept channels, softmax, o = p v.
 * scores (nullable) receives s for query head 0 ... hq-1, [hq][L]. */
int oracle_decode_dense(int d, int hq, int hkv, int pct, int L, const double *t_k,
                        const double *t_q, const double *k, const double *v, const double *q,
                        double *out, double *scores)
{
    if (hkv <= 0 || hq % hkv || L < 1) return 1;
    int G = hq / hkv, nk = oracle_n_keep(d, pct);
    double *kp = (double *)malloc(sizeof(double) * (size_t)L * hkv * d);
    for (int t = 0; t < L; ++t)
        for (int j = 0; j < hkv; ++j)
            oracle_transform_f64(d, t_k + (size_t)j * d * d, k + ((size_t)t * hkv + j) * d,
                                 kp + ((size_t)t * hkv + j) * d);
    double *qp = (double *)malloc(sizeof(double) * (size_t)d);
    double *a = (double *)malloc(sizeof(double) * (size_t)d);
    double *s = (double *)malloc(sizeof(double) * (size_t)L);
    int16_t *sel = (int16_t *)malloc(sizeof(int16_t) * (size_t)d);
    char *in_s = (char *)malloc((size_t)d);
    for (int h = 0; h < hq; ++h) {
        int j = h / G;
        oracle_transform_f64(d, t_q + (size_t)j * d * d, q + (size_t)h * d, qp);
        for (int c = 0; c < d; ++c) a[c] = fabs(qp[c]);
        oracle_select(d, a, nk, sel);
        memset(in_s, 0, (size_t)d);
        for (int r = 0; r < nk; ++r) in_s[sel[r]] = 1;
        double mx = -INFINITY;
        for (int t = 0; t < L; ++t) {
            const double *kr = kp + ((size_t)t * hkv + j) * d;
            double acc = 0.0;
            for (int c = 0; c < d; ++c)
                if (in_s[c]) acc += qp[c] * kr[c];
            s[t] = acc / sqrt((double)d);
            if (scores) scores[(size_t)h * L + t] = s[t];
            if (s[t] > mx) mx = s[t];
        }
        double den = 0.0;
        for (int t = 0; t < L; ++t) { s[t] = exp(s[t] - mx); den += s[t]; }
        double *o = out + (size_t)h * d;
        for (int c = 0; c < d; ++c) o[c] = 0.0;
        for (int t = 0; t < L; ++t) {
            const double *vr = v + ((size_t)t * hkv + j) * d;
            for (int c = 0; c < d; ++c) o[c] += (s[t] / den) * vr[c];
        }
    }
    free(kp); free(qp); free(a); free(s); free(sel); free(in_s);
    return 0;
}

/* ------------------------------------------------------------------------
 * (0) calibrated transform pair -- the step before the path ("Paired
 * transforms instead of shared rotation": partial key whitening combined
 * with a query-aligned basis, guided by calibrated query and key
 * statistics).  Written out from its definition:
 *
 *   C_K = K^T K / n + eps I,  eps = 1e-6 * trace(K^T K / n) / d
 *   P   = C_K^(alpha/2)                       (alpha = 1/2: partial whitening)
 *   C_Q = P (Q^T Q / m) P                     (second moment of P q)
 *   C_Q = U diag(mu) U^T, mu descending, each column of U signed so that its
 *         entry of largest magnitude (lowest index on ties) is positive
 *   T_K = U^T P^-1,  T_Q = U^T P              (so T_Q = T_K^-T, q'.k' = q.k)
 *
 * Matrix functions and eigenvectors come from a cyclic Jacobi
 * eigen-solver (plain rotations until the off-diagonal mass vanishes).
 * ---------------------------------------------------------------------- */

/* Eigen-decomposition of the symmetric d x d matrix A (destroyed): eigenvalues
 * in w[], eigenvectors as the columns of V (row-major V[i*d + k]). */
static void jacobi_eigen(int d, double *A, double *w, double *V)
{
    for (int i = 0; i < d; ++i)
        for (int k = 0; k < d; ++k) V[(size_t)i * d + k] = (i == k) ? 1.0 : 0.0;
    for (int sweep = 0; sweep < 100; ++sweep) {
        double off = 0.0, tot = 0.0;
        for (int i = 0; i < d; ++i)
            for (int k = 0; k < d; ++k) {
                const double a = A[(size_t)i * d + k] * A[(size_t)i * d + k];
                tot += a;
                if (i != k) off += a;
            }
        if (off <= 1e-30 * tot) break;
        for (int p = 0; p < d - 1; ++p)
            for (int q = p + 1; q < d; ++q) {
                const double apq = A[(size_t)p * d + q];
                if (apq == 0.0) continue;
                const double app = A[(size_t)p * d + p], aqq = A[(size_t)q * d + q];
                const double theta = (aqq - app) / (2.0 * apq);
                const double t = (theta >= 0.0 ? 1.0 : -1.0) / (fabs(theta) + sqrt(theta * theta + 1.0));
                const double c = 1.0 / sqrt(t * t + 1.0), s = t * c;
                for (int k = 0; k < d; ++k) {       /* A <- A J (columns p, q) */
                    const double akp = A[(size_t)k * d + p], akq = A[(size_t)k * d + q];
                    A[(size_t)k * d + p] = c * akp - s * akq;
                    A[(size_t)k * d + q] = s * akp + c * akq;
                }
                for (int k = 0; k < d; ++k) {       /* A <- J^T A (rows p, q) */
                    const double apk = A[(size_t)p * d + k], aqk = A[(size_t)q * d + k];
                    A[(size_t)p * d + k] = c * apk - s * aqk;
                    A[(size_t)q * d + k] = s * apk + c * aqk;
                }
                for (int k = 0; k < d; ++k) {       /* V <- V J */
                    const double vkp = V[(size_t)k * d + p], vkq = V[(size_t)k * d + q];
                    V[(size_t)k * d + p] = c * vkp - s * vkq;
                    V[(size_t)k * d + q] = s * vkp + c * vkq;
                }
            }
    }
    for (int i = 0; i < d; ++i) w[i] = A[(size_t)i * d + i];
}

/* B = V diag(f(w)) V^T with f(x) = x^e. */
static void sym_power(int d, const double *w, const double *V, double e, double *B)
{
    for (int i = 0; i < d; ++i)
        for (int k = 0; k < d; ++k) {
            double acc = 0.0;
            for (int j = 0; j < d; ++j) acc += V[(size_t)i * d + j] * pow(w[j], e) * V[(size_t)k * d + j];
            B[(size_t)i * d + k] = acc;
        }
}

int oracle_calibrate(int d, long long n, long long m, double alpha, const double *K, const double *Q,
                     double *t_k, double *t_q)
{
    if (d <= 0 || n <= 0 || m <= 0) return 1;
    const size_t dd = (size_t)d * d;
    double *A = (double *)calloc(dd, sizeof(double));
    double *V = (double *)malloc(dd * sizeof(double));
    double *w = (double *)malloc((size_t)d * sizeof(double));
    double *P = (double *)malloc(dd * sizeof(double));
    double *Pi = (double *)malloc(dd * sizeof(double));
    double *S = (double *)calloc(dd, sizeof(double));
    double *U = (double *)malloc(dd * sizeof(double));
    double *mu = (double *)malloc((size_t)d * sizeof(double));
    int *ord = (int *)malloc((size_t)d * sizeof(int));
    /* key second moment plus a small ridge */
    for (long long r = 0; r < n; ++r)
        for (int i = 0; i < d; ++i)
            for (int k = 0; k < d; ++k) A[(size_t)i * d + k] += K[r * d + i] * K[r * d + k];
    double tr = 0.0;
    for (int i = 0; i < d; ++i) tr += A[(size_t)i * d + i] / (double)n;
    for (size_t i = 0; i < dd; ++i) A[i] /= (double)n;
    for (int i = 0; i < d; ++i) A[(size_t)i * d + i] += 1e-6 * tr / d;
    jacobi_eigen(d, A, w, V);
    sym_power(d, w, V, alpha / 2.0, P);
    sym_power(d, w, V, -alpha / 2.0, Pi);
    /* query second moment in the partially whitened frame: P (Q^T Q / m) P */
    double *M = (double *)calloc(dd, sizeof(double));
    for (long long r = 0; r < m; ++r)
        for (int i = 0; i < d; ++i)
            for (int k = 0; k < d; ++k) M[(size_t)i * d + k] += Q[r * d + i] * Q[r * d + k];
    for (size_t i = 0; i < dd; ++i) M[i] /= (double)m;
    for (int i = 0; i < d; ++i)
        for (int k = 0; k < d; ++k) {
            double acc = 0.0;
            for (int a = 0; a < d; ++a)
                for (int b = 0; b < d; ++b) acc += P[(size_t)i * d + a] * M[(size_t)a * d + b] * P[(size_t)b * d + k];
            S[(size_t)i * d + k] = acc;
        }
    jacobi_eigen(d, S, mu, U);
    /* order by descending energy (stable), fix signs */
    for (int i = 0; i < d; ++i) ord[i] = i;
    for (int i = 1; i < d; ++i) {
        const int x = ord[i];
        int j = i - 1;
        while (j >= 0 && mu[ord[j]] < mu[x]) { ord[j + 1] = ord[j]; --j; }
        ord[j + 1] = x;
    }
    for (int c = 0; c < d; ++c) {
        const int src = ord[c];
        int arg = 0;
        for (int i = 1; i < d; ++i)
            if (fabs(U[(size_t)i * d + src]) > fabs(U[(size_t)arg * d + src])) arg = i;
        const double sgn = U[(size_t)arg * d + src] < 0.0 ? -1.0 : 1.0;
        /* row c of T_K = (column src of U)^T P^-1, row c of T_Q = (column src)^T P */
        for (int k = 0; k < d; ++k) {
            double ak = 0.0, bk = 0.0;
            for (int i = 0; i < d; ++i) {
                ak += sgn * U[(size_t)i * d + src] * Pi[(size_t)i * d + k];
                bk += sgn * U[(size_t)i * d + src] * P[(size_t)i * d + k];
            }
            t_k[(size_t)c * d + k] = ak;
            t_q[(size_t)c * d + k] = bk;
        }
    }
    free(A); free(V); free(w); free(P); free(Pi); free(S); free(U); free(mu); free(ord); free(M);
    return 0;
}
