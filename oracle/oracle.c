/*
 * fp64 CPU oracle for the YOCO++ cross-layer KV cache hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library calls, links or
 * includes this file; only the tests, the smoke check and the benchmark's
 * CPU-baseline leg load it.  It shares no code with the CUDA sources.
 *
 * What it computes, and where the definitions come from:
 *
 *   orc_compose      YOCO++: Enhancing YOCO with KV Residual Connections,
 *                    section 2 ("method"), the two composition equations:
 *                    X'_i = lambda * (alpha_{i,1} * X_1 + alpha_{i,2} * X_i)
 *                    for X in {K, V}, elementwise, evaluated literally
 *                    (inner weighted sum first, then the product with lambda).
 *   orc_round_bf16   rounding of a composed value to the cache's storage type
 *                    (bf16, round-to-nearest-even, directly from fp64).
 *   orc_attention    the cross-decoder's attention over the shared cache
 *                    (You Only Cache Once, abstract: the cross-decoder reuses
 *                    the cached KVs through cross-attention): for one query
 *                    head, s_t = scale * <q, K_t>, p = softmax(s), out =
 *                    sum_t p_t V_t, written as the textbook two-pass softmax
 *                    (max, then exponentials and their sum).  A one-token
 *                    query needs no causal mask inside the cache.
 *   orc_causal_attention
 *                    a self-decoder layer's prefill attention over the cache
 *                    it stores (YOCO++: Enhancing YOCO with KV Residual
 *                    Connections, section 2, cache strategy; section 3,
 *                    prefill): a token at cache position t attends causally
 *                    to positions 0..t, i.e. orc_attention of its query over
 *                    the first t + 1 cached rows.
 *   orc_attention_partial / orc_lse_combine
 *                    the same attention restricted to a token range, kept
 *                    unnormalised as (max, sum of exponentials, weighted sum),
 *                    and the exact log-sum-exp merge of such ranges.  These
 *                    exist to pin the split-and-merge identity that any
 *                    split-K implementation relies on.
 *
 * Inputs are read exactly: bf16 by widening its bit pattern, fp32 and fp64 as
 * they are.  All arithmetic is fp64.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

enum { ORC_BF16 = 0, ORC_F32 = 1, ORC_F64 = 2 };

static double load(const void* base, int dtype, int64_t i) {
    if (dtype == ORC_BF16) {
        uint32_t u = (uint32_t)((const uint16_t*)base)[i] << 16;
        float f;
        memcpy(&f, &u, 4);
        return (double)f;
    }
    if (dtype == ORC_F32) return (double)((const float*)base)[i];
    return ((const double*)base)[i];
}

/* Composition of one tensor pair (YOCO++ section 2, composition equations). */
void orc_compose(const void* x1, const void* xi, int dtype, int64_t n,
                 double a1, double a2, double lam, double* out) {
    for (int64_t j = 0; j < n; ++j) {
        double inner = a1 * load(x1, dtype, j) + a2 * load(xi, dtype, j);
        out[j] = lam * inner;
    }
}

/* fp64 -> bf16, round to nearest, ties to even, straight from fp64. */
static uint16_t to_bf16(double x) {
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (isnan(x)) return 0x7FC0;
    if (a == 0.0) return sign;
    int e;
    double m = frexp(a, &e);            /* a = m * 2^e, m in [0.5, 1) */
    int bits = 8;                        /* significant bits of a normal bf16 */
    if (e - 1 < -126) bits = 8 - (-126 - (e - 1));   /* subnormal range */
    double r = nearbyint(ldexp(m, bits)); /* default mode: nearest-even */
    double y = ldexp(r, e - bits);
    if (y > 3.38953138925153547590e38) return sign | 0x7F80;  /* overflow */
    float f = (float)y;                  /* exact: y has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    return sign | (uint16_t)(u >> 16);
}

void orc_round_bf16(const double* x, int64_t n, uint16_t* out) {
    for (int64_t j = 0; j < n; ++j) out[j] = to_bf16(x[j]);
}

void orc_round_f32(const double* x, int64_t n, float* out) {
    for (int64_t j = 0; j < n; ++j) out[j] = (float)x[j];
}

/*
 * Attention of G query heads that share one KV head, over tokens
 * [t0, t1) of K, V ([len][d] rows of the given dtype).
 *   q      [G][d] fp64 (exact values of the query)
 *   scores scratch [t1 - t0] fp64
 * Writes the unnormalised triple per head: m[h] = max_t s_t,
 * l[h] = sum_t exp(s_t - m[h]), o[h][c] = sum_t exp(s_t - m[h]) V_t[c].
 * An empty range gives m = -inf, l = 0, o = 0.
 */
void orc_attention_partial(const double* q, const void* K, const void* V, int dtype,
                           int64_t t0, int64_t t1, int d, int G, double scale,
                           double* scores, double* m, double* l, double* o) {
    for (int h = 0; h < G; ++h) {
        const double* qh = q + (int64_t)h * d;
        double mx = -INFINITY;
        for (int64_t t = t0; t < t1; ++t) {
            double dot = 0.0;
            for (int c = 0; c < d; ++c) dot += qh[c] * load(K, dtype, t * d + c);
            double s = scale * dot;
            scores[t - t0] = s;
            if (s > mx) mx = s;
        }
        double sum = 0.0;
        double* oh = o + (int64_t)h * d;
        for (int c = 0; c < d; ++c) oh[c] = 0.0;
        for (int64_t t = t0; t < t1; ++t) {
            double p = exp(scores[t - t0] - mx);
            sum += p;
            for (int c = 0; c < d; ++c) oh[c] += p * load(V, dtype, t * d + c);
        }
        m[h] = mx;
        l[h] = sum;
    }
}

/* Exact merge of unnormalised range results into the softmax-weighted output:
 * M = max_s m_s; out = sum_s e^{m_s - M} o_s / sum_s e^{m_s - M} l_s.
 * m, l: [nparts][G]; o: [nparts][G][d]; out: [G][d].  No parts -> zeros. */
void orc_lse_combine(int nparts, const double* m, const double* l, const double* o,
                     int G, int d, double* out) {
    for (int h = 0; h < G; ++h) {
        double M = -INFINITY;
        for (int s = 0; s < nparts; ++s)
            if (m[s * G + h] > M) M = m[s * G + h];
        double L = 0.0;
        double* oh = out + (int64_t)h * d;
        for (int c = 0; c < d; ++c) oh[c] = 0.0;
        if (M == -INFINITY) continue;
        for (int s = 0; s < nparts; ++s) {
            double w = exp(m[s * G + h] - M);
            L += w * l[s * G + h];
            for (int c = 0; c < d; ++c) oh[c] += w * o[((int64_t)s * G + h) * d + c];
        }
        for (int c = 0; c < d; ++c) oh[c] /= L;
    }
}

/*
 * Softmax attention over a whole sequence (two passes).
 *   q [G][d] fp64, K/V [len][d], out [G][d] fp64,
 *   weights: optional [G][len] fp64 (the softmax probabilities p_t).
 * len == 0 gives out = 0 (no tokens to attend to).
 */
void orc_attention(const double* q, const void* K, const void* V, int dtype, int64_t len,
                   int d, int G, double scale, double* scores, double* out, double* weights) {
    for (int h = 0; h < G; ++h) {
        const double* qh = q + (int64_t)h * d;
        double* oh = out + (int64_t)h * d;
        for (int c = 0; c < d; ++c) oh[c] = 0.0;
        if (len == 0) continue;
        /* pass 1: logits and their maximum */
        double mx = -INFINITY;
        for (int64_t t = 0; t < len; ++t) {
            double dot = 0.0;
            for (int c = 0; c < d; ++c) dot += qh[c] * load(K, dtype, t * d + c);
            scores[t] = scale * dot;
            if (scores[t] > mx) mx = scores[t];
        }
        /* pass 2: normaliser, then the probability-weighted sum of values */
        double Z = 0.0;
        for (int64_t t = 0; t < len; ++t) Z += exp(scores[t] - mx);
        for (int64_t t = 0; t < len; ++t) {
            double p = exp(scores[t] - mx) / Z;
            if (weights) weights[(int64_t)h * len + t] = p;
            for (int c = 0; c < d; ++c) oh[c] += p * load(V, dtype, t * d + c);
        }
    }
}

/*
 * Causal attention of a chunk of n query rows over a layer's own cache.
 * Row j of q [n][d] (fp64) is the token at cache position p0 + j; it attends
 * to cache positions 0 .. p0 + j of K/V [len][d] (len >= p0 + n), so its
 * output is the one-query orc_attention over the first p0 + j + 1 rows.
 *   scores: scratch of at least p0 + n doubles;  out [n][d] fp64.
 */
void orc_causal_attention(const double* q, const void* K, const void* V, int dtype, int64_t p0, int64_t n,
                          int d, double scale, double* scores, double* out) {
    for (int64_t j = 0; j < n; ++j) {
        const int64_t visible = p0 + j + 1;
        orc_attention(q + j * d, K, V, dtype, visible, d, 1, scale, scores, out + j * d, NULL);
    }
}
