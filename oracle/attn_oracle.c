/*
 * attn_oracle.c -- f64 CPU oracle for states-form KV-cache attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file; only the tests, __graft_entry__.smoke() and the CPU
 * baseline leg of bench.py do.  It shares no code, header or constant with
 * the CUDA library.
 *
 * What it computes (the plain definition, no blocking, no online softmax):
 *
 *   For a query row at absolute position `pos` of a sequence whose cached
 *   rows start at row `kv_base`, and query head h with KV head
 *   g = h / (n_q_heads / n_kv_heads):
 *
 *     visible keys  J = [lo, pos],  lo = (window > 0) ? max(0, pos-window+1) : 0
 *     s_j   = scale * sum_t q[h,t] * k[kv_base+j, g, t]          (j in J)
 *     m     = max_j s_j   (NaN as soon as any s_j is NaN)
 *     o[h,:] = sum_j exp(s_j - m) v[kv_base+j, g, :] / sum_j exp(s_j - m)
 *     J empty (pos < 0)  ->  o = 0 exactly.
 *
 * Sources on the pages:
 *   - Karume v0.8.0 release notes, "Breaking Changes", the softmax NaN item:
 *     the row max is NaN-preserving, and a fully masked row of fused
 *     attention yields exactly 0.
 *   - Karume v0.12.0 release notes, "Performance", first three items: the
 *     states-form attention over the KV "state" buffers (QK, softmax
 *     statistics, PV), whose parallel variants differ from the reference
 *     reduction only by reduction order and are checked against an f64
 *     reference.
 *   - Karume v0.8.0 release notes, "Features", the run-time window item: the
 *     KV cache is a run-time capacity that chunked prefill fills in chunks of
 *     at most 768 rows; each chunk row attends to every cached row before it
 *     and to the chunk rows up to itself (causal).
 *   The sliding window, head grouping (8 query heads per KV head), head_dim
 *   256 and scale 1/sqrt(256) are not on the pages; they are parameters here.
 *
 * Inputs are read in their stored format (f32, f16 or bf16 bit patterns) and
 * widened to double exactly by the decoders below, written from the IEEE 754
 * binary16 definition and from bfloat16 being the upper half of binary32.
 *
 * Parity status: pinned (Python decimal brute force, torch f64 SDPA special
 * case, closed forms and invariants in tests/test_oracle.py).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_F32 = 0, ORC_F16 = 1, ORC_BF16 = 2, ORC_F64 = 3 };

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
static double orc_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int ex = (h >> 10) & 0x1f;
    int fr = h & 0x3ff;
    double mag;
    if (ex == 0)
        mag = ldexp((double)fr, -24);               /* subnormal: fr * 2^-14 * 2^-10 */
    else if (ex == 31)
        mag = fr ? NAN : INFINITY;
    else
        mag = ldexp((double)(fr + 1024), ex - 25);  /* 1.fr * 2^(ex-15) */
    return sign ? -mag : mag;
}

/* bfloat16 is the upper 16 bits of an IEEE 754 binary32. */
static double orc_bf16_to_double(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double orc_load(const void *base, int dtype, int64_t idx)
{
    switch (dtype) {
    case ORC_F32: return (double)((const float *)base)[idx];
    case ORC_F16: return orc_half_to_double(((const uint16_t *)base)[idx]);
    case ORC_BF16: return orc_bf16_to_double(((const uint16_t *)base)[idx]);
    case ORC_F64: return ((const double *)base)[idx];
    default: return NAN;
    }
}

/* Exposed so a test can compare the decoders with library conversions. */
double oracle_decode_element(const void *base, int dtype, int64_t idx)
{
    return orc_load(base, dtype, idx);
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/*
 * q      : [n_query][n_q_heads][head_dim], dtype q_dtype
 * k, v   : rows of [n_kv_heads][head_dim], dtype kv_dtype; row r at r*n_kv_heads*head_dim
 * kv_base: [n_query] first row of the query's sequence
 * pos    : [n_query] absolute position of the query (pos < 0: no visible key)
 * out    : [n_query][n_q_heads][head_dim] doubles
 * Returns 0, or -1 on a bad argument.
 */
int oracle_attention(const void *q, int q_dtype,
                     const void *k, const void *v, int kv_dtype,
                     const int64_t *kv_base, const int64_t *pos,
                     int64_t n_query, int n_q_heads, int n_kv_heads, int head_dim,
                     int window, double scale, double *out)
{
    if (!q || !k || !v || !kv_base || !pos || !out) return -1;
    if (n_query < 0 || n_q_heads <= 0 || n_kv_heads <= 0 || head_dim <= 0) return -1;
    if (n_q_heads % n_kv_heads != 0) return -1;
    const int group = n_q_heads / n_kv_heads;
    const int64_t n_pairs = n_query * (int64_t)n_q_heads;
    int failed = 0;

#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t pr = 0; pr < n_pairs; ++pr) {
        const int64_t i = pr / n_q_heads;
        const int h = (int)(pr % n_q_heads);
        const int g = h / group;
        double *o = out + pr * head_dim;
        const int64_t p = pos[i];
        int64_t lo = 0;
        if (window > 0 && p - window + 1 > 0) lo = p - window + 1;
        const int64_t n = (p >= lo) ? p - lo + 1 : 0;
        for (int t = 0; t < head_dim; ++t) o[t] = 0.0;
        if (n == 0) continue;                      /* fully masked row -> exactly 0 */

        double *s = (double *)malloc((size_t)n * sizeof(double));
        double *qd = (double *)malloc((size_t)head_dim * sizeof(double));
        if (!s || !qd) {
            free(s); free(qd);
#pragma omp atomic write
            failed = 1;
            continue;
        }
        const int64_t q_off = pr * head_dim;
        for (int t = 0; t < head_dim; ++t) qd[t] = orc_load(q, q_dtype, q_off + t);

        /* pass 1: scores and their NaN-preserving maximum */
        double m = -INFINITY;
        int any_nan = 0;
        for (int64_t j = 0; j < n; ++j) {
            const int64_t row = kv_base[i] + lo + j;
            const int64_t k_off = (row * n_kv_heads + g) * (int64_t)head_dim;
            double dot = 0.0;
            for (int t = 0; t < head_dim; ++t) dot += qd[t] * orc_load(k, kv_dtype, k_off + t);
            s[j] = scale * dot;
            if (isnan(s[j])) any_nan = 1;
            else if (s[j] > m) m = s[j];
        }
        if (any_nan) m = NAN;

        /* pass 2: exp weights, their sum, and the weighted sum of V rows */
        double den = 0.0;
        for (int64_t j = 0; j < n; ++j) {
            const double w = exp(s[j] - m);
            const int64_t row = kv_base[i] + lo + j;
            const int64_t v_off = (row * n_kv_heads + g) * (int64_t)head_dim;
            den += w;
            for (int t = 0; t < head_dim; ++t) o[t] += w * orc_load(v, kv_dtype, v_off + t);
        }
        for (int t = 0; t < head_dim; ++t) o[t] /= den;
        free(s);
        free(qd);
    }
    return failed ? -1 : 0;
}
