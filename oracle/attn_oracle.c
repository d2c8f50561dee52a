/*
 * attn_oracle.c - plain fp64 CPU reference for exact self-attention forward.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the library's product path links, loads or
 * calls this file; only the tests, the smoke check and the benchmark's CPU
 * baseline do. It shares no code, header or constant with the CUDA kernels.
 *
 * What it computes (the plain three-step definition of attention, "FlashAttention
 * by hand", paragraph on the conventional computation): for every query row the
 * logits against every visible key are formed, a softmax is taken over that row
 * so that its weights sum to one, and the weights multiply the value rows. The
 * softmax row is materialised in full; there is no tiling, no online update and
 * no reordering. Alongside the output row it reports the log-sum-exp of the
 * scaled logits (natural log), the per-row statistic that partial results are
 * combined with (ATTENTION2D, section 3: fragment-local statistics combined in
 * stages).
 *
 * Readings adopted where the pages say nothing:
 *   - logits are scale * <q_i, k_j> with scale passed in (1/sqrt(d) in every
 *     workload); the scale enters as the double of the float the GPU receives;
 *   - causal masking (HOF SWIFT Attention, section 3, Transform stage) keeps key j
 *     for query i when kv_off + j <= q_off + i, positions being global;
 *   - a row with no visible key has O = 0 and LSE = -inf;
 *   - grouped heads: query head h reads key/value head h / (Hq / Hkv).
 *
 * Inputs are the exact bf16 bit patterns the GPU receives, widened to double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double bf16_bits_to_double(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * One query row of one head.
 *   qrow: d bf16 values; kh, vh: Nkv x d bf16 values of the matching kv head.
 *   s: scratch of Nkv doubles. p_out: optional Nkv doubles receiving the
 *   softmax row (zeros at masked keys).
 */
static void attend_one_row(const uint16_t *qrow, const uint16_t *kh, const uint16_t *vh,
                           int64_t Nkv, int d, int causal, int64_t qpos, int64_t kv_off,
                           double scale, double *s, double *o_row, double *lse_out,
                           double *p_out)
{
    /* visible keys: j < Nkv and, if causal, kv_off + j <= qpos */
    int64_t nvis = Nkv;
    if (causal) {
        int64_t last = qpos - kv_off; /* largest visible j */
        if (last < 0)
            nvis = 0;
        else if (last + 1 < Nkv)
            nvis = last + 1;
    }
    for (int c = 0; c < d; ++c)
        o_row[c] = 0.0;
    if (p_out)
        for (int64_t j = 0; j < Nkv; ++j)
            p_out[j] = 0.0;
    if (nvis == 0) {
        *lse_out = -INFINITY;
        return;
    }

    /* step 1: logits */
    for (int64_t j = 0; j < nvis; ++j) {
        double acc = 0.0;
        const uint16_t *krow = kh + j * (int64_t)d;
        for (int c = 0; c < d; ++c)
            acc += bf16_bits_to_double(qrow[c]) * bf16_bits_to_double(krow[c]);
        s[j] = scale * acc;
    }

    /* step 2: softmax over the row (max subtracted so that exp cannot overflow) */
    double m = s[0];
    for (int64_t j = 1; j < nvis; ++j)
        if (s[j] > m)
            m = s[j];
    double l = 0.0;
    for (int64_t j = 0; j < nvis; ++j) {
        s[j] = exp(s[j] - m);
        l += s[j];
    }
    for (int64_t j = 0; j < nvis; ++j)
        s[j] /= l; /* s now holds the softmax row P_i. */
    if (p_out)
        for (int64_t j = 0; j < nvis; ++j)
            p_out[j] = s[j];

    /* step 3: weights times values */
    for (int64_t j = 0; j < nvis; ++j) {
        const uint16_t *vrow = vh + j * (int64_t)d;
        for (int c = 0; c < d; ++c)
            o_row[c] += s[j] * bf16_bits_to_double(vrow[c]);
    }
    *lse_out = m + log(l);
}

/*
 * Attention forward for a chosen list of query rows (the same list for every head).
 *
 *   q: [B, Hq, Nq, d] bf16 bits; k, v: [B, Hkv, Nkv, d] bf16 bits, all dense.
 *   rows: nrows indices in [0, Nq).
 *   o: [B, Hq, nrows, d] doubles; lse: [B, Hq, nrows] doubles.
 *   p: optional [B, Hq, nrows, Nkv] doubles receiving the softmax rows.
 *   nthreads: OpenMP threads (<= 0: the runtime's default).
 * Returns 0, or -1 on a bad argument, or -2 if scratch memory cannot be had.
 */
int oracle_attention_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                          int B, int Hq, int Hkv, int64_t Nq, int64_t Nkv, int d,
                          int causal, int64_t q_off, int64_t kv_off, double scale,
                          const int64_t *rows, int64_t nrows, double *o, double *lse,
                          double *p, int nthreads)
{
    if (!q || !k || !v || !rows || !o || !lse || B < 1 || Hq < 1 || Hkv < 1 ||
        Hq % Hkv != 0 || Nq < 1 || Nkv < 1 || d < 1 || nrows < 0)
        return -1;
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= Nq)
            return -1;

    const int group = Hq / Hkv;
    const int64_t total = (int64_t)B * Hq * nrows;
    int failed = 0;
#ifdef _OPENMP
    if (nthreads <= 0)
        nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads) reduction(| : failed)
#endif
    {
        double *s = (double *)malloc((size_t)Nkv * sizeof(double));
        if (!s) {
            failed = 1;
        } else {
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 4)
#endif
            for (int64_t t = 0; t < total; ++t) {
                const int64_t r = t % nrows;
                const int64_t bh = t / nrows;
                const int h = (int)(bh % Hq);
                const int b = (int)(bh / Hq);
                const int g = h / group;
                const int64_t i = rows[r];
                const uint16_t *qrow = q + (((int64_t)b * Hq + h) * Nq + i) * d;
                const uint16_t *kh = k + ((int64_t)b * Hkv + g) * Nkv * d;
                const uint16_t *vh = v + ((int64_t)b * Hkv + g) * Nkv * d;
                attend_one_row(qrow, kh, vh, Nkv, d, causal, q_off + i, kv_off, scale, s,
                               o + t * d, lse + t, p ? p + t * Nkv : NULL);
            }
            free(s);
        }
    }
    (void)nthreads;
    return failed ? -2 : 0;
}

/* Number of OpenMP threads a call with nthreads <= 0 would use. */
int oracle_default_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
