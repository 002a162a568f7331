/*
 * mla_oracle.c -- plain fp64 CPU oracle for Multi-head Latent Attention (MLA)
 * decode.  TEST INFRASTRUCTURE ONLY: tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py are the only callers.  The CUDA
 * library never links, loads or calls this file, and this file uses nothing
 * from the CUDA library (no shared headers, helpers, tables or constants).
 *
 * What it computes.  MLA decode is the running example, ablation subject and
 * headline benchmark of "TileLang: Bridging Programmability and Performance in
 * Modern Neural Kernels" (papernotes.org summary, section "一个完整示例：FlashMLA
 * 的两阶段优化" and the main-results table "主实验", row FlashMLA); the hackmd
 * essay "TileLang 完整解析" benchmarks it in section "FlashMLA Benchmark".  The
 * pages describe the kernel as two GEMMs around a softmax (S = Q K^T, then
 * P V) but never write the formula, so this file writes out the textbook
 * definition of scaled-dot-product attention over a shared latent cache:
 *
 *   for every sequence b, query token t < Sq, head h < H, with L = seqlens[b]:
 *     s_j          = scale * sum_{d < d_qk} q[b,t,h,d] * kv[b,j,d]      (j < L)
 *     m            = max_j s_j
 *     l            = sum_j exp(s_j - m)
 *     out[b,t,h,e] = sum_j exp(s_j - m) * kv[b,j,e] / l                (e < d_v)
 *     lse[b,t,h]   = m + ln(l)                                   (natural log)
 *
 * Attention sinks (optional).  A sink is one extra logit per head, sigma_h,
 * in the units of the scaled scores, that enters the softmax denominator and
 * carries no value.  The TileLang summary lists an attention-sink kernel in
 * its main-results table (section "主实验", row "Attention Sinks") and notes
 * in "关键发现" that it is a small change to standard attention; it prints no
 * formula, so this is the plain reading:
 *     m   = max(sigma_h, max_j s_j)
 *     l   = sum_j exp(s_j - m) + exp(sigma_h - m)
 *     out = sum_j exp(s_j - m) * kv[b,j,e] / l,     lse = m + ln(l)
 * and an empty sequence gives out = 0, lse = sigma_h.  sigma_h = -inf is the
 * sink-free definition above, bit for bit.
 *
 * Keys are the d_qk-wide latent rows (512 latent + 64 rope = 576 for MLA) and
 * the values are the first d_v (= 512) columns of the very same rows.  The Sq
 * query tokens of a sequence all see keys 0..L-1 (no mask between them).  An
 * empty sequence (L = 0) gives out = 0 and lse = -inf.
 *
 * Arithmetic: every bf16 input is widened exactly to double; sums run in
 * index order in double; exp/log are the C library's double routines.  Two
 * passes (max, then sum): no base-2 trick, no online rescaling, no splitting,
 * no blocking.  Parallelism: OpenMP over independent (b, t, h) rows only.
 *
 * Parity pins (tests/test_oracle.py, CPU only): closed forms (single key,
 * identical keys, q = 0, two keys), invariants (permutation of keys, a shared
 * additive score shift, head and token independence), brute force in 50-digit
 * decimal arithmetic on tiny shapes, and torch's fp64 scaled_dot_product_
 * attention as an independent library routine.  The FP8-cache section at the
 * end is pinned by the format's closed-form code values, torch's own E4M3
 * decoding of all 256 codes, torch's fp64 attention over the dequantised
 * cache, a single-key closed form, a scale-trade invariant, and equality with
 * the bf16 definition when every value is exact in bf16.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Exact widening of a bfloat16 bit pattern: bf16 is the top half of an IEEE
 * binary32, so shifting the bits up gives the float, and float -> double is
 * exact. */
static double bf16_bits_to_double(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* One output row (b, t, h): the definition above, written out. `scores` is a
 * caller-owned scratch array of at least L doubles; `sink` is sigma_h, or
 * -INFINITY for no sink. */
static void attend_one_row(const uint16_t *q_row, const uint16_t *kv_seq,
                           int64_t L, int64_t d_qk, int64_t d_v, double scale, double sink,
                           double *scores, double *out_row, double *lse_out)
{
    if (L <= 0) {
        for (int64_t e = 0; e < d_v; ++e) out_row[e] = 0.0;
        *lse_out = sink;
        return;
    }
    /* s_j = scale * <q, k_j> over all d_qk columns (latent + rope). */
    for (int64_t j = 0; j < L; ++j) {
        const uint16_t *k_row = kv_seq + j * d_qk;
        double dot = 0.0;
        for (int64_t d = 0; d < d_qk; ++d)
            dot += bf16_bits_to_double(q_row[d]) * bf16_bits_to_double(k_row[d]);
        scores[j] = scale * dot;
    }
    /* m = max(sink, max_j s_j) */
    double m = scores[0];
    for (int64_t j = 1; j < L; ++j)
        if (scores[j] > m) m = scores[j];
    if (sink > m) m = sink;
    /* w_j = exp(s_j - m), l = sum_j w_j + exp(sink - m) (the sink term is 0 for no sink) */
    double l = 0.0;
    for (int64_t j = 0; j < L; ++j) {
        scores[j] = exp(scores[j] - m);
        l += scores[j];
    }
    l += exp(sink - m);
    /* out_e = sum_j w_j * v_j[e] / l, with v_j = first d_v columns of row j */
    for (int64_t e = 0; e < d_v; ++e) out_row[e] = 0.0;
    for (int64_t j = 0; j < L; ++j) {
        const uint16_t *v_row = kv_seq + j * d_qk;
        const double w = scores[j];
        for (int64_t e = 0; e < d_v; ++e)
            out_row[e] += w * bf16_bits_to_double(v_row[e]);
    }
    for (int64_t e = 0; e < d_v; ++e) out_row[e] /= l;
    *lse_out = m + log(l);
}

/*
 * Full oracle.
 *   q       : bf16 bits, [B, Sq, H, d_qk] contiguous
 *   kv      : bf16 bits, [B, L_max, d_qk] contiguous (values = first d_v cols)
 *   seqlens : int32 [B], 0 <= seqlens[b] <= L_max
 *   sinks   : double [H] sink logits, or NULL for none
 *   out     : double [B, Sq, H, d_v];  lse : double [B, Sq, H]
 * Returns 0 on success, -1 on bad arguments, -2 on allocation failure.
 */
int oracle_mla_decode_sinks(const uint16_t *q, const uint16_t *kv, const int32_t *seqlens,
                            int64_t B, int64_t Sq, int64_t H, int64_t L_max,
                            int64_t d_qk, int64_t d_v, double scale, const double *sinks,
                            double *out, double *lse, int num_threads)
{
    if (!q || !kv || !seqlens || !out || !lse) return -1;
    if (B < 0 || Sq < 1 || H < 1 || L_max < 0 || d_qk < 1 || d_v < 1 || d_v > d_qk) return -1;
    for (int64_t b = 0; b < B; ++b)
        if (seqlens[b] < 0 || seqlens[b] > L_max) return -1;
    const int64_t rows = B * Sq * H;
    int failed = 0;
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#else
    (void)num_threads;
#endif
#pragma omp parallel
    {
        double *scores = (double *)malloc(sizeof(double) * (size_t)(L_max > 0 ? L_max : 1));
        if (!scores) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < rows; ++r) {
                const int64_t b = r / (Sq * H);
                const double sink = sinks ? sinks[r % H] : -INFINITY;
                attend_one_row(q + r * d_qk, kv + b * L_max * d_qk, seqlens[b],
                               d_qk, d_v, scale, sink, scores, out + r * d_v, lse + r);
            }
            free(scores);
        }
    }
    return failed ? -2 : 0;
}

int oracle_mla_decode(const uint16_t *q, const uint16_t *kv, const int32_t *seqlens,
                      int64_t B, int64_t Sq, int64_t H, int64_t L_max,
                      int64_t d_qk, int64_t d_v, double scale,
                      double *out, double *lse, int num_threads)
{
    return oracle_mla_decode_sinks(q, kv, seqlens, B, Sq, H, L_max, d_qk, d_v, scale, NULL, out, lse,
                                   num_threads);
}

/*
 * Sampled oracle: the same definition for a caller-chosen list of flattened
 * row indices r = (b * Sq + t) * H + h, so that full-size workloads can be
 * checked row by row.  out is [n_rows, d_v], lse is [n_rows]; sinks as above.
 */
int oracle_mla_decode_rows_sinks(const uint16_t *q, const uint16_t *kv, const int32_t *seqlens,
                                 int64_t B, int64_t Sq, int64_t H, int64_t L_max,
                                 int64_t d_qk, int64_t d_v, double scale, const double *sinks,
                                 const int64_t *row_ids, int64_t n_rows,
                                 double *out, double *lse, int num_threads)
{
    if (!q || !kv || !seqlens || !row_ids || !out || !lse) return -1;
    if (B < 0 || Sq < 1 || H < 1 || L_max < 0 || d_qk < 1 || d_v < 1 || d_v > d_qk) return -1;
    for (int64_t i = 0; i < n_rows; ++i)
        if (row_ids[i] < 0 || row_ids[i] >= B * Sq * H) return -1;
    for (int64_t b = 0; b < B; ++b)
        if (seqlens[b] < 0 || seqlens[b] > L_max) return -1;
    int failed = 0;
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#else
    (void)num_threads;
#endif
#pragma omp parallel
    {
        double *scores = (double *)malloc(sizeof(double) * (size_t)(L_max > 0 ? L_max : 1));
        if (!scores) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t i = 0; i < n_rows; ++i) {
                const int64_t r = row_ids[i];
                const int64_t b = r / (Sq * H);
                const double sink = sinks ? sinks[r % H] : -INFINITY;
                attend_one_row(q + r * d_qk, kv + b * L_max * d_qk, seqlens[b],
                               d_qk, d_v, scale, sink, scores, out + i * d_v, lse + i);
            }
            free(scores);
        }
    }
    return failed ? -2 : 0;
}

int oracle_mla_decode_rows(const uint16_t *q, const uint16_t *kv, const int32_t *seqlens,
                           int64_t B, int64_t Sq, int64_t H, int64_t L_max,
                           int64_t d_qk, int64_t d_v, double scale,
                           const int64_t *row_ids, int64_t n_rows,
                           double *out, double *lse, int num_threads)
{
    return oracle_mla_decode_rows_sinks(q, kv, seqlens, B, Sq, H, L_max, d_qk, d_v, scale, NULL, row_ids,
                                        n_rows, out, lse, num_threads);
}

/* Number of OpenMP threads a parallel region of this library would use. */
int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------
 * MHA decode (the second workload on the same skeleton): standard
 * multi-head attention with a separate V tensor and grouped KV heads.  The
 * TileLang summary lists MHA in its main-results table (section "主实验",
 * row "MHA", matched against FlashAttention-3) and uses it as the base the
 * attention-sink variant differs from ("关键发现").  No formula is printed;
 * this is the textbook definition:
 *
 *   for sequence b, token t < Sq, head h < H, kv head hk = h / (H / Hkv),
 *   with L = seqlens[b]:
 *     s_j          = scale * sum_{d < D} q[b,t,h,d] * k[b,j,hk,d]      (j < L)
 *     out[b,t,h,e] = sum_j exp(s_j - m) * v[b,j,hk,e] / l              (e < Dv)
 *     lse[b,t,h]   = m + ln(l),   m = max_j s_j,   l = sum_j exp(s_j - m)
 *
 * Same arithmetic rules as above (exact widening, index-order sums, two
 * passes, no blocking); L = 0 gives out = 0, lse = -inf.  With attention
 * sinks the same per-head sink logit sigma_h as in the latent-cache entry
 * point above (natural-log units, not scaled, no value) enters the max and
 * the denominator: m = max(sigma_h, max_j s_j), l = sum_j exp(s_j - m) +
 * exp(sigma_h - m); an empty sequence gives out = 0, lse = sigma_h.
 *   q : bf16 [B, Sq, H, D];  k : bf16 [B, L_max, Hkv, D];  v : bf16 [B, L_max, Hkv, Dv]
 *   sinks : double [H] or NULL (no sinks)
 *   out : double [B, Sq, H, Dv];  lse : double [B, Sq, H]
 * ------------------------------------------------------------------------ */
static void mha_one_row(const uint16_t *q_row, const uint16_t *k_seq, const uint16_t *v_seq,
                        int64_t L, int64_t Hkv, int64_t hk, int64_t D, int64_t Dv, double scale, double sink,
                        double *scores, double *out_row, double *lse_out)
{
    if (L <= 0) {
        for (int64_t e = 0; e < Dv; ++e) out_row[e] = 0.0;
        *lse_out = sink;
        return;
    }
    for (int64_t j = 0; j < L; ++j) {
        const uint16_t *k_row = k_seq + (j * Hkv + hk) * D;
        double dot = 0.0;
        for (int64_t d = 0; d < D; ++d)
            dot += bf16_bits_to_double(q_row[d]) * bf16_bits_to_double(k_row[d]);
        scores[j] = scale * dot;
    }
    double m = scores[0];
    for (int64_t j = 1; j < L; ++j)
        if (scores[j] > m) m = scores[j];
    if (sink > m) m = sink;
    double l = 0.0;
    for (int64_t j = 0; j < L; ++j) {
        scores[j] = exp(scores[j] - m);
        l += scores[j];
    }
    l += exp(sink - m);
    for (int64_t e = 0; e < Dv; ++e) out_row[e] = 0.0;
    for (int64_t j = 0; j < L; ++j) {
        const uint16_t *v_row = v_seq + (j * Hkv + hk) * Dv;
        const double w = scores[j];
        for (int64_t e = 0; e < Dv; ++e)
            out_row[e] += w * bf16_bits_to_double(v_row[e]);
    }
    for (int64_t e = 0; e < Dv; ++e) out_row[e] /= l;
    *lse_out = m + log(l);
}

int oracle_mha_decode_sinks(const uint16_t *q, const uint16_t *k, const uint16_t *v, const int32_t *seqlens,
                            int64_t B, int64_t Sq, int64_t H, int64_t Hkv, int64_t L_max, int64_t D, int64_t Dv,
                            double scale, const double *sinks, double *out, double *lse, int num_threads)
{
    if (!q || !k || !v || !seqlens || !out || !lse) return -1;
    if (B < 0 || Sq < 1 || H < 1 || Hkv < 1 || H % Hkv != 0 || L_max < 0 || D < 1 || Dv < 1) return -1;
    for (int64_t b = 0; b < B; ++b)
        if (seqlens[b] < 0 || seqlens[b] > L_max) return -1;
    const int64_t rows = B * Sq * H;
    const int64_t group = H / Hkv;
    int failed = 0;
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#else
    (void)num_threads;
#endif
#pragma omp parallel
    {
        double *scores = (double *)malloc(sizeof(double) * (size_t)(L_max > 0 ? L_max : 1));
        if (!scores) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < rows; ++r) {
                const int64_t b = r / (Sq * H);
                const int64_t h = r % H;
                const double sink = sinks ? sinks[h] : -INFINITY;
                mha_one_row(q + r * D, k + b * L_max * Hkv * D, v + b * L_max * Hkv * Dv, seqlens[b], Hkv,
                            h / group, D, Dv, scale, sink, scores, out + r * Dv, lse + r);
            }
            free(scores);
        }
    }
    return failed ? -2 : 0;
}

int oracle_mha_decode(const uint16_t *q, const uint16_t *k, const uint16_t *v, const int32_t *seqlens,
                      int64_t B, int64_t Sq, int64_t H, int64_t Hkv, int64_t L_max, int64_t D, int64_t Dv,
                      double scale, double *out, double *lse, int num_threads)
{
    return oracle_mha_decode_sinks(q, k, v, seqlens, B, Sq, H, Hkv, L_max, D, Dv, scale, NULL, out, lse,
                                   num_threads);
}

/* ------------------------------------------------------------------------
 * FP8 latent cache.  The same MLA decode, with the cache stored as 8-bit
 * floating-point codes and one dequantization scale for the whole cache.
 * The hackmd essay "TileLang 完整解析" (section "冷靜看待：TileLang 的局限與挑戰")
 * names FP8 as the precision where TileLang's kernels trail or fail, and
 * prints no format; the plain reading taken here is the common one for a
 * quantized KV cache:
 *
 *   every element of kv[b, j, d] is an OCP "E4M3" code (1 sign bit, 4
 *   exponent bits with bias 7, 3 mantissa bits; exponent field 0 encodes
 *   subnormals (m / 8) 2^-6; S.1111.111 is NaN; there are no infinities;
 *   largest finite magnitude 448), and the cached value is
 *       kv_value = kv_scale * e4m3(code)
 *   with kv_scale > 0 one fp32 number for the whole cache.
 *
 * The attention is then the definition at the top of this file applied to
 * those values (sinks included): q stays bf16, keys are all 576 dequantized
 * columns, values their first 512.  Arithmetic: each code is decoded exactly
 * to double, multiplied by kv_scale in double (exact: 4 x 24 significand
 * bits), and the rest is the same two-pass fp64 computation.
 * ------------------------------------------------------------------------ */
static double e4m3_to_double(uint8_t code)
{
    const int sign = code >> 7;
    const int ex = (code >> 3) & 15;
    const int man = code & 7;
    double v;
    if (ex == 15 && man == 7) return NAN;
    if (ex == 0)
        v = ldexp((double)man / 8.0, -6);           /* subnormal: 0.mmm x 2^(1 - 7) */
    else
        v = ldexp(1.0 + (double)man / 8.0, ex - 7); /* normal: 1.mmm x 2^(e - 7) */
    return sign ? -v : v;
}

double oracle_e4m3_to_double(uint8_t code) { return e4m3_to_double(code); }

/* One output row over an FP8 cache; as attend_one_row, with k_j[d] =
 * kv_scale * e4m3(kv_seq[j, d]). */
static void attend_one_row_fp8(const uint16_t *q_row, const uint8_t *kv_seq, double kv_scale,
                               int64_t L, int64_t d_qk, int64_t d_v, double scale, double sink,
                               double *scores, double *out_row, double *lse_out)
{
    if (L <= 0) {
        for (int64_t e = 0; e < d_v; ++e) out_row[e] = 0.0;
        *lse_out = sink;
        return;
    }
    for (int64_t j = 0; j < L; ++j) {
        const uint8_t *k_row = kv_seq + j * d_qk;
        double dot = 0.0;
        for (int64_t d = 0; d < d_qk; ++d)
            dot += bf16_bits_to_double(q_row[d]) * (kv_scale * e4m3_to_double(k_row[d]));
        scores[j] = scale * dot;
    }
    double m = scores[0];
    for (int64_t j = 1; j < L; ++j)
        if (scores[j] > m) m = scores[j];
    if (sink > m) m = sink;
    double l = 0.0;
    for (int64_t j = 0; j < L; ++j) {
        scores[j] = exp(scores[j] - m);
        l += scores[j];
    }
    l += exp(sink - m);
    for (int64_t e = 0; e < d_v; ++e) out_row[e] = 0.0;
    for (int64_t j = 0; j < L; ++j) {
        const uint8_t *v_row = kv_seq + j * d_qk;
        const double w = scores[j];
        for (int64_t e = 0; e < d_v; ++e)
            out_row[e] += w * (kv_scale * e4m3_to_double(v_row[e]));
    }
    for (int64_t e = 0; e < d_v; ++e) out_row[e] /= l;
    *lse_out = m + log(l);
}

/*
 * FP8-cache oracle for caller-chosen flattened rows r = (b * Sq + t) * H + h
 * (row_ids = NULL: every row, in order, n_rows ignored).
 *   q : bf16 bits [B, Sq, H, d_qk];  kv : E4M3 codes [B, L_max, d_qk]
 *   kv_scale : the cache's dequantization scale;  sinks : double [H] or NULL
 *   out : double [n, d_v];  lse : double [n]
 */
int oracle_mla_decode_fp8_rows(const uint16_t *q, const uint8_t *kv, double kv_scale, const int32_t *seqlens,
                               int64_t B, int64_t Sq, int64_t H, int64_t L_max,
                               int64_t d_qk, int64_t d_v, double scale, const double *sinks,
                               const int64_t *row_ids, int64_t n_rows,
                               double *out, double *lse, int num_threads)
{
    if (!q || !kv || !seqlens || !out || !lse) return -1;
    if (B < 0 || Sq < 1 || H < 1 || L_max < 0 || d_qk < 1 || d_v < 1 || d_v > d_qk) return -1;
    if (!isfinite(kv_scale)) return -1;
    const int64_t all = B * Sq * H;
    if (!row_ids) n_rows = all;
    for (int64_t i = 0; row_ids && i < n_rows; ++i)
        if (row_ids[i] < 0 || row_ids[i] >= all) return -1;
    for (int64_t b = 0; b < B; ++b)
        if (seqlens[b] < 0 || seqlens[b] > L_max) return -1;
    int failed = 0;
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#else
    (void)num_threads;
#endif
#pragma omp parallel
    {
        double *scores = (double *)malloc(sizeof(double) * (size_t)(L_max > 0 ? L_max : 1));
        if (!scores) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t i = 0; i < n_rows; ++i) {
                const int64_t r = row_ids ? row_ids[i] : i;
                const int64_t b = r / (Sq * H);
                const double sink = sinks ? sinks[r % H] : -INFINITY;
                attend_one_row_fp8(q + r * d_qk, kv + b * L_max * d_qk, kv_scale, seqlens[b],
                                   d_qk, d_v, scale, sink, scores, out + i * d_v, lse + i);
            }
            free(scores);
        }
    }
    return failed ? -2 : 0;
}
