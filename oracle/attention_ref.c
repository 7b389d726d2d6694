/*
 * attention_ref.c -- CPU fp64 reference for masked softmax attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or
 * calls this file; only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no code, header or table with the CUDA
 * library.
 *
 * What it computes is the plain definition of attention, row by row:
 *
 *   s_k = scale * (q_t . k_k)            for every allowed key k
 *   M   = max_k s_k
 *   p_k = exp(s_k - M) / sum_j exp(s_j - M)
 *   o_t = sum_k p_k v_k,    lse_t = M + ln(sum_j exp(s_j - M))
 *
 * Sources (page title, then the passage):
 *  - "Self-Attention 이후: 트랜스포머 다음에 올 것들", section "셀프 어텐션이
 *    비싼 이유": scores are Q K^T divided by sqrt(d_k), then a row softmax,
 *    then a product with V.
 *  - Newsletter on Softmax/FlashAttention, section "수치 안정성이라는 숨은
 *    비용": the row maximum is subtracted before exp; the result is unchanged.
 *  - "Flux Attention: 효율적인 LLM 추론을 위한 문맥 인식형 하이브리드
 *    어텐션", implementation paragraph: the sparse path works on 64-token
 *    blocks and keeps 128 sink tokens.  The allowed key set of a sparse row is
 *    given here as a dense block mask, built by the Python side of the oracle
 *    from a brute-force enumeration of the block rule.
 *
 * Causality: key k is allowed for query t only when k <= t (decoder prefill).
 * The query head h reads key/value head floor(h / G), G = Hq / Hkv.
 *
 * Inputs are raw bf16 bit patterns (uint16); each is widened to fp64 exactly.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf16_bits_to_double(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16; /* bf16 is the top half of an fp32 */
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * One output row.  `allowed(k)` is decided by the caller through key_ok,
 * an array of n_keys flags (1 = key attended).  Keys are rows of `kbase`
 * and `vbase` at a stride of `kv_row_stride` elements.
 */
static void attend_one_row(const uint16_t *q_row, const uint16_t *kbase,
                           const uint16_t *vbase, long kv_row_stride, int D,
                           long n_keys, const uint8_t *key_ok, double scale,
                           double *scores, double *out, double *lse_out)
{
    double q[512];
    for (int d = 0; d < D; ++d) q[d] = bf16_bits_to_double(q_row[d]);

    double M = -INFINITY;
    for (long k = 0; k < n_keys; ++k) {
        if (!key_ok[k]) continue;
        const uint16_t *kr = kbase + k * kv_row_stride;
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += q[d] * bf16_bits_to_double(kr[d]);
        scores[k] = dot * scale;
        if (scores[k] > M) M = scores[k];
    }
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    if (M == -INFINITY) { /* no key allowed: empty sum, output 0 */
        if (lse_out) *lse_out = -INFINITY;
        return;
    }
    double denom = 0.0;
    for (long k = 0; k < n_keys; ++k) {
        if (!key_ok[k]) continue;
        double p = exp(scores[k] - M);
        denom += p;
        const uint16_t *vr = vbase + k * kv_row_stride;
        for (int d = 0; d < D; ++d) out[d] += p * bf16_bits_to_double(vr[d]);
    }
    for (int d = 0; d < D; ++d) out[d] /= denom;
    if (lse_out) *lse_out = M + log(denom);
}

/*
 * Prefill rows.
 *   q: [B, S, Hq, D] bf16 bits;  k, v: [B, S, Hkv, D] bf16 bits
 *   block_mask: NULL for full causal attention, else a dense [nqb, nkb]
 *               byte mask (nqb = nkb = ceil(S / blk)); key k is allowed for
 *               query t iff k <= t and block_mask[(t/blk)*nkb + k/blk] != 0.
 *   rows: n_rows triples (b, h, t); out: [n_rows, D]; lse: [n_rows] or NULL.
 * Returns 0, or -1 on a bad argument.
 */
int oracle_attention_rows(const uint16_t *q, const uint16_t *k,
                          const uint16_t *v, int B, int S, int Hq, int Hkv,
                          int D, double scale, const uint8_t *block_mask,
                          int blk, const int64_t *rows, long n_rows,
                          double *out, double *lse)
{
    if (D <= 0 || D > 512 || Hkv <= 0 || Hq % Hkv != 0 || S <= 0 || B <= 0)
        return -1;
    if (block_mask && blk <= 0) return -1;
    const int G = Hq / Hkv;
    const long nkb = block_mask ? (S + blk - 1) / blk : 0;
    int bad = 0;

#pragma omp parallel
    {
        double *scores = (double *)malloc(sizeof(double) * (size_t)S);
        uint8_t *key_ok = (uint8_t *)malloc((size_t)S);
#pragma omp for schedule(dynamic, 4)
        for (long r = 0; r < n_rows; ++r) {
            const long b = rows[3 * r + 0], h = rows[3 * r + 1], t = rows[3 * r + 2];
            if (b < 0 || b >= B || h < 0 || h >= Hq || t < 0 || t >= S) {
                bad = 1;
                continue;
            }
            const long kvh = h / G;
            for (long kk = 0; kk < S; ++kk) {
                int ok = kk <= t;
                if (ok && block_mask) ok = block_mask[(t / blk) * nkb + kk / blk] != 0;
                key_ok[kk] = (uint8_t)ok;
            }
            const uint16_t *q_row = q + ((b * S + t) * Hq + h) * (long)D;
            const uint16_t *kb = k + (b * (long)S * Hkv + kvh) * (long)D;
            const uint16_t *vb = v + (b * (long)S * Hkv + kvh) * (long)D;
            attend_one_row(q_row, kb, vb, (long)Hkv * D, D, S, key_ok, scale,
                           scores, out + r * (long)D, lse ? lse + r : NULL);
        }
        free(scores);
        free(key_ok);
    }
    return bad ? -1 : 0;
}

/*
 * Decode: one query token per sequence, at position L-1 where L = seqlens[b]
 * (the cache holds L tokens including the current one).
 *   q: [B, Hq, D];  kc, vc: [B, Lmax, Hkv, D];  out: [B, Hq, D]; lse: [B, Hq]
 *   key_block_ok: NULL for full attention over keys 0..L-1, else per batch
 *                 element a row of nkb = ceil(Lmax/blk) flags: key k is
 *                 allowed iff k <= L-1 and key_block_ok[b*nkb + k/blk] != 0.
 */
int oracle_decode(const uint16_t *q, const uint16_t *kc, const uint16_t *vc,
                  const int32_t *seqlens, int B, int Lmax, int Hq, int Hkv,
                  int D, double scale, const uint8_t *key_block_ok, int blk,
                  double *out, double *lse)
{
    if (D <= 0 || D > 512 || Hkv <= 0 || Hq % Hkv != 0 || Lmax <= 0 || B <= 0)
        return -1;
    if (key_block_ok && blk <= 0) return -1;
    for (int b = 0; b < B; ++b)
        if (seqlens[b] < 1 || seqlens[b] > Lmax) return -1;
    const int G = Hq / Hkv;
    const long nkb = key_block_ok ? (Lmax + blk - 1) / blk : 0;

#pragma omp parallel
    {
        double *scores = (double *)malloc(sizeof(double) * (size_t)Lmax);
        uint8_t *key_ok = (uint8_t *)malloc((size_t)Lmax);
#pragma omp for schedule(dynamic, 1)
        for (long bh = 0; bh < (long)B * Hq; ++bh) {
            const long b = bh / Hq, h = bh % Hq, kvh = h / G;
            const long L = seqlens[b];
            for (long kk = 0; kk < L; ++kk) {
                int ok = 1;
                if (key_block_ok) ok = key_block_ok[b * nkb + kk / blk] != 0;
                key_ok[kk] = (uint8_t)ok;
            }
            const uint16_t *q_row = q + (b * Hq + h) * (long)D;
            const uint16_t *kb = kc + (b * (long)Lmax * Hkv + kvh) * (long)D;
            const uint16_t *vb = vc + (b * (long)Lmax * Hkv + kvh) * (long)D;
            attend_one_row(q_row, kb, vb, (long)Hkv * D, D, L, key_ok, scale,
                           scores, out + bh * (long)D, lse ? lse + bh : NULL);
        }
        free(scores);
        free(key_ok);
    }
    return 0;
}

/* Number of OpenMP threads the calls above use (for the baseline report). */
int oracle_num_threads(void)
{
    int n = 1;
#pragma omp parallel
    {
#pragma omp single
        {
#ifdef _OPENMP
            extern int omp_get_num_threads(void);
            n = omp_get_num_threads();
#endif
        }
    }
    return n;
}
