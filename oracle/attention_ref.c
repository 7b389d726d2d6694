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

/*
 * Gradients (reverse-mode chain rule through the definition above).  With
 * an upstream gradient dO_t of the output row o_t:
 *
 *   dV_k  += p_k dO_t                       (o_t = sum_k p_k v_k)
 *   dp_k   = dO_t . v_k
 *   ds_k   = p_k (dp_k - sum_j p_j dp_j)    (Jacobian of the row softmax)
 *   dQ_t   = scale * sum_k ds_k k_k         (s_k = scale * q_t . k_k)
 *   dK_k  += scale * ds_k q_t
 *
 * backward_row() fills p[] and ds[] of one query row over its allowed keys;
 * the three entry points below accumulate what they are asked for.
 */
static void backward_row(const uint16_t *q_row, const uint16_t *do_row,
                         const uint16_t *kbase, const uint16_t *vbase,
                         long kv_row_stride, int D, long n_keys,
                         const uint8_t *key_ok, double scale, double *p,
                         double *ds)
{
    double q[512], go[512];
    for (int d = 0; d < D; ++d) {
        q[d] = bf16_bits_to_double(q_row[d]);
        go[d] = bf16_bits_to_double(do_row[d]);
    }
    double M = -INFINITY;
    for (long k = 0; k < n_keys; ++k) {
        p[k] = 0.0;
        ds[k] = 0.0;
        if (!key_ok[k]) continue;
        const uint16_t *kr = kbase + k * kv_row_stride;
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += q[d] * bf16_bits_to_double(kr[d]);
        p[k] = dot * scale; /* the score, for now */
        if (p[k] > M) M = p[k];
    }
    if (M == -INFINITY) return; /* no key: output 0, all gradients 0 */
    double denom = 0.0;
    for (long k = 0; k < n_keys; ++k) {
        if (!key_ok[k]) continue;
        p[k] = exp(p[k] - M);
        denom += p[k];
    }
    double pdp = 0.0; /* sum_j p_j dp_j */
    for (long k = 0; k < n_keys; ++k) {
        if (!key_ok[k]) continue;
        p[k] /= denom;
        const uint16_t *vr = vbase + k * kv_row_stride;
        double dp = 0.0;
        for (int d = 0; d < D; ++d) dp += go[d] * bf16_bits_to_double(vr[d]);
        ds[k] = dp; /* dp, for now */
        pdp += p[k] * dp;
    }
    for (long k = 0; k < n_keys; ++k)
        if (key_ok[k]) ds[k] = p[k] * (ds[k] - pdp);
}

static void causal_key_flags(long t, long S, const uint8_t *block_mask, int blk,
                             long nkb, uint8_t *key_ok)
{
    for (long kk = 0; kk < S; ++kk) {
        int ok = kk <= t;
        if (ok && block_mask) ok = block_mask[(t / blk) * nkb + kk / blk] != 0;
        key_ok[kk] = (uint8_t)ok;
    }
}

/*
 * Full backward.  q, dout: [B, S, Hq, D]; k, v: [B, S, Hkv, D] (bf16 bits);
 * block_mask / blk as in oracle_attention_rows.  dq: [B, S, Hq, D],
 * dk, dv: [B, S, Hkv, D], fp64, overwritten.  A key/value head's gradient
 * sums the contributions of all G query heads that read it.
 */
int oracle_attention_backward(const uint16_t *q, const uint16_t *k,
                              const uint16_t *v, const uint16_t *dout, int B,
                              int S, int Hq, int Hkv, int D, double scale,
                              const uint8_t *block_mask, int blk, double *dq,
                              double *dk, double *dv)
{
    if (D <= 0 || D > 512 || Hkv <= 0 || Hq % Hkv != 0 || S <= 0 || B <= 0)
        return -1;
    if (block_mask && blk <= 0) return -1;
    const int G = Hq / Hkv;
    const long nkb = block_mask ? (S + blk - 1) / blk : 0;
    const long kvs = (long)Hkv * D;

#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * (size_t)S);
        double *ds = (double *)malloc(sizeof(double) * (size_t)S);
        uint8_t *key_ok = (uint8_t *)malloc((size_t)S);
        /* one task per (batch, kv head): it owns that head's dK and dV */
#pragma omp for schedule(dynamic, 1)
        for (long bk = 0; bk < (long)B * Hkv; ++bk) {
            const long b = bk / Hkv, kvh = bk % Hkv;
            const uint16_t *kb = k + (b * (long)S * Hkv + kvh) * (long)D;
            const uint16_t *vb = v + (b * (long)S * Hkv + kvh) * (long)D;
            double *dkb = dk + (b * (long)S * Hkv + kvh) * (long)D;
            double *dvb = dv + (b * (long)S * Hkv + kvh) * (long)D;
            for (long kk = 0; kk < S; ++kk)
                for (int d = 0; d < D; ++d) dkb[kk * kvs + d] = dvb[kk * kvs + d] = 0.0;
            for (int g = 0; g < G; ++g) {
                const long h = kvh * G + g;
                for (long t = 0; t < S; ++t) {
                    const long row = (b * S + t) * Hq + h;
                    causal_key_flags(t, S, block_mask, blk, nkb, key_ok);
                    backward_row(q + row * D, dout + row * D, kb, vb, kvs, D, S,
                                 key_ok, scale, p, ds);
                    double *dqr = dq + row * D;
                    for (int d = 0; d < D; ++d) dqr[d] = 0.0;
                    for (long kk = 0; kk <= t; ++kk) {
                        if (!key_ok[kk]) continue;
                        for (int d = 0; d < D; ++d) {
                            dqr[d] += scale * ds[kk] * bf16_bits_to_double(kb[kk * kvs + d]);
                            dkb[kk * kvs + d] +=
                                scale * ds[kk] * bf16_bits_to_double(q[row * D + d]);
                            dvb[kk * kvs + d] +=
                                p[kk] * bf16_bits_to_double(dout[row * D + d]);
                        }
                    }
                }
            }
        }
        free(p);
        free(ds);
        free(key_ok);
    }
    return 0;
}

/*
 * dQ of selected query rows (b, h, t) only: each needs its own row alone.
 * dq: [n_rows, D] fp64.
 */
int oracle_attention_backward_qrows(const uint16_t *q, const uint16_t *k,
                                    const uint16_t *v, const uint16_t *dout,
                                    int B, int S, int Hq, int Hkv, int D,
                                    double scale, const uint8_t *block_mask,
                                    int blk, const int64_t *rows, long n_rows,
                                    double *dq)
{
    if (D <= 0 || D > 512 || Hkv <= 0 || Hq % Hkv != 0 || S <= 0 || B <= 0)
        return -1;
    if (block_mask && blk <= 0) return -1;
    const int G = Hq / Hkv;
    const long nkb = block_mask ? (S + blk - 1) / blk : 0;
    const long kvs = (long)Hkv * D;
    int bad = 0;

#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * (size_t)S);
        double *ds = (double *)malloc(sizeof(double) * (size_t)S);
        uint8_t *key_ok = (uint8_t *)malloc((size_t)S);
#pragma omp for schedule(dynamic, 4)
        for (long r = 0; r < n_rows; ++r) {
            const long b = rows[3 * r + 0], h = rows[3 * r + 1], t = rows[3 * r + 2];
            if (b < 0 || b >= B || h < 0 || h >= Hq || t < 0 || t >= S) {
                bad = 1;
                continue;
            }
            const long kvh = h / G, row = (b * S + t) * Hq + h;
            const uint16_t *kb = k + (b * (long)S * Hkv + kvh) * (long)D;
            const uint16_t *vb = v + (b * (long)S * Hkv + kvh) * (long)D;
            causal_key_flags(t, S, block_mask, blk, nkb, key_ok);
            backward_row(q + row * D, dout + row * D, kb, vb, kvs, D, S, key_ok,
                         scale, p, ds);
            double *dqr = dq + r * (long)D;
            for (int d = 0; d < D; ++d) dqr[d] = 0.0;
            for (long kk = 0; kk <= t; ++kk)
                if (key_ok[kk])
                    for (int d = 0; d < D; ++d)
                        dqr[d] += scale * ds[kk] * bf16_bits_to_double(kb[kk * kvs + d]);
        }
        free(p);
        free(ds);
        free(key_ok);
    }
    return bad ? -1 : 0;
}

/*
 * dK and dV of selected key rows of one (batch b, kv head kvh): every query
 * row of the G heads that read this kv head contributes, so each of those
 * rows is evaluated in full; only the requested keys are accumulated.
 * keys: n_keys positions; dk, dv: [n_keys, D] fp64.
 */
int oracle_attention_backward_keyrows(const uint16_t *q, const uint16_t *k,
                                      const uint16_t *v, const uint16_t *dout,
                                      int B, int S, int Hq, int Hkv, int D,
                                      double scale, const uint8_t *block_mask,
                                      int blk, int b, int kvh,
                                      const int64_t *keys, long n_keys,
                                      double *dk, double *dv)
{
    if (D <= 0 || D > 512 || Hkv <= 0 || Hq % Hkv != 0 || S <= 0 || B <= 0)
        return -1;
    if (block_mask && blk <= 0) return -1;
    if (b < 0 || b >= B || kvh < 0 || kvh >= Hkv) return -1;
    for (long i = 0; i < n_keys; ++i)
        if (keys[i] < 0 || keys[i] >= S) return -1;
    const int G = Hq / Hkv;
    const long nkb = block_mask ? (S + blk - 1) / blk : 0;
    const long kvs = (long)Hkv * D;
    const uint16_t *kb = k + ((long)b * S * Hkv + kvh) * (long)D;
    const uint16_t *vb = v + ((long)b * S * Hkv + kvh) * (long)D;
    for (long i = 0; i < n_keys * D; ++i) dk[i] = dv[i] = 0.0;

#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * (size_t)S);
        double *ds = (double *)malloc(sizeof(double) * (size_t)S);
        uint8_t *key_ok = (uint8_t *)malloc((size_t)S);
        double *dk_l = (double *)calloc((size_t)(n_keys * D), sizeof(double));
        double *dv_l = (double *)calloc((size_t)(n_keys * D), sizeof(double));
#pragma omp for schedule(dynamic, 8)
        for (long gt = 0; gt < (long)G * S; ++gt) {
            const long h = (long)kvh * G + gt / S, t = gt % S;
            const long row = ((long)b * S + t) * Hq + h;
            causal_key_flags(t, S, block_mask, blk, nkb, key_ok);
            int any = 0;
            for (long i = 0; i < n_keys; ++i) any |= key_ok[keys[i]];
            if (!any) continue;
            backward_row(q + row * D, dout + row * D, kb, vb, kvs, D, S, key_ok,
                         scale, p, ds);
            for (long i = 0; i < n_keys; ++i) {
                const long kk = keys[i];
                if (!key_ok[kk]) continue;
                for (int d = 0; d < D; ++d) {
                    dk_l[i * D + d] += scale * ds[kk] * bf16_bits_to_double(q[row * D + d]);
                    dv_l[i * D + d] += p[kk] * bf16_bits_to_double(dout[row * D + d]);
                }
            }
        }
#pragma omp critical
        for (long i = 0; i < n_keys * D; ++i) {
            dk[i] += dk_l[i];
            dv[i] += dv_l[i];
        }
        free(p);
        free(ds);
        free(key_ok);
        free(dk_l);
        free(dv_l);
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
