/*
 * mla_oracle.c -- plain fp64 CPU oracle for the MLA prefill core and its
 * output projection.
 *
 * TEST INFRASTRUCTURE ONLY. The product library never links, loads or calls
 * this file; only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do. It shares no code, header or constant with the CUDA kernels.
 *
 * What it computes (page "Kimi K2 · Mix and project", code excerpts
 * modeling_deepseek.py 799-840 and 848-852):
 *
 *   for every batch b, head h and query row i:
 *     s_ij = scale * ( sum_{d<Dn} q_nope[b,h,i,d] * k_nope[b,h,j,d]
 *                    + sum_{d<Dr} q_pe[b,h,i,d]   * k_pe[b,0,j,d] )
 *            + ( mask ? M[b,0,i,j] : (j <= i ? 0 : -inf) )
 *     p_ij = exp(s_ij - max_j s_ij) / sum_j exp(s_ij - max_j s_ij)
 *     attn[b,i,h*Dv + e] = sum_j p_ij * v[b,h,j,e]
 *   out[r,n] = sum_k attn[r,k] * W_o[n,k]            (no bias)
 *
 * - The query and key of every head are the concatenation of a non-rotary
 *   part and a rotary part; the key's rotary part is one tensor shared by all
 *   heads (the excerpt builds query_states / key_states that way, and the
 *   page's summary says the key's rotated part is the shared rotary key).
 *   The concatenation is written out here as the sum of the two partial dot
 *   products, which is the same number.
 * - The scale multiplies the matmul result; the mask is added afterwards
 *   (excerpt: "* self.softmax_scale", then "attn_weights + attention_mask").
 * - The softmax runs over the key axis (dim=-1).
 * - Heads are merged by transpose(1,2) + reshape, so column h*Dv+e holds
 *   head h, value dim e.
 * - o_proj is nn.Linear(H*Dv -> D, bias=False): out = attn . W_o^T with
 *   W_o stored [D, H*Dv] (out, in).
 *
 * Implementation choices, kept deliberately plain:
 * - Everything in double precision on the exact bf16 input values (the
 *   bf16 -> double widening is exact). No intermediate rounding.
 * - Two-pass exact softmax: all scores of a row first, then the max, then the
 *   exponentials and their sum, then the value mix. No tiling, no online
 *   rescaling.
 * - A row whose every score is -inf (possible only with an explicit mask) has
 *   no defined softmax; it is written as zeros and reported in fully_masked.
 * - Any subset of rows can be evaluated: row i of a batch depends only on
 *   query row i and on the keys/values (and mask row i), so a sampled row is
 *   exactly the corresponding row of the full result.
 * - Rows are spread over OpenMP threads; each (row, head) is independent.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* bf16 is the upper half of an IEEE binary32; widening it is exact. */
static double bf16_bits_to_double(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int mla_oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void mla_oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/*
 * Attention for a list of query rows.
 *
 * Inputs are bf16 bit patterns, contiguous:
 *   q_nope [B,H,T,Dn]  q_pe [B,H,T,Dr]  k_nope [B,H,T,Dn]
 *   k_pe   [B,1,T,Dr]  v    [B,H,T,Dv]
 *   mask   [B,1,T,mask_ld] (only the first T entries of a row are used) or NULL
 * scale is the softmax scale.
 * The rows to evaluate are (row_b[r], row_i[r]) for r < nrows.
 *
 * Outputs (double):
 *   out          [nrows, H*Dv]   merged head outputs of each requested row
 *   probs        [nrows, H, T]   the softmax row, or NULL to skip
 *   fully_masked [nrows, H]      1 where every key was -inf, or NULL
 *
 * Returns 0, or -1 on an argument error.
 */
int mla_oracle_attn_rows(const uint16_t *q_nope, const uint16_t *q_pe,
                         const uint16_t *k_nope, const uint16_t *k_pe,
                         const uint16_t *v, const uint16_t *mask,
                         int64_t mask_ld, int B, int H, int T, int Dn, int Dr,
                         int Dv, double scale, const int64_t *row_b,
                         const int64_t *row_i, int64_t nrows, double *out,
                         double *probs, uint8_t *fully_masked)
{
    if (B < 1 || H < 1 || T < 1 || Dn < 0 || Dr < 0 || Dv < 1 || nrows < 0)
        return -1;
    if (!q_nope && Dn > 0) return -1;
    if (!k_nope && Dn > 0) return -1;
    if (!q_pe && Dr > 0) return -1;
    if (!k_pe && Dr > 0) return -1;
    if (!v || !out || (nrows > 0 && (!row_b || !row_i))) return -1;
    if (mask && mask_ld < T) return -1;
    for (int64_t r = 0; r < nrows; ++r)
        if (row_b[r] < 0 || row_b[r] >= B || row_i[r] < 0 || row_i[r] >= T)
            return -1;

    const int64_t work = nrows * (int64_t)H;
    int bad_alloc = 0;

#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)T);
        double *qv = (double *)malloc(sizeof(double) * (size_t)(Dn + Dr + 1));
        double *acc = (double *)malloc(sizeof(double) * (size_t)Dv);
        if (!s || !qv || !acc) {
#pragma omp atomic write
            bad_alloc = 1;
        }
#pragma omp for schedule(dynamic, 4)
        for (int64_t w = 0; w < work; ++w) {
            if (!s || !qv || !acc) continue;
            /* consecutive work items share a head, so the threads stream the
               same keys and values */
            const int h = (int)(w / nrows);
            const int64_t r = w % nrows;
            const int64_t b = row_b[r];
            const int64_t i = row_i[r];
            const int64_t bh = b * H + h;

            /* the query row, non-rotary part then rotary part */
            for (int d = 0; d < Dn; ++d)
                qv[d] = bf16_bits_to_double(q_nope[(bh * T + i) * Dn + d]);
            for (int d = 0; d < Dr; ++d)
                qv[Dn + d] = bf16_bits_to_double(q_pe[(bh * T + i) * Dr + d]);

            /* pass 1: every score of the row, and its maximum */
            double smax = -INFINITY;
            for (int64_t j = 0; j < T; ++j) {
                double add;
                if (mask) {
                    add = bf16_bits_to_double(mask[(b * T + i) * mask_ld + j]);
                } else {
                    add = (j <= i) ? 0.0 : -INFINITY;
                }
                double sj;
                if (isinf(add) && add < 0) {
                    sj = -INFINITY;
                } else {
                    double dot = 0.0;
                    for (int d = 0; d < Dn; ++d)
                        dot += qv[d] * bf16_bits_to_double(k_nope[(bh * T + j) * Dn + d]);
                    for (int d = 0; d < Dr; ++d)
                        dot += qv[Dn + d] * bf16_bits_to_double(k_pe[(b * T + j) * Dr + d]);
                    sj = scale * dot + add;
                }
                s[j] = sj;
                if (sj > smax) smax = sj;
            }

            double *prow = probs ? probs + (r * H + h) * (int64_t)T : NULL;
            double *orow = out + r * (int64_t)H * Dv + (int64_t)h * Dv;
            if (isinf(smax) && smax < 0) {
                /* no key is allowed: the softmax is undefined */
                for (int e = 0; e < Dv; ++e) orow[e] = 0.0;
                if (prow)
                    for (int64_t j = 0; j < T; ++j) prow[j] = 0.0;
                if (fully_masked) fully_masked[r * H + h] = 1;
                continue;
            }
            if (fully_masked) fully_masked[r * H + h] = 0;

            /* pass 2: exponentials and their sum */
            double denom = 0.0;
            for (int64_t j = 0; j < T; ++j) {
                double e = (isinf(s[j]) && s[j] < 0) ? 0.0 : exp(s[j] - smax);
                s[j] = e;
                denom += e;
            }

            /* pass 3: normalised weights, then the value mix */
            for (int e = 0; e < Dv; ++e) acc[e] = 0.0;
            for (int64_t j = 0; j < T; ++j) {
                const double p = s[j] / denom;
                if (prow) prow[j] = p;
                if (p == 0.0) continue;
                const uint16_t *vrow = v + (bh * T + j) * Dv;
                for (int e = 0; e < Dv; ++e)
                    acc[e] += p * bf16_bits_to_double(vrow[e]);
            }
            for (int e = 0; e < Dv; ++e) orow[e] = acc[e];
        }
        free(s);
        free(qv);
        free(acc);
    }
    return bad_alloc ? -2 : 0;
}

/*
 * Output projection, nn.Linear without bias: out[r,n] = sum_k a[r,k] W[n,k].
 *   a [nrows, K] double, W [N, K] bf16 bits, out [nrows, N] double.
 * Page "Kimi K2 · Mix and project", excerpt modeling_deepseek.py 848-852
 * (o_proj applied to the merged heads) and the page's parameter table
 * (8,192 x 7,168 weights).
 */
int mla_oracle_oproj_rows(const double *a, const uint16_t *W, int64_t nrows,
                          int N, int K, double *out)
{
    if (nrows < 0 || N < 1 || K < 1 || !W || !out || (nrows > 0 && !a))
        return -1;
    const int64_t work = nrows * (int64_t)N;
#pragma omp parallel for schedule(static)
    for (int64_t w = 0; w < work; ++w) {
        const int64_t r = w / N;
        const int64_t n = w % N;
        const double *arow = a + r * (int64_t)K;
        const uint16_t *wrow = W + n * (int64_t)K;
        double acc = 0.0;
        for (int k = 0; k < K; ++k) acc += arow[k] * bf16_bits_to_double(wrow[k]);
        out[r * (int64_t)N + n] = acc;
    }
    return 0;
}
