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
 * and, for the FP8 form of o_proj (end of this file), the e4m3 codes, the
 * dynamic per-token and 128 x 128 block quantisers and the block-scaled
 * product; the YaRN rotation of the rotary parts (section "rotary"), for
 * callers that pass q_pe and k_pe unrotated; and the up-projection of the
 * compressed KV latent into k_nope and v (section "latent").
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
static int attn_rows_impl(const uint16_t *q_nope, const uint16_t *q_pe,
                          const uint16_t *k_nope, const uint16_t *k_pe,
                          const uint16_t *v, const uint16_t *mask,
                          int64_t mask_ld, int B, int H, int T, int Dn, int Dr,
                          int Dv, double scale, const int64_t *row_b,
                          const int64_t *row_i, int64_t nrows, double *out,
                          double *probs, uint8_t *fully_masked,
                          const int64_t *pos, const double *inv_freq,
                          double attn_factor, const double *k_nope_f64,
                          const double *v_f64);

int mla_oracle_attn_rows(const uint16_t *q_nope, const uint16_t *q_pe,
                         const uint16_t *k_nope, const uint16_t *k_pe,
                         const uint16_t *v, const uint16_t *mask,
                         int64_t mask_ld, int B, int H, int T, int Dn, int Dr,
                         int Dv, double scale, const int64_t *row_b,
                         const int64_t *row_i, int64_t nrows, double *out,
                         double *probs, uint8_t *fully_masked)
{
    return attn_rows_impl(q_nope, q_pe, k_nope, k_pe, v, mask, mask_ld, B, H, T,
                          Dn, Dr, Dv, scale, row_b, row_i, nrows, out, probs,
                          fully_masked, NULL, NULL, 1.0, NULL, NULL);
}

/* ================================================================ rotary
 *
 * The rotary parts are rotated right before the query and key are assembled
 * (page "Kimi K2 · Mix and project", excerpt modeling_deepseek.py 799-840:
 * cos, sin = self.rotary_emb(...); apply_rotary_pos_emb(q_pe, k_pe, cos, sin,
 * position_ids)). The pages print neither function's body. What they do
 * print is the configuration (page "Kimi K2 · Block input", config.json):
 * qk_rope_head_dim 64, rope_theta 50000, rope_scaling {type yarn, factor 32,
 * original_max_position_embeddings 4096, beta_fast 1, beta_slow 1, mscale 1,
 * mscale_all_dim 1}. The readings taken here, from the published YaRN method
 * (Peng et al., "YaRN: Efficient Context Window Extension of Large Language
 * Models", 2023: NTK-by-parts interpolation plus an attention factor):
 *
 * - Pair i (i < Dr/2) of a rotary vector is its elements 2i and 2i+1, rotated
 *   as one complex number by the angle position * inv_freq[i]:
 *     out[2i]   = f * (x[2i] cos a - x[2i+1] sin a)
 *     out[2i+1] = f * (x[2i+1] cos a + x[2i] sin a)
 *   with f the attention factor below. (An implementation may store the
 *   rotated pair elsewhere in the vector, e.g. first halves then second
 *   halves; as long as query and key are stored alike, every score is the
 *   same number.)
 * - The base frequencies are theta^(-2i/Dr). YaRN keeps them (extrapolation)
 *   for the fast-rotating pairs and divides them by `factor` (interpolation)
 *   for the slow ones, with a linear ramp between two pair indices:
 *     d(n)  = Dr * ln(L / (2 pi n)) / (2 ln theta)     (L = original max positions;
 *             the pair index that turns n times over L positions)
 *     low   = max(floor(d(beta_fast)), 0), high = min(ceil(d(beta_slow)), Dr - 1)
 *             (high = low + 0.001 when they coincide)
 *     ramp  = clamp((i - low) / (high - low), 0, 1)
 *     inv_freq[i] = theta^(-2i/Dr) * ((1 - ramp) + ramp / factor)
 *   With the printed values (beta_fast = beta_slow = 1) low = 19, high = 20:
 *   pairs 0..19 keep their frequency, pairs 20..31 are divided by 32.
 * - The attention factor multiplies cos and sin:
 *     f = m(factor, mscale) / m(factor, mscale_all_dim),
 *     m(s, k) = 1 if s <= 1 else 0.1 k ln(s) + 1,
 *   which is exactly 1 for the printed mscale = mscale_all_dim = 1.
 * - Query and key rotate with the same position_ids (the excerpt passes one
 *   position_ids to apply_rotary_pos_emb); without them positions are 0..T-1.
 */

int mla_oracle_yarn_inv_freq(int Dr, double theta, double factor,
                             double orig_max_pos, double beta_fast,
                             double beta_slow, double *inv_freq)
{
    if (Dr < 2 || (Dr & 1) || !(theta > 1.0) || !(factor > 0.0) ||
        !(orig_max_pos > 0.0) || !(beta_fast > 0.0) || !(beta_slow > 0.0) ||
        !inv_freq)
        return -1;
    const double two_pi = 2.0 * acos(-1.0);
    const double d_fast = Dr * log(orig_max_pos / (two_pi * beta_fast)) / (2.0 * log(theta));
    const double d_slow = Dr * log(orig_max_pos / (two_pi * beta_slow)) / (2.0 * log(theta));
    double low = floor(d_fast), high = ceil(d_slow);
    if (low < 0.0) low = 0.0;
    if (high > Dr - 1) high = Dr - 1;
    if (high == low) high += 0.001;
    for (int i = 0; i < Dr / 2; ++i) {
        const double base = pow(theta, -2.0 * i / Dr);
        double ramp = (i - low) / (high - low);
        if (ramp < 0.0) ramp = 0.0;
        if (ramp > 1.0) ramp = 1.0;
        inv_freq[i] = base * (1.0 - ramp) + (base / factor) * ramp;
    }
    return 0;
}

static double yarn_m(double s, double k)
{
    return s <= 1.0 ? 1.0 : 0.1 * k * log(s) + 1.0;
}

double mla_oracle_yarn_attn_factor(double factor, double mscale, double mscale_all_dim)
{
    return yarn_m(factor, mscale) / yarn_m(factor, mscale_all_dim);
}

/* Rotate one rotary vector of Dr bf16 values at position p (double out). */
static void rotate_row(const uint16_t *x, int Dr, int64_t p, const double *inv_freq,
                       double f, double *out)
{
    for (int i = 0; i < Dr / 2; ++i) {
        const double a = (double)p * inv_freq[i];
        const double c = f * cos(a), sn = f * sin(a);
        const double x0 = bf16_bits_to_double(x[2 * i]);
        const double x1 = bf16_bits_to_double(x[2 * i + 1]);
        out[2 * i] = x0 * c - x1 * sn;
        out[2 * i + 1] = x1 * c + x0 * sn;
    }
}

/* Rotated copies of n rotary vectors x [n, Dr] at positions pos[n]. */
int mla_oracle_rope_rotate(const uint16_t *x, int64_t n, int Dr, const int64_t *pos,
                           const double *inv_freq, double attn_factor, double *out)
{
    if (n < 0 || Dr < 2 || (Dr & 1) || (n > 0 && (!x || !pos || !inv_freq || !out)))
        return -1;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; ++r)
        rotate_row(x + r * Dr, Dr, pos[r], inv_freq, attn_factor, out + r * Dr);
    return 0;
}

/*
 * mla_oracle_attn_rows with the rotary parts given unrotated: q_pe and k_pe
 * are rotated here (as above) at positions pos [B, T] before the scores.
 */
int mla_oracle_attn_rows_rope(const uint16_t *q_nope, const uint16_t *q_pe,
                              const uint16_t *k_nope, const uint16_t *k_pe,
                              const uint16_t *v, const uint16_t *mask,
                              int64_t mask_ld, int B, int H, int T, int Dn, int Dr,
                              int Dv, double scale, const int64_t *pos,
                              const double *inv_freq, double attn_factor,
                              const int64_t *row_b, const int64_t *row_i,
                              int64_t nrows, double *out, double *probs,
                              uint8_t *fully_masked)
{
    if (!pos || !inv_freq || Dr < 2 || (Dr & 1)) return -1;
    return attn_rows_impl(q_nope, q_pe, k_nope, k_pe, v, mask, mask_ld, B, H, T,
                          Dn, Dr, Dv, scale, row_b, row_i, nrows, out, probs,
                          fully_masked, pos, inv_freq, attn_factor, NULL, NULL);
}

/* ================================================================ latent
 *
 * The non-rotary key parts and the values come from the compressed KV
 * latent: config.json (page "Kimi K2 · Block input") gives kv_lora_rank 512,
 * num_attention_heads 64, qk_nope_head_dim 128, v_head_dim 128 and
 * attention_bias false, and the excerpt of page "Kimi K2 · Mix and project"
 * starts from per-head k_nope and value_states. The pages print nothing in
 * between; the reading taken here is the plain linear up-projection, one
 * bias-free nn.Linear(512 -> 64 * (128 + 128)) applied to each token's
 * latent:
 *   kv[b,t,n] = sum_{c<R} c_kv[b,t,c] * W[n,c]                  (W [H*(Dn+Dv), R])
 *   k_nope[b,h,t,e] = kv[b,t,h*(Dn+Dv) + e]          (e < Dn)
 *   v[b,h,t,e]      = kv[b,t,h*(Dn+Dv) + Dn + e]     (e < Dv)
 * i.e. the output is viewed per head as Dn + Dv values, the non-rotary key
 * part first, then the value.
 */

/* k_nope [B,H,T,Dn] and v [B,H,T,Dv] (double) from c_kv [B,T,R] and W. */
int mla_oracle_kv_up(const uint16_t *c_kv, const uint16_t *W, int B, int T, int R,
                     int H, int Dn, int Dv, double *k_nope, double *v)
{
    if (B < 1 || T < 1 || R < 1 || H < 1 || Dn < 0 || Dv < 1 || !c_kv || !W || !v ||
        (Dn > 0 && !k_nope))
        return -1;
    const int per_head = Dn + Dv;
    const int64_t work = (int64_t)B * T * H;
#pragma omp parallel for schedule(static)
    for (int64_t w = 0; w < work; ++w) {
        const int64_t bt = w / H;
        const int h = (int)(w % H);
        const int64_t b = bt / T, t = bt % T;
        const uint16_t *x = c_kv + bt * R;
        for (int n = 0; n < per_head; ++n) {
            const uint16_t *wrow = W + ((int64_t)h * per_head + n) * R;
            double acc = 0.0;
            for (int c = 0; c < R; ++c)
                acc += bf16_bits_to_double(x[c]) * bf16_bits_to_double(wrow[c]);
            if (n < Dn)
                k_nope[((b * H + h) * T + t) * Dn + n] = acc;
            else
                v[((b * H + h) * T + t) * Dv + (n - Dn)] = acc;
        }
    }
    return 0;
}

/*
 * Attention whose non-rotary keys and values are given in double (the
 * up-projection's exact result above) instead of bf16; q_pe, k_pe as in
 * mla_oracle_attn_rows (rotated).
 */
int mla_oracle_attn_rows_kv64(const uint16_t *q_nope, const uint16_t *q_pe,
                              const double *k_nope, const uint16_t *k_pe,
                              const double *v, const uint16_t *mask,
                              int64_t mask_ld, int B, int H, int T, int Dn, int Dr,
                              int Dv, double scale, const int64_t *row_b,
                              const int64_t *row_i, int64_t nrows, double *out,
                              double *probs, uint8_t *fully_masked)
{
    if (!v || (Dn > 0 && !k_nope)) return -1;
    return attn_rows_impl(q_nope, q_pe, NULL, k_pe, NULL, mask, mask_ld, B, H, T,
                          Dn, Dr, Dv, scale, row_b, row_i, nrows, out, probs,
                          fully_masked, NULL, NULL, 1.0, k_nope, v);
}

static int attn_rows_impl(const uint16_t *q_nope, const uint16_t *q_pe,
                          const uint16_t *k_nope, const uint16_t *k_pe,
                          const uint16_t *v, const uint16_t *mask,
                          int64_t mask_ld, int B, int H, int T, int Dn, int Dr,
                          int Dv, double scale, const int64_t *row_b,
                          const int64_t *row_i, int64_t nrows, double *out,
                          double *probs, uint8_t *fully_masked,
                          const int64_t *pos, const double *inv_freq,
                          double attn_factor, const double *k_nope_f64,
                          const double *v_f64)
{
    if (B < 1 || H < 1 || T < 1 || Dn < 0 || Dr < 0 || Dv < 1 || nrows < 0)
        return -1;
    if (!q_nope && Dn > 0) return -1;
    if (!k_nope && !k_nope_f64 && Dn > 0) return -1;
    if (!q_pe && Dr > 0) return -1;
    if (!k_pe && Dr > 0) return -1;
    if ((!v && !v_f64) || !out || (nrows > 0 && (!row_b || !row_i))) return -1;
    if (mask && mask_ld < T) return -1;
    for (int64_t r = 0; r < nrows; ++r)
        if (row_b[r] < 0 || row_b[r] >= B || row_i[r] < 0 || row_i[r] >= T)
            return -1;

    /* the shared rotary key, rotated once for every (b, j) when rotating */
    double *k_rot = NULL;
    if (pos && Dr > 0) {
        k_rot = (double *)malloc(sizeof(double) * (size_t)B * (size_t)T * (size_t)Dr);
        if (!k_rot) return -2;
        mla_oracle_rope_rotate(k_pe, (int64_t)B * T, Dr, pos, inv_freq, attn_factor, k_rot);
    }

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
            if (k_rot)
                rotate_row(q_pe + (bh * T + i) * Dr, Dr, pos[b * T + i], inv_freq,
                           attn_factor, qv + Dn);
            else
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
                    if (k_nope_f64)
                        for (int d = 0; d < Dn; ++d)
                            dot += qv[d] * k_nope_f64[(bh * T + j) * Dn + d];
                    else
                        for (int d = 0; d < Dn; ++d)
                            dot += qv[d] * bf16_bits_to_double(k_nope[(bh * T + j) * Dn + d]);
                    if (k_rot)
                        for (int d = 0; d < Dr; ++d)
                            dot += qv[Dn + d] * k_rot[(b * T + j) * Dr + d];
                    else
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
                if (v_f64) {
                    const double *vrow = v_f64 + (bh * T + j) * Dv;
                    for (int e = 0; e < Dv; ++e) acc[e] += p * vrow[e];
                } else {
                    const uint16_t *vrow = v + (bh * T + j) * Dv;
                    for (int e = 0; e < Dv; ++e)
                        acc[e] += p * bf16_bits_to_double(vrow[e]);
                }
            }
            for (int e = 0; e < Dv; ++e) orow[e] = acc[e];
        }
        free(s);
        free(qv);
        free(acc);
    }
    free(k_rot);
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

/* ================================================================ FP8 o_proj
 *
 * The checkpoint stores its projection weights as 8-bit floats (page "Kimi
 * K2 · Transformer blocks", configuration excerpt moonshotai/Kimi-K2-Instruct
 * config.json, quantization_config: quant_method fp8, fmt e4m3,
 * activation_scheme dynamic, weight_block_size [128, 128]). The page gives
 * those four fields and nothing more; the readings taken here:
 *
 * - e4m3 is the 8-bit float with 1 sign bit, 4 exponent bits (bias 7) and 3
 *   mantissa bits: exponent field 0 holds the subnormals m * 2^-9, fields
 *   1..15 hold (1 + m/8) * 2^(e-7), there are no infinities, and the two
 *   codes with every exponent and mantissa bit set are NaN. The largest
 *   finite value is 448.
 * - weight_block_size [128, 128]: one fp32 scale per 128 x 128 block of
 *   W_o [N, K], and W_o[n,k] ~= value(code[n,k]) * scale[n/128][k/128].
 * - activation_scheme dynamic: the activations' scales are computed from the
 *   data at run time, one per token and per 128-wide group of input
 *   features (the weight block's extent along K).
 * - A group's scale is amax / 448 in fp32 (1 for a group of zeros), and each
 *   element's code is the e4m3 value nearest to x / scale, computed in fp32,
 *   ties to the even code, magnitudes above 448 saturating to 448.
 *
 * The product is then, with a_s[g][m] the activation scales and w_s[j][g]
 * the weight scales,
 *   out[m,n] = sum_g a_s[g][m] * w_s[n/128][g]
 *                    * sum_{k in group g} value(qa[m,k]) * value(qw[n,k]).
 * Each group's inner sum is exact in double (the products of two e4m3
 * values have at most 8 significant bits and span less than 2^40).
 */

#define FP8_GROUP 128
#define E4M3_MAX 448.0

/* Value of an e4m3 code, from the bit fields (NaN for the two NaN codes). */
static double e4m3_value(uint8_t c)
{
    const int sign = c >> 7;
    const int e = (c >> 3) & 15;
    const int m = c & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -v : v;
}

double mla_oracle_e4m3_decode(uint8_t c) { return e4m3_value(c); }

/*
 * Code of the e4m3 value nearest to y: bisection over the non-negative finite
 * codes 0..126 (their values increase with the code), ties to the code whose
 * mantissa is even, |y| > 448 saturating to 448, the sign bit copied from y
 * (so -0 and negatives that round to zero give 0x80).
 */
uint8_t mla_oracle_e4m3_encode(float y)
{
    const uint8_t sign = signbit(y) ? 0x80 : 0x00;
    if (isnan(y))
        return (uint8_t)(sign | 0x7F);
    const double a = fabs((double)y);
    if (a >= E4M3_MAX)
        return (uint8_t)(sign | 0x7E);
    /* largest code lo with value(lo) <= a */
    int lo = 0, hi = 126;
    while (lo < hi) {
        const int mid = (lo + hi + 1) / 2;
        if (e4m3_value((uint8_t)mid) <= a)
            lo = mid;
        else
            hi = mid - 1;
    }
    uint8_t c = (uint8_t)lo;
    if (lo < 126) {
        const double below = a - e4m3_value((uint8_t)lo);
        const double above = e4m3_value((uint8_t)(lo + 1)) - a;
        if (above < below || (above == below && (lo & 1)))
            c = (uint8_t)(lo + 1);
    }
    return (uint8_t)(sign | c);
}

/* Scale of a group whose largest magnitude is amax (fp32 arithmetic). */
static float group_scale(float amax)
{
    return amax > 0.0f ? amax / 448.0f : 1.0f;
}

static float bf16_bits_to_float(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Codes of one group of n bf16 values at x (stride 1) with its scale. */
static float quant_group(const uint16_t *x, int n, uint8_t *q)
{
    float amax = 0.0f;
    for (int i = 0; i < n; ++i) {
        const float a = fabsf(bf16_bits_to_float(x[i]));
        if (a > amax)
            amax = a;
    }
    const float s = group_scale(amax);
    for (int i = 0; i < n; ++i) {
        const float y = bf16_bits_to_float(x[i]) / s;
        q[i] = mla_oracle_e4m3_encode(y);
    }
    return s;
}

/*
 * Dynamic activation quantisation: x [M, K] bf16 bits (row-major) ->
 * q [M, K] e4m3 codes and scale [K/128][M] (group-major). Returns -1 on an
 * argument error.
 */
int mla_oracle_quant_rows_fp8(const uint16_t *x, int64_t M, int K, uint8_t *q, float *scale)
{
    if (!x || !q || !scale || M < 1 || K < FP8_GROUP || K % FP8_GROUP != 0)
        return -1;
    const int G = K / FP8_GROUP;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int g = 0; g < G; ++g) {
            const int64_t off = m * (int64_t)K + (int64_t)g * FP8_GROUP;
            scale[(int64_t)g * M + m] = quant_group(x + off, FP8_GROUP, q + off);
        }
    return 0;
}

/*
 * Block weight quantisation: W [N, K] bf16 bits -> q [N, K] e4m3 codes and
 * scale [N/128][K/128]. Returns -1 on an argument error.
 */
int mla_oracle_quant_weight_fp8(const uint16_t *W, int N, int K, uint8_t *q, float *scale)
{
    if (!W || !q || !scale || N < FP8_GROUP || K < FP8_GROUP || N % FP8_GROUP != 0 ||
        K % FP8_GROUP != 0)
        return -1;
    const int NB = N / FP8_GROUP, KB = K / FP8_GROUP;
#pragma omp parallel for schedule(static)
    for (int64_t blk = 0; blk < (int64_t)NB * KB; ++blk) {
        const int nb = (int)(blk / KB), kb = (int)(blk % KB);
        float amax = 0.0f;
        for (int r = 0; r < FP8_GROUP; ++r) {
            const uint16_t *row = W + (int64_t)(nb * FP8_GROUP + r) * K + kb * FP8_GROUP;
            for (int i = 0; i < FP8_GROUP; ++i) {
                const float a = fabsf(bf16_bits_to_float(row[i]));
                if (a > amax)
                    amax = a;
            }
        }
        const float s = group_scale(amax);
        scale[blk] = s;
        for (int r = 0; r < FP8_GROUP; ++r) {
            const int64_t off = (int64_t)(nb * FP8_GROUP + r) * K + kb * FP8_GROUP;
            for (int i = 0; i < FP8_GROUP; ++i)
                q[off + i] = mla_oracle_e4m3_encode(bf16_bits_to_float(W[off + i]) / s);
        }
    }
    return 0;
}

/*
 * The block-scaled product for a list of rows:
 *   out[r, n] = sum_g a_s[g][rows[r]] * w_s[n/128][g]
 *                     * sum_{k in g} value(qa[rows[r], k]) * value(qw[n, k])
 * qa [M, K] codes with a_scale [K/128][M]; qw [N, K] codes with
 * w_scale [N/128][K/128]; out [nrows, N] double. Returns -1 on an argument
 * error.
 */
int mla_oracle_oproj_fp8_rows(const uint8_t *qa, const float *a_scale, int64_t M,
                              const int64_t *rows, int64_t nrows, const uint8_t *qw,
                              const float *w_scale, int N, int K, double *out)
{
    if (!qa || !a_scale || !rows || !qw || !w_scale || !out || M < 1 || nrows < 0 ||
        N < FP8_GROUP || K < FP8_GROUP || N % FP8_GROUP != 0 || K % FP8_GROUP != 0)
        return -1;
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= M)
            return -1;
    double value[256];
    for (int c = 0; c < 256; ++c)
        value[c] = e4m3_value((uint8_t)c);
    const int G = K / FP8_GROUP;
    const int64_t work = nrows * (int64_t)N;
#pragma omp parallel for schedule(static)
    for (int64_t w = 0; w < work; ++w) {
        const int64_t r = w / N;
        const int n = (int)(w % N);
        const int64_t m = rows[r];
        const uint8_t *arow = qa + m * (int64_t)K;
        const uint8_t *wrow = qw + (int64_t)n * K;
        double acc = 0.0;
        for (int g = 0; g < G; ++g) {
            double block = 0.0;
            for (int i = 0; i < FP8_GROUP; ++i) {
                const int k = g * FP8_GROUP + i;
                block += value[arow[k]] * value[wrow[k]];
            }
            acc += (double)a_scale[(int64_t)g * M + m] *
                   (double)w_scale[(int64_t)(n / FP8_GROUP) * G + g] * block;
        }
        out[w] = acc;
    }
    return 0;
}
