/*
 * mla_oracle.c -- plain, slow, fp64 CPU oracle for Multi-head Latent Attention
 * (MLA) decode over a paged latent cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  The product path (the
 * CUDA library under head_latent_attention_10_b200/) never calls it and shares
 * no code, header, table or helper with it.
 *
 * What it computes, and where each step is stated:
 *
 *   DeepSeek-V2 paper review (jiphyeonjeon.kr), section 2, the basic linear
 *   forms:  c^KV_t = W^DKV h_t,  k^C_t = W^UK c^KV_t,  v^C_t = W^UV c^KV_t.
 *   DeepSeek-V3 report summary (xyznot.com), Method 1 (MLA):
 *           k^R_t = RoPE(W^KR h_t),  k_{t,i} = [k^C_{t,i}; k^R_t], and only
 *           c^KV_t and k^R_t are cached.
 *   DeepSeek-V2 paper review, section 3 (decoupled RoPE): per-head content
 *           query/key of 128 dims, per-head RoPE query of 64 dims, one RoPE key
 *           of 64 dims per token shared by all heads;
 *           l_ij = (q^C . k^C + q^R . k^R) / sqrt(128 + 64),
 *           a_ij = softmax_j(l_ij).
 *   DeepSeek-V2 paper review, section 2 (matrix absorption):
 *           (q^C)^T U^K c = ((U^K)^T q^C)^T c  and
 *           sum_j a_ij U^V c_j = U^V sum_j a_ij c_j,
 *           u_t = sum_i O_i U^V_i (sum_j a_ij c_j).
 *
 * mla_oracle_decode_expanded() is the textbook expanded form: it builds
 * k^C = U^K c and v^C = U^V c for every visible token and head, then runs a
 * max-subtracted softmax.  mla_oracle_decode_latent() is the absorbed form
 * (attention directly against the latent, value = latent); it exists so the
 * tests can check the absorption identity and the latent output of the decode
 * call on its own.
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *   - RoPE pairs adjacent elements (x_{2k}, x_{2k+1}) and rotates them by
 *     pos * base^(-2k/d_r); base 10000.
 *   - The token at logical position j of a sequence has RoPE position j.  The
 *     cache holds the raw (unrotated) RoPE key; the oracle rotates it here.
 *   - With s query tokens per sequence of length L, query t sees the cache
 *     positions j <= L - s + t.  A query with no visible key gives a zero
 *     output and lse = -inf.
 *   - Paged layout: logical position j of sequence b lives in physical block
 *     block_table[b*max_blocks + j/block_size], slot j % block_size; a row is
 *     [c^KV (d_c values) | k^R (d_r values)] in bf16.
 *
 * Inputs of bf16 storage are passed as uint16 bit patterns and widened to
 * double exactly; every other input and every output is double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double bf16_bits_to_f64(uint16_t v)
{
    uint32_t u = ((uint32_t)v) << 16;
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

/* RoPE of one d_r-vector at position pos: pair k = (x[2k], x[2k+1]) is turned
 * by the angle pos * theta_k, theta_k = base^(-2k/d_r). */
void mla_oracle_rope(const double *x, int d_r, double pos, double base, double *y)
{
    for (int k = 0; k < d_r / 2; ++k) {
        double theta = pow(base, -2.0 * (double)k / (double)d_r);
        double ang = pos * theta;
        double c = cos(ang), s = sin(ang);
        double x0 = x[2 * k], x1 = x[2 * k + 1];
        y[2 * k] = x0 * c - x1 * s;
        y[2 * k + 1] = x0 * s + x1 * c;
    }
}

/* RoPE of N rows x [N][d_r] at positions pos[N] (the cache's k^R part). */
void mla_oracle_rope_rows(int N, int d_r, const double *x, const int32_t *pos, double base,
                          double *y)
{
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n)
        mla_oracle_rope(x + (size_t)n * d_r, d_r, (double)pos[n], base, y + (size_t)n * d_r);
}

/* Append projection (step a1): for each of T tokens,
 *   c^KV = W^DKV h           (W^DKV: [d_c][d] row-major)
 *   k^R  = RoPE(W^KR h, pos) (W^KR : [d_r][d] row-major)
 * h: [T][d] bf16 bits; outputs c_out [T][d_c], kr_out [T][d_r]. */
void mla_oracle_kv_project(int T, int d, int d_c, int d_r,
                           const uint16_t *h, const uint16_t *w_dkv,
                           const uint16_t *w_kr, const int32_t *pos,
                           double rope_base, double *c_out, double *kr_out)
{
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        double *kr = (double *)malloc(sizeof(double) * (size_t)d_r);
        for (int r = 0; r < d_c; ++r) {
            double acc = 0.0;
            for (int k = 0; k < d; ++k)
                acc += bf16_bits_to_f64(w_dkv[(size_t)r * d + k]) *
                       bf16_bits_to_f64(h[(size_t)t * d + k]);
            c_out[(size_t)t * d_c + r] = acc;
        }
        for (int r = 0; r < d_r; ++r) {
            double acc = 0.0;
            for (int k = 0; k < d; ++k)
                acc += bf16_bits_to_f64(w_kr[(size_t)r * d + k]) *
                       bf16_bits_to_f64(h[(size_t)t * d + k]);
            kr[r] = acc;
        }
        mla_oracle_rope(kr, d_r, (double)pos[t], rope_base, kr_out + (size_t)t * d_r);
        free(kr);
    }
}

/* Query absorption (step a2): for token t and head i,
 *   out[t][i][0:d_c]       = (U^K_i)^T q^C_{t,i}     (U^K_i: [d_h][d_c])
 *   out[t][i][d_c:d_c+d_r] = RoPE(q^R_{t,i}, q_pos[t])   (copied if q_pos == NULL)
 * q_nope [T][H][d_h], q_rope [T][H][d_r], w_uk [H][d_h][d_c]. */
void mla_oracle_absorb_q(int T, int H, int d_h, int d_c, int d_r,
                         const double *q_nope, const double *q_rope,
                         const int32_t *q_pos, const double *w_uk,
                         double rope_base, double *out)
{
    const int D = d_c + d_r;
#pragma omp parallel for schedule(static)
    for (int ti = 0; ti < T * H; ++ti) {
        int t = ti / H, i = ti % H;
        const double *q = q_nope + (size_t)ti * d_h;
        const double *U = w_uk + (size_t)i * d_h * d_c;
        double *o = out + (size_t)ti * D;
        for (int c = 0; c < d_c; ++c) {
            double acc = 0.0;
            for (int k = 0; k < d_h; ++k)
                acc += U[(size_t)k * d_c + c] * q[k];
            o[c] = acc;
        }
        const double *qr = q_rope + (size_t)ti * d_r;
        if (q_pos)
            mla_oracle_rope(qr, d_r, (double)q_pos[t], rope_base, o + d_c);
        else
            for (int r = 0; r < d_r; ++r)
                o[d_c + r] = qr[r];
    }
}

/* Cache row of logical position j in sequence b, or NULL if the block table
 * entry is out of range. */
static const uint16_t *cache_row(const uint16_t *cache, int num_blocks,
                                 const int32_t *block_table, int max_blocks,
                                 int block_size, int D, int b, int j)
{
    int blk = block_table[(size_t)b * max_blocks + j / block_size];
    if (blk < 0 || blk >= num_blocks)
        return NULL;
    return cache + ((size_t)blk * block_size + (size_t)(j % block_size)) * D;
}

/* Expanded-form decode (steps a3-a5 and a7 without absorption), for a list of
 * n_pairs (row, head) pairs; row = b*s + t.
 *   cache       [num_blocks][block_size][d_c+d_r] bf16 bits, raw k^R
 *   q_nope      [B*s][H][d_h]      content query q^C
 *   q_rope      [B*s][H][d_r]      RoPE query, raw if q_pos != NULL
 *   w_uk, w_uv  [H][d_h][d_c]
 * Outputs: out [n_pairs][d_h] = o_{t,i}, lse [n_pairs] (natural log of the
 * softmax denominator of the scaled logits), probs (optional, may be NULL):
 * [n_pairs][probs_stride] attention weights over positions 0..probs_stride-1.
 * Returns 0, or -1 if a block table entry is out of range. */
int mla_oracle_decode_expanded(int B, int s, int H, int d_c, int d_r, int d_h,
                               int block_size, double rope_base,
                               const uint16_t *cache, int num_blocks,
                               const int32_t *block_table, int max_blocks,
                               const int32_t *seq_lens,
                               const double *q_nope, const double *q_rope,
                               const int32_t *q_pos,
                               const double *w_uk, const double *w_uv,
                               int n_pairs, const int32_t *pair_row,
                               const int32_t *pair_head,
                               double *out, double *lse,
                               double *probs, int probs_stride)
{
    const int D = d_c + d_r;
    const double scale = 1.0 / sqrt((double)(d_h + d_r));
    int bad = 0;
    (void)B;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int p = 0; p < n_pairs; ++p) {
        const int row = pair_row[p], i = pair_head[p];
        const int b = row / s, t = row % s;
        const int L = seq_lens[b];
        const int n_vis = L - s + t + 1;
        double *o = out + (size_t)p * d_h;
        for (int k = 0; k < d_h; ++k) o[k] = 0.0;
        if (probs)
            for (int j = 0; j < probs_stride; ++j) probs[(size_t)p * probs_stride + j] = 0.0;
        if (n_vis <= 0) {
            lse[p] = -INFINITY;
            continue;
        }
        const double *Uk = w_uk + (size_t)i * d_h * d_c;
        const double *Uv = w_uv + (size_t)i * d_h * d_c;
        const double *qc = q_nope + ((size_t)row * H + i) * d_h;
        double *qr = (double *)malloc(sizeof(double) * (size_t)d_r);
        double *c = (double *)malloc(sizeof(double) * (size_t)d_c);
        double *kr_raw = (double *)malloc(sizeof(double) * (size_t)d_r);
        double *kr = (double *)malloc(sizeof(double) * (size_t)d_r);
        double *kc = (double *)malloc(sizeof(double) * (size_t)d_h);
        double *score = (double *)malloc(sizeof(double) * (size_t)n_vis);
        const double *qr_in = q_rope + ((size_t)row * H + i) * d_r;
        if (q_pos)
            mla_oracle_rope(qr_in, d_r, (double)q_pos[row], rope_base, qr);
        else
            memcpy(qr, qr_in, sizeof(double) * (size_t)d_r);

        /* logits l_j = (q^C . k^C_j + q^R . k^R_j) / sqrt(d_h + d_r) */
        for (int j = 0; j < n_vis; ++j) {
            const uint16_t *rowp = cache_row(cache, num_blocks, block_table, max_blocks,
                                             block_size, D, b, j);
            if (!rowp) { bad = 1; score[j] = -INFINITY; continue; }
            for (int m = 0; m < d_c; ++m) c[m] = bf16_bits_to_f64(rowp[m]);
            for (int m = 0; m < d_r; ++m) kr_raw[m] = bf16_bits_to_f64(rowp[d_c + m]);
            mla_oracle_rope(kr_raw, d_r, (double)j, rope_base, kr);
            for (int k = 0; k < d_h; ++k) {          /* k^C = U^K c */
                double acc = 0.0;
                for (int m = 0; m < d_c; ++m) acc += Uk[(size_t)k * d_c + m] * c[m];
                kc[k] = acc;
            }
            double dot = 0.0;
            for (int k = 0; k < d_h; ++k) dot += qc[k] * kc[k];
            for (int m = 0; m < d_r; ++m) dot += qr[m] * kr[m];
            score[j] = dot * scale;
        }
        /* textbook softmax, max-subtracted */
        double mx = -INFINITY;
        for (int j = 0; j < n_vis; ++j) if (score[j] > mx) mx = score[j];
        double den = 0.0;
        for (int j = 0; j < n_vis; ++j) { score[j] = exp(score[j] - mx); den += score[j]; }
        lse[p] = mx + log(den);
        /* o = sum_j a_j v^C_j,  v^C_j = U^V c_j */
        for (int j = 0; j < n_vis; ++j) {
            const double a = score[j] / den;
            if (probs && j < probs_stride) probs[(size_t)p * probs_stride + j] = a;
            const uint16_t *rowp = cache_row(cache, num_blocks, block_table, max_blocks,
                                             block_size, D, b, j);
            if (!rowp) continue;
            for (int m = 0; m < d_c; ++m) c[m] = bf16_bits_to_f64(rowp[m]);
            for (int k = 0; k < d_h; ++k) {
                double acc = 0.0;
                for (int m = 0; m < d_c; ++m) acc += Uv[(size_t)k * d_c + m] * c[m];
                o[k] += a * acc;
            }
        }
        free(qr); free(c); free(kr_raw); free(kr); free(kc); free(score);
    }
    return bad ? -1 : 0;
}

/* Absorbed-form decode over the latent (steps a3-a6 as one exact softmax):
 *   l_j = (q_abs[0:d_c] . c^KV_j + q_abs[d_c:] . RoPE(k^R_j, j)) / sqrt(d_h+d_r)
 *   out = sum_j softmax_j(l) c^KV_j            (value = latent, U^V not applied)
 * q_abs [B*s][H][d_c+d_r]: absorbed content query followed by the already
 * rotated RoPE query.  Outputs out [n_pairs][d_c], lse [n_pairs].
 * Returns 0, or -1 if a block table entry is out of range. */
int mla_oracle_decode_latent(int B, int s, int H, int d_c, int d_r, int d_h,
                             int block_size, double rope_base,
                             const uint16_t *cache, int num_blocks,
                             const int32_t *block_table, int max_blocks,
                             const int32_t *seq_lens, const double *q_abs,
                             int n_pairs, const int32_t *pair_row,
                             const int32_t *pair_head,
                             double *out, double *lse)
{
    const int D = d_c + d_r;
    const double scale = 1.0 / sqrt((double)(d_h + d_r));
    int bad = 0;
    (void)B;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int p = 0; p < n_pairs; ++p) {
        const int row = pair_row[p], i = pair_head[p];
        const int b = row / s, t = row % s;
        const int n_vis = seq_lens[b] - s + t + 1;
        double *o = out + (size_t)p * d_c;
        for (int m = 0; m < d_c; ++m) o[m] = 0.0;
        if (n_vis <= 0) { lse[p] = -INFINITY; continue; }
        const double *q = q_abs + ((size_t)row * H + i) * D;
        double *score = (double *)malloc(sizeof(double) * (size_t)n_vis);
        double *kr_raw = (double *)malloc(sizeof(double) * (size_t)d_r);
        double *kr = (double *)malloc(sizeof(double) * (size_t)d_r);
        for (int j = 0; j < n_vis; ++j) {
            const uint16_t *rowp = cache_row(cache, num_blocks, block_table, max_blocks,
                                             block_size, D, b, j);
            if (!rowp) { bad = 1; score[j] = -INFINITY; continue; }
            double dot = 0.0;
            for (int m = 0; m < d_c; ++m) dot += q[m] * bf16_bits_to_f64(rowp[m]);
            for (int m = 0; m < d_r; ++m) kr_raw[m] = bf16_bits_to_f64(rowp[d_c + m]);
            mla_oracle_rope(kr_raw, d_r, (double)j, rope_base, kr);
            for (int m = 0; m < d_r; ++m) dot += q[d_c + m] * kr[m];
            score[j] = dot * scale;
        }
        double mx = -INFINITY;
        for (int j = 0; j < n_vis; ++j) if (score[j] > mx) mx = score[j];
        double den = 0.0;
        for (int j = 0; j < n_vis; ++j) { score[j] = exp(score[j] - mx); den += score[j]; }
        lse[p] = mx + log(den);
        for (int j = 0; j < n_vis; ++j) {
            const uint16_t *rowp = cache_row(cache, num_blocks, block_table, max_blocks,
                                             block_size, D, b, j);
            if (!rowp) continue;
            const double a = score[j] / den;
            for (int m = 0; m < d_c; ++m) o[m] += a * bf16_bits_to_f64(rowp[m]);
        }
        free(score); free(kr_raw); free(kr);
    }
    return bad ? -1 : 0;
}

/* The absorbed-form decode of mla_oracle_decode_latent for every head of a
 * list of rows: out [n_rows][H][d_c], lse [n_rows][H].  Each output takes the
 * same arithmetic in the same order as there (per key: the dot over the
 * latent, then over the rotated RoPE key, times the scale; then the
 * max-subtracted softmax over j ascending and the weighted latent sum over j
 * ascending), so the two agree bit for bit.  Only the loop nest differs: the
 * work is split over (row, group of up to 16 heads), and each key row is
 * widened and its RoPE part turned once per group instead of once per head,
 * which keeps whole batches affordable.  Returns 0, or -1 if a block table
 * entry is out of range. */
int mla_oracle_decode_latent_rows(int B, int s, int H, int d_c, int d_r, int d_h,
                                  int block_size, double rope_base,
                                  const uint16_t *cache, int num_blocks,
                                  const int32_t *block_table, int max_blocks,
                                  const int32_t *seq_lens, const double *q_abs,
                                  int n_rows, const int32_t *rows,
                                  double *out, double *lse)
{
    const int D = d_c + d_r;
    const double scale = 1.0 / sqrt((double)(d_h + d_r));
    const int G = 16;
    const int n_grp = (H + G - 1) / G;
    int bad = 0;
    (void)B;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int task = 0; task < n_rows * n_grp; ++task) {
        const int ri = task / n_grp, h0 = (task % n_grp) * G;
        const int h1 = h0 + G < H ? h0 + G : H, nh = h1 - h0;
        const int row = rows[ri];
        const int b = row / s, t = row % s;
        const int n_vis = seq_lens[b] - s + t + 1;
        for (int h = h0; h < h1; ++h) {
            double *o = out + ((size_t)ri * H + h) * d_c;
            for (int m = 0; m < d_c; ++m) o[m] = 0.0;
            lse[(size_t)ri * H + h] = -INFINITY;
        }
        if (n_vis <= 0) continue;
        double *score = (double *)malloc(sizeof(double) * (size_t)nh * (size_t)n_vis);
        double *den = (double *)malloc(sizeof(double) * (size_t)nh);
        double *c = (double *)malloc(sizeof(double) * (size_t)d_c);
        double *kr_raw = (double *)malloc(sizeof(double) * (size_t)d_r);
        double *kr = (double *)malloc(sizeof(double) * (size_t)d_r);
        for (int j = 0; j < n_vis; ++j) {
            const uint16_t *rowp = cache_row(cache, num_blocks, block_table, max_blocks,
                                             block_size, D, b, j);
            if (!rowp) {
                bad = 1;
                for (int h = 0; h < nh; ++h) score[(size_t)h * n_vis + j] = -INFINITY;
                continue;
            }
            for (int m = 0; m < d_c; ++m) c[m] = bf16_bits_to_f64(rowp[m]);
            for (int m = 0; m < d_r; ++m) kr_raw[m] = bf16_bits_to_f64(rowp[d_c + m]);
            mla_oracle_rope(kr_raw, d_r, (double)j, rope_base, kr);
            for (int h = 0; h < nh; ++h) {
                const double *q = q_abs + ((size_t)row * H + h0 + h) * D;
                double dot = 0.0;
                for (int m = 0; m < d_c; ++m) dot += q[m] * c[m];
                for (int m = 0; m < d_r; ++m) dot += q[d_c + m] * kr[m];
                score[(size_t)h * n_vis + j] = dot * scale;
            }
        }
        for (int h = 0; h < nh; ++h) {
            double *sc = score + (size_t)h * n_vis;
            double mx = -INFINITY;
            for (int j = 0; j < n_vis; ++j) if (sc[j] > mx) mx = sc[j];
            double dn = 0.0;
            for (int j = 0; j < n_vis; ++j) { sc[j] = exp(sc[j] - mx); dn += sc[j]; }
            den[h] = dn;
            lse[(size_t)ri * H + h0 + h] = mx + log(dn);
        }
        for (int j = 0; j < n_vis; ++j) {
            const uint16_t *rowp = cache_row(cache, num_blocks, block_table, max_blocks,
                                             block_size, D, b, j);
            if (!rowp) continue;
            for (int m = 0; m < d_c; ++m) c[m] = bf16_bits_to_f64(rowp[m]);
            for (int h = 0; h < nh; ++h) {
                const double a = score[(size_t)h * n_vis + j] / den[h];
                double *o = out + ((size_t)ri * H + h0 + h) * d_c;
                for (int m = 0; m < d_c; ++m) o[m] += a * c[m];
            }
        }
        free(score); free(den); free(c); free(kr_raw); free(kr);
    }
    return bad ? -1 : 0;
}

/* ------------------------------------------------------------------ FP8 cache
 * Row f1: the latent cache stored in 8-bit floating point.  The pages say the
 * deployed model keeps its KV cache at about 6 bits per element and its
 * weights in FP8 (DeepSeek-V2 paper review, sections 4 and 9), and that FP8
 * values are E4M3 with fine-grained scaling factors (DeepSeek-V3 report
 * summary, the FP8 training framework).  Reading used here: each cached row
 * [c^KV | k^R (rotated)] is stored as E4M3 codes with one fp32 scale for its
 * c^KV part and one for its k^R part, scale = amax / 448 (448 is the largest
 * finite E4M3 value), code = E4M3(x / scale) rounded to nearest-even and
 * saturated.  The scale and the quotient are taken in fp32, the precision the
 * GPU quantizer uses, so both sides make the same integer decision.
 *
 * E4M3 (OCP 8-bit floating point): 1 sign bit, 4 exponent bits with bias 7,
 * 3 mantissa bits.  Exponent 1..15: (-1)^s 2^(e-7) (1 + m/8), except e = 15,
 * m = 7, which is NaN; exponent 0: (-1)^s 2^-6 (m/8).  No infinities. */
double mla_oracle_e4m3_value(uint8_t code)
{
    const int sgn = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sgn ? -v : v;
}

void mla_oracle_e4m3_values(int n, const uint8_t *codes, double *out)
{
    for (int i = 0; i < n; ++i) out[i] = mla_oracle_e4m3_value(codes[i]);
}

/* Nearest E4M3 code to x, ties to the even code, magnitudes above 448
 * saturated to 448; found by comparing x with every finite value. */
uint8_t mla_oracle_e4m3_encode(float x)
{
    if (x != x) return 0x7F;
    const double a = fabs((double)x);
    int best = 0;
    double best_err = INFINITY;
    for (int c = 0; c <= 0x7E; ++c) {
        const double err = fabs(mla_oracle_e4m3_value((uint8_t)c) - a);
        if (err < best_err || (err == best_err && (c & 1) == 0)) {
            best = c;
            best_err = err;
        }
    }
    if (a > 448.0) best = 0x7E;
    return (uint8_t)((signbit(x) ? 0x80 : 0) | best);
}

void mla_oracle_e4m3_encode_n(int n, const float *x, uint8_t *codes)
{
#pragma omp parallel for schedule(static)
    for (int i = 0; i < n; ++i) codes[i] = mla_oracle_e4m3_encode(x[i]);
}

/* Quantizer of the FP8 cache: rows [N][d_c + d_r] fp32 -> codes [N][d_c + d_r]
 * and scales [N][2] (c^KV part, k^R part); an all-zero part gets scale 1. */
void mla_oracle_quantize_rows(int N, int d_c, int d_r, const float *rows, uint8_t *codes, float *scales)
{
    const int D = d_c + d_r;
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) {
        for (int part = 0; part < 2; ++part) {
            const int c0 = part ? d_c : 0, c1 = part ? D : d_c;
            float amax = 0.0f;
            for (int c = c0; c < c1; ++c) {
                const float a = fabsf(rows[(size_t)n * D + c]);
                if (a > amax) amax = a;
            }
            const float sc = amax > 0.0f ? amax / 448.0f : 1.0f;
            scales[2 * (size_t)n + part] = sc;
            for (int c = c0; c < c1; ++c)
                codes[(size_t)n * D + c] = mla_oracle_e4m3_encode(rows[(size_t)n * D + c] / sc);
        }
    }
}

/* Absorbed-form decode over the FP8 cache, every head of a list of rows (the
 * arithmetic of mla_oracle_decode_latent_rows on dequantized rows):
 *   c_j = E4M3(code) * scale_c,  k^R_j = E4M3(code) * scale_r (already rotated)
 *   l_j = (q_abs[0:d_c] . c_j + q_abs[d_c:] . k^R_j) / sqrt(d_h + d_r)
 *   out = sum_j softmax_j(l) c_j
 * codes [num_blocks][block_size][d_c+d_r] uint8, scales [num_blocks][block_size][2]
 * fp32; out [n_rows][H][d_c], lse [n_rows][H].  Returns 0, or -1 if a block
 * table entry is out of range. */
int mla_oracle_decode_latent_fp8_rows(int B, int s, int H, int d_c, int d_r, int d_h, int block_size,
                                      const uint8_t *codes, const float *scales, int num_blocks,
                                      const int32_t *block_table, int max_blocks, const int32_t *seq_lens,
                                      const double *q_abs, int n_rows, const int32_t *rows, double *out,
                                      double *lse)
{
    const int D = d_c + d_r;
    const double scale = 1.0 / sqrt((double)(d_h + d_r));
    const int G = 16;
    const int n_grp = (H + G - 1) / G;
    int bad = 0;
    (void)B;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int task = 0; task < n_rows * n_grp; ++task) {
        const int ri = task / n_grp, h0 = (task % n_grp) * G;
        const int h1 = h0 + G < H ? h0 + G : H, nh = h1 - h0;
        const int row = rows[ri];
        const int b = row / s, t = row % s;
        const int n_vis = seq_lens[b] - s + t + 1;
        for (int h = h0; h < h1; ++h) {
            double *o = out + ((size_t)ri * H + h) * d_c;
            for (int m = 0; m < d_c; ++m) o[m] = 0.0;
            lse[(size_t)ri * H + h] = -INFINITY;
        }
        if (n_vis <= 0) continue;
        double *score = (double *)malloc(sizeof(double) * (size_t)nh * (size_t)n_vis);
        double *den = (double *)malloc(sizeof(double) * (size_t)nh);
        double *x = (double *)malloc(sizeof(double) * (size_t)D);
        for (int j = 0; j < n_vis; ++j) {
            const int blk = block_table[(size_t)b * max_blocks + j / block_size];
            if (blk < 0 || blk >= num_blocks) {
                bad = 1;
                for (int h = 0; h < nh; ++h) score[(size_t)h * n_vis + j] = -INFINITY;
                continue;
            }
            const size_t slot = (size_t)blk * block_size + (size_t)(j % block_size);
            for (int m = 0; m < D; ++m)
                x[m] = mla_oracle_e4m3_value(codes[slot * D + m]) * (double)scales[2 * slot + (m < d_c ? 0 : 1)];
            for (int h = 0; h < nh; ++h) {
                const double *q = q_abs + ((size_t)row * H + h0 + h) * D;
                double dot = 0.0;
                for (int m = 0; m < d_c; ++m) dot += q[m] * x[m];
                for (int m = d_c; m < D; ++m) dot += q[m] * x[m];
                score[(size_t)h * n_vis + j] = dot * scale;
            }
        }
        for (int h = 0; h < nh; ++h) {
            double *sc = score + (size_t)h * n_vis;
            double mx = -INFINITY;
            for (int j = 0; j < n_vis; ++j) if (sc[j] > mx) mx = sc[j];
            double dn = 0.0;
            for (int j = 0; j < n_vis; ++j) { sc[j] = exp(sc[j] - mx); dn += sc[j]; }
            den[h] = dn;
            lse[(size_t)ri * H + h0 + h] = mx + log(dn);
        }
        for (int j = 0; j < n_vis; ++j) {
            const int blk = block_table[(size_t)b * max_blocks + j / block_size];
            if (blk < 0 || blk >= num_blocks) continue;
            const size_t slot = (size_t)blk * block_size + (size_t)(j % block_size);
            for (int m = 0; m < d_c; ++m)
                x[m] = mla_oracle_e4m3_value(codes[slot * D + m]) * (double)scales[2 * slot];
            for (int h = 0; h < nh; ++h) {
                const double a = score[(size_t)h * n_vis + j] / den[h];
                double *o = out + ((size_t)ri * H + h0 + h) * d_c;
                for (int m = 0; m < d_c; ++m) o[m] += a * x[m];
            }
        }
        free(score); free(den); free(x);
    }
    return bad ? -1 : 0;
}

/* ------------------------------------------------------- append extras (f4)
 * DeepSeek-V2 paper review, section 2: the deployed model also puts an
 * RMSNorm after the compressed latent; the long-context passage: the 4K
 * pre-training context is extended with YaRN, scale 40.  The pages give no
 * further constants; the readings used here (listed in the design notes):
 *   - RMSNorm of the latent row: c_m <- c_m / sqrt(mean(c^2) + eps) * w_m.
 *   - YaRN frequencies (the NTK-by-parts interpolation of the YaRN method):
 *     pair k has theta_k = base^(-2k/d_r) and wavelength lambda_k =
 *     2 pi / theta_k; r_k = L0 / lambda_k rotations over the original
 *     context L0; ramp g = clamp((r_k - alpha) / (beta - alpha), 0, 1);
 *     theta'_k = (1 - g) theta_k / s + g theta_k.  With s <= 1 the plain
 *     RoPE frequencies are used. */
void mla_oracle_rmsnorm_rows(int N, int d, const double *x, const double *w, double eps, double *y)
{
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) {
        double ss = 0.0;
        for (int m = 0; m < d; ++m) ss += x[(size_t)n * d + m] * x[(size_t)n * d + m];
        const double inv = 1.0 / sqrt(ss / (double)d + eps);
        for (int m = 0; m < d; ++m) y[(size_t)n * d + m] = x[(size_t)n * d + m] * inv * w[m];
    }
}

void mla_oracle_yarn_theta(int d_r, double base, double s, double L0, double alpha, double beta, double *theta)
{
    const double pi = 3.14159265358979323846;
    for (int k = 0; k < d_r / 2; ++k) {
        const double th = pow(base, -2.0 * (double)k / (double)d_r);
        if (s <= 1.0) {
            theta[k] = th;
            continue;
        }
        const double r = L0 / (2.0 * pi / th);
        double g = (r - alpha) / (beta - alpha);
        if (g < 0.0) g = 0.0;
        if (g > 1.0) g = 1.0;
        theta[k] = (1.0 - g) * th / s + g * th;
    }
}

/* RoPE of rows [N][d_r] at positions pos[N] with given frequencies theta[d_r/2]:
 * pair k = (x[2k], x[2k+1]) turned by pos * theta[k]. */
void mla_oracle_rope_rows_theta(int N, int d_r, const double *x, const int32_t *pos, const double *theta,
                                double *y)
{
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n)
        for (int k = 0; k < d_r / 2; ++k) {
            const double ang = (double)pos[n] * theta[k];
            const double c = cos(ang), sn = sin(ang);
            const double x0 = x[(size_t)n * d_r + 2 * k], x1 = x[(size_t)n * d_r + 2 * k + 1];
            y[(size_t)n * d_r + 2 * k] = x0 * c - x1 * sn;
            y[(size_t)n * d_r + 2 * k + 1] = x0 * sn + x1 * c;
        }
}

/* Up-projection (step a7): out_heads[t][i] = U^V_i latent[t][i]
 * latent [T][H][d_c], w_uv [H][d_h][d_c] -> out_heads [T][H][d_h]. */
void mla_oracle_up_v(int T, int H, int d_h, int d_c, const double *latent,
                     const double *w_uv, double *out_heads)
{
#pragma omp parallel for schedule(static)
    for (int ti = 0; ti < T * H; ++ti) {
        const int i = ti % H;
        const double *x = latent + (size_t)ti * d_c;
        const double *U = w_uv + (size_t)i * d_h * d_c;
        for (int k = 0; k < d_h; ++k) {
            double acc = 0.0;
            for (int m = 0; m < d_c; ++m) acc += U[(size_t)k * d_c + m] * x[m];
            out_heads[(size_t)ti * d_h + k] = acc;
        }
    }
}

/* Output projection: u_t = sum_i O_i o_{t,i}, with O = W^O [d_model][H*d_h]
 * whose column block i is O_i.  heads [T][H*d_h] -> u [T][d_model]. */
void mla_oracle_out_proj(int T, int H, int d_h, int d_model, const double *heads,
                         const double *w_o, double *u)
{
    const int K = H * d_h;
#pragma omp parallel for schedule(static)
    for (int td = 0; td < T * d_model; ++td) {
        const int t = td / d_model, r = td % d_model;
        double acc = 0.0;
        for (int i = 0; i < H; ++i)
            for (int k = 0; k < d_h; ++k)
                acc += w_o[(size_t)r * K + (size_t)i * d_h + k] * heads[(size_t)t * K + (size_t)i * d_h + k];
        u[td] = acc;
    }
}

/* ------------------------------------------------- weight pre-absorption (f3)
 * DeepSeek-V2 paper review, section 2: at inference W^UK can be absorbed into
 * the query's up-projection and W^UV into the output projection, so that the
 * attention runs on the latent directly; the query path compresses to
 * c^Q = W^DQ h (width d_q, 1536 in V2) and q^C_i = W^UQ_i c^Q.
 *   W^QK_i = (U^K_i)^T W^UQ_i     [d_c][d_q]: q~_i = W^QK_i c^Q
 *   W^OV[:, i d_c : (i+1) d_c] = O_i U^V_i     [d_model][H d_c]:
 *                                  u = sum_i W^OV_i o~_i
 * w_uq [H][d_h][d_q], w_uk, w_uv [H][d_h][d_c], w_o [d_model][H d_h]. */
void mla_oracle_fold_qk(int H, int d_h, int d_c, int d_q, const double *w_uq, const double *w_uk, double *w_qk)
{
#pragma omp parallel for collapse(2) schedule(static)
    for (int i = 0; i < H; ++i)
        for (int c = 0; c < d_c; ++c) {
            double *out = w_qk + ((size_t)i * d_c + c) * d_q;
            for (int q = 0; q < d_q; ++q) out[q] = 0.0;
            for (int k = 0; k < d_h; ++k) {
                const double u = w_uk[((size_t)i * d_h + k) * d_c + c];
                const double *row = w_uq + ((size_t)i * d_h + k) * d_q;
                for (int q = 0; q < d_q; ++q) out[q] += u * row[q];
            }
        }
}

void mla_oracle_fold_ov(int H, int d_h, int d_c, int d_model, const double *w_o, const double *w_uv, double *w_ov)
{
#pragma omp parallel for collapse(2) schedule(static)
    for (int m = 0; m < d_model; ++m)
        for (int i = 0; i < H; ++i) {
            double *out = w_ov + (size_t)m * H * d_c + (size_t)i * d_c;
            for (int c = 0; c < d_c; ++c) out[c] = 0.0;
            for (int k = 0; k < d_h; ++k) {
                const double o = w_o[(size_t)m * H * d_h + (size_t)i * d_h + k];
                const double *row = w_uv + ((size_t)i * d_h + k) * d_c;
                for (int c = 0; c < d_c; ++c) out[c] += o * row[c];
            }
        }
}

/* Absorbed query from the compressed query latent with the folded weights:
 * q_abs[t][i] = [W^QK_i c_q[t] | RoPE(q_rope[t][i], q_pos[t])] (copied if
 * q_pos is NULL).  c_q [T][d_q], q_rope [T][H][d_r], w_qk [H][d_c][d_q]. */
void mla_oracle_absorb_q_folded(int T, int H, int d_c, int d_q, int d_r, const double *c_q, const double *q_rope,
                                const int32_t *q_pos, const double *w_qk, double base, double *q_abs)
{
    const int D = d_c + d_r;
#pragma omp parallel for collapse(2) schedule(static)
    for (int t = 0; t < T; ++t)
        for (int i = 0; i < H; ++i) {
            double *o = q_abs + ((size_t)t * H + i) * D;
            const double *x = c_q + (size_t)t * d_q;
            for (int c = 0; c < d_c; ++c) {
                const double *w = w_qk + ((size_t)i * d_c + c) * d_q;
                double acc = 0.0;
                for (int q = 0; q < d_q; ++q) acc += w[q] * x[q];
                o[c] = acc;
            }
            const double *r = q_rope + ((size_t)t * H + i) * d_r;
            if (q_pos)
                mla_oracle_rope(r, d_r, (double)q_pos[t], base, o + d_c);
            else
                for (int m = 0; m < d_r; ++m) o[d_c + m] = r[m];
        }
}

/* Output projection with the folded weights: u[t] = sum_i W^OV_i latent[t][i],
 * latent [T][H][d_c], w_ov [d_model][H d_c]. */
void mla_oracle_up_out_folded(int T, int H, int d_c, int d_model, const double *latent, const double *w_ov,
                              double *u)
{
#pragma omp parallel for collapse(2) schedule(static)
    for (int t = 0; t < T; ++t)
        for (int m = 0; m < d_model; ++m) {
            const double *w = w_ov + (size_t)m * H * d_c;
            const double *x = latent + (size_t)t * H * d_c;
            double acc = 0.0;
            for (int j = 0; j < H * d_c; ++j) acc += w[j] * x[j];
            u[(size_t)t * d_model + m] = acc;
        }
}
