/*
 * dsa_oracle.c -- plain, slow, fp64 CPU oracle for the DeepSeek-Sparse-Attention
 * hot path of GLM-5.2 (lightning indexer -> causal top-k -> absorbed sparse MLA,
 * with IndexShare reuse).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call this code:
 * only the test-suite, the smoke check and the CPU-baseline leg of the benchmark
 * load it.  It shares no source, header, table or helper with the CUDA library.
 *
 * Every function takes the exact input values as float32 (a bf16 value widens to
 * float32 without rounding) and computes in double precision, one output at a
 * time, in the order the definition states.  Loops over independent outputs may
 * run on several OpenMP threads; that changes no arithmetic.
 *
 * Sources (page title, section):
 *  [TM]  "GLM-5.2 -- Model techniques map" (models.inteligile.com), section
 *        "Checked in its code", rows "Indexer-selected sparse attention (DeepSeek
 *        Sparse Attention)", "Multi-head latent attention", "Learnable attention
 *        sink", "Partial RoPE", "QK normalization".
 *  [AE]  "GLM-5.2 -- LLM architectures explained", sections "Modelled costs"
 *        and "Every architecture field".
 *  [HA]  "GLM 5.2 -- Hermosa AI", sections "78 layers, IndexShare pattern" and
 *        "MLA + DSA with IndexShare".
 *  [LA]  "GLM-5.2 -- LLM atlas" (French), section "Champs bruts du config.json".
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - indexer score  score(t,s) = sum_h w[t,h] * max(0, q_idx[t,h] . k_idx[s]),
 *    no further scale constant; w is a float32 input;
 *  - a query at position t sees cache rows s = 0..t (its own row included);
 *  - top-k keeps min(topk, t+1) rows; among equal scores the lower position wins;
 *    the kept positions are reported in ascending order, padded with -1;
 *  - attention is the absorbed MLA form: per head the query is a d_lat latent
 *    part plus a d_rope RoPE part, dotted with the cached row [c | r];
 *    probabilities are a plain softmax (no sink); the output is sum_j p_j c_j;
 *  - IndexShare: layer 0 of a group selects, every later layer of the group
 *    reuses that selection unchanged.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Lightning-indexer scores  [TM "Indexer-selected sparse attention": the indexer
 * scores past tokens per head; shapes index_n_heads=32, index_head_dim=128; one
 * indexer key per token shared by all heads ("k = k_norm(wk(h)) ... [B, S, 1, D]",
 * row "QK normalization")].
 *
 *   q      [n_q][heads][dim]                 indexer queries (post-RoPE)
 *   w      [n_q][heads]                      head weights
 *   k      k[q_seq[i]*k_seq_stride + s*k_row_stride + d]   indexer keys
 *   scores [n_q][L]   out; entry s of row i is the score for s <= q_pos[i],
 *                     NaN for s > q_pos[i] (not visible)
 */
void oracle_index_scores(int n_q, int heads, int dim, const float *q, const float *w,
                         const float *k, int64_t k_seq_stride, int64_t k_row_stride,
                         const int32_t *q_seq, const int32_t *q_pos, int L, double *scores) {
    int64_t total = (int64_t)n_q * L;
#pragma omp parallel for schedule(static)
    for (int64_t e = 0; e < total; e++) {
        int i = (int)(e / L);
        int s = (int)(e % L);
        if (s > q_pos[i]) {
            scores[e] = NAN;
            continue;
        }
        const float *key = k + (int64_t)q_seq[i] * k_seq_stride + (int64_t)s * k_row_stride;
        double score = 0.0;
        for (int h = 0; h < heads; h++) {
            const float *qh = q + ((int64_t)i * heads + h) * dim;
            double dot = 0.0;
            for (int d = 0; d < dim; d++) dot += (double)qh[d] * (double)key[d];
            double relu = dot > 0.0 ? dot : 0.0;
            score += (double)w[(int64_t)i * heads + h] * relu;
        }
        scores[e] = score;
    }
}

/*
 * One OCP 8-bit floating-point E4M3 value (the variant without infinities),
 * decoded from the format's definition: a sign bit, a 4-bit exponent with bias
 * 7 and a 3-bit mantissa; exponent field 0 is subnormal (m/8 * 2^-6); exponent
 * and mantissa all ones (0x7F, 0xFF) is NaN.  Largest finite magnitude 448.
 */
double oracle_e4m3_to_double(uint8_t c) {
    int sign = c >> 7, e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    double mag = (e == 0) ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -mag : mag;
}

/*
 * Lightning-indexer scores with 8-bit E4M3 queries and keys, each scaled per
 * row (the FP8 variant; same definition as oracle_index_scores on the exact
 * operand values):
 *   q[i][h][d] = e4m3(q8[i][h][d]) * q_scale[i*heads + h]        (q_scale NULL = 1)
 *   k[s][d]    = e4m3(k8[q_seq[i]*k_seq_stride + s*k_row_stride + d])
 *                * k_scale[q_seq[i]*ks_seq_stride + s]           (k_scale NULL = 1)
 * Every product and sum in double precision.
 */
void oracle_index_scores_e4m3(int n_q, int heads, int dim, const uint8_t *q8, const float *q_scale,
                              const float *w, const uint8_t *k8, const float *k_scale, int64_t k_seq_stride,
                              int64_t k_row_stride, int64_t ks_seq_stride, const int32_t *q_seq,
                              const int32_t *q_pos, int L, double *scores) {
    double lut[256];
    for (int c = 0; c < 256; c++) lut[c] = oracle_e4m3_to_double((uint8_t)c);
    int64_t total = (int64_t)n_q * L;
#pragma omp parallel for schedule(static)
    for (int64_t e = 0; e < total; e++) {
        int i = (int)(e / L);
        int s = (int)(e % L);
        if (s > q_pos[i]) {
            scores[e] = NAN;
            continue;
        }
        const uint8_t *key = k8 + (int64_t)q_seq[i] * k_seq_stride + (int64_t)s * k_row_stride;
        double ks = k_scale ? (double)k_scale[(int64_t)q_seq[i] * ks_seq_stride + s] : 1.0;
        double score = 0.0;
        for (int h = 0; h < heads; h++) {
            const uint8_t *qh = q8 + ((int64_t)i * heads + h) * dim;
            double qs = q_scale ? (double)q_scale[(int64_t)i * heads + h] : 1.0;
            double dot = 0.0;
            for (int d = 0; d < dim; d++) dot += (lut[qh[d]] * qs) * (lut[key[d]] * ks);
            double relu = dot > 0.0 ? dot : 0.0;
            score += (double)w[(int64_t)i * heads + h] * relu;
        }
        scores[e] = score;
    }
}

/* Candidate for the top-k ordering: larger score first, then lower position. */
typedef struct {
    double score;
    int32_t pos;
} cand_t;

static int by_score_then_pos(const void *a, const void *b) {
    const cand_t *x = (const cand_t *)a, *y = (const cand_t *)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    return (x->pos < y->pos) ? -1 : (x->pos > y->pos);
}

static int by_pos(const void *a, const void *b) {
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x < y) ? -1 : (x > y);
}

/*
 * Causal top-k  [TM "Indexer-selected sparse attention": "topk = min(index_topk,
 * ...)" then the indices of the topk largest scores, as int32 [B, S, topk]].
 * The pages take the minimum over the key length; the visible length t+1 is used
 * here, so masked positions are never chosen.  A full sort is used (the plain
 * definition), then the kept positions are re-sorted ascending.
 *
 *   scores [n_q][L] (only s <= q_pos[i] is read), idx [n_q][topk] out, cnt [n_q] out
 */
void oracle_topk(int n_q, int L, const double *scores, const int32_t *q_pos, int topk,
                 int32_t *idx, int32_t *cnt) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < n_q; i++) {
        int n = q_pos[i] + 1;
        int kk = topk < n ? topk : n;
        cand_t *c = (cand_t *)malloc(sizeof(cand_t) * (size_t)n);
        for (int s = 0; s < n; s++) {
            double v = scores[(int64_t)i * L + s];
            if (v == 0.0) v = 0.0; /* -0.0 and +0.0 are the same score */
            c[s].score = v;
            c[s].pos = s;
        }
        qsort(c, (size_t)n, sizeof(cand_t), by_score_then_pos);
        int32_t *row = idx + (int64_t)i * topk;
        for (int j = 0; j < kk; j++) row[j] = c[j].pos;
        qsort(row, (size_t)kk, sizeof(int32_t), by_pos);
        for (int j = kk; j < topk; j++) row[j] = -1;
        cnt[i] = kk;
        free(c);
    }
}

/*
 * Absorbed MLA attention of one query head over a list of cache rows
 * [TM "Multi-head latent attention": kv_a_proj_with_mqa yields kv_lora_rank +
 * qk_rope_head_dim = 512 + 64 per token; kv_b_proj up-projects the 512-dim latent
 * per head; "Learnable attention sink": a plain float32 softmax with no extra
 * logit; "Partial RoPE": 192 nope + 64 rope dims per head].
 * In absorbed form the up-projection W_UK is folded into the query, so each head's
 * logit is scale * (q_lat . c_s + q_rope . r_s) and the output is the
 * probability-weighted sum of the latents c_s (W_UV is applied outside).
 *
 *   qh   [d_lat + d_rope]             the head's query
 *   rows list of n_rows pointers to cache rows [c (d_lat) | r (d_rope)]
 *   out  [d_lat]  lse (natural log of the softmax normaliser, logits scaled)
 */
static void attend_one_head(const float *qh, const float *const *rows, int n_rows, int d_lat,
                            int d_rope, double scale, double *logit_buf, double *out,
                            double *lse) {
    int dk = d_lat + d_rope;
    double m = -INFINITY;
    for (int j = 0; j < n_rows; j++) {
        double dot = 0.0;
        for (int d = 0; d < dk; d++) dot += (double)qh[d] * (double)rows[j][d];
        logit_buf[j] = scale * dot;
        if (logit_buf[j] > m) m = logit_buf[j];
    }
    double l = 0.0;
    for (int j = 0; j < n_rows; j++) {
        logit_buf[j] = exp(logit_buf[j] - m); /* unnormalised probability */
        l += logit_buf[j];
    }
    for (int d = 0; d < d_lat; d++) out[d] = 0.0;
    for (int j = 0; j < n_rows; j++) {
        double p = logit_buf[j] / l;
        for (int d = 0; d < d_lat; d++) out[d] += p * (double)rows[j][d];
    }
    *lse = m + log(l);
}

/*
 * Sparse absorbed MLA: each query attends only to its selected rows
 * [TM "Indexer-selected sparse attention": each query attends only to the
 * index_topk selected tokens through an additive sparse mask -- the mask is 0 on
 * selected rows and -inf elsewhere, so attending over the selected rows alone is
 * the same computation].
 *
 *   q    [n_q][heads][d_lat + d_rope]
 *   kv   row s of sequence b at kv + b*kv_seq_stride + s*kv_row_stride
 *   idx  [n_q][topk] selected positions (first cnt[i] entries used)
 *   out  [n_q][heads][d_lat]   lse [n_q][heads] (may be NULL)
 */
void oracle_sparse_mla(int n_q, int heads, int d_lat, int d_rope, double scale, const float *q,
                       const float *kv, int64_t kv_seq_stride, int64_t kv_row_stride,
                       const int32_t *q_seq, const int32_t *idx, const int32_t *cnt, int topk,
                       double *out, double *lse) {
    int dk = d_lat + d_rope;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t e = 0; e < (int64_t)n_q * heads; e++) {
        int i = (int)(e / heads);
        int n_rows = cnt[i];
        const float **rows = (const float **)malloc(sizeof(float *) * (size_t)(n_rows > 0 ? n_rows : 1));
        double *buf = (double *)malloc(sizeof(double) * (size_t)(n_rows > 0 ? n_rows : 1));
        const float *base = kv + (int64_t)q_seq[i] * kv_seq_stride;
        for (int j = 0; j < n_rows; j++)
            rows[j] = base + (int64_t)idx[(int64_t)i * topk + j] * kv_row_stride;
        double l;
        attend_one_head(q + e * dk, rows, n_rows, d_lat, d_rope, scale, buf, out + e * d_lat, &l);
        if (lse) lse[e] = l;
        free(rows);
        free(buf);
    }
}

/*
 * Dense causal absorbed MLA over every visible row s = 0..q_pos[i]: the textbook
 * causal attention the sparse form reduces to when topk >= t+1.
 */
void oracle_dense_mla(int n_q, int heads, int d_lat, int d_rope, double scale, const float *q,
                      const float *kv, int64_t kv_seq_stride, int64_t kv_row_stride,
                      const int32_t *q_seq, const int32_t *q_pos, double *out, double *lse) {
    int dk = d_lat + d_rope;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t e = 0; e < (int64_t)n_q * heads; e++) {
        int i = (int)(e / heads);
        int n_rows = q_pos[i] + 1;
        const float **rows = (const float **)malloc(sizeof(float *) * (size_t)n_rows);
        double *buf = (double *)malloc(sizeof(double) * (size_t)n_rows);
        const float *base = kv + (int64_t)q_seq[i] * kv_seq_stride;
        for (int s = 0; s < n_rows; s++) rows[s] = base + (int64_t)s * kv_row_stride;
        double l;
        attend_one_head(q + e * dk, rows, n_rows, d_lat, d_rope, scale, buf, out + e * d_lat, &l);
        if (lse) lse[e] = l;
        free(rows);
        free(buf);
    }
}

/* Value of a bf16 bit pattern: the upper half of an IEEE binary32. */
static double bf16_bits_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * attend_one_head on rows already widened to double: rows is [n_rows][d_lat +
 * d_rope], row j = [c_j | r_j].  The same steps in the same order.
 */
static void attend_one_head_f64(const float *qh, const double *rows, int n_rows, int d_lat, int d_rope,
                                double scale, double *logit_buf, double *out, double *lse) {
    int dk = d_lat + d_rope;
    double m = -INFINITY;
    for (int j = 0; j < n_rows; j++) {
        double dot = 0.0;
        for (int d = 0; d < dk; d++) dot += (double)qh[d] * rows[(int64_t)j * dk + d];
        logit_buf[j] = scale * dot;
        if (logit_buf[j] > m) m = logit_buf[j];
    }
    double l = 0.0;
    for (int j = 0; j < n_rows; j++) {
        logit_buf[j] = exp(logit_buf[j] - m);
        l += logit_buf[j];
    }
    for (int d = 0; d < d_lat; d++) out[d] = 0.0;
    for (int j = 0; j < n_rows; j++) {
        double p = logit_buf[j] / l;
        for (int d = 0; d < d_lat; d++) out[d] += p * rows[(int64_t)j * dk + d];
    }
    *lse = m + log(l);
}

/*
 * Sparse absorbed MLA over a cache that keeps the latent in 8 bits (the FP8
 * variant: "GLM-5.2 -- Model techniques map" lists FP8 inference under
 * inference quantization, and the key-facts table of "GLM-5.2 -- LLM atlas"
 * gives fp8 as the precision; the cache format below is this oracle's reading,
 * the pages give none).  Row s of sequence b is the byte string at
 * kv8 + b*kv_seq_stride + s*kv_row_stride (strides in bytes):
 *   bytes [0, d_lat)                    E4M3 codes c8[d] of the latent
 *   bytes [d_lat, d_lat + 2*d_rope)     the RoPE key r as bf16, little-endian
 *   bytes [d_lat + 2*d_rope, + 4)       float32 scale sigma, little-endian
 * and the latent the attention sees is c[d] = sigma * e4m3(c8[d]).  Every
 * selected row is widened to double exactly (one product per latent value) and
 * attended as in oracle_sparse_mla.
 */
void oracle_sparse_mla_fp8(int n_q, int heads, int d_lat, int d_rope, double scale, const float *q,
                           const uint8_t *kv8, int64_t kv_seq_stride, int64_t kv_row_stride,
                           const int32_t *q_seq, const int32_t *idx, const int32_t *cnt, int topk,
                           double *out, double *lse) {
    int dk = d_lat + d_rope;
    double lut[256];
    for (int c = 0; c < 256; c++) lut[c] = oracle_e4m3_to_double((uint8_t)c);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t e = 0; e < (int64_t)n_q * heads; e++) {
        int i = (int)(e / heads);
        int n_rows = cnt[i];
        size_t nr = (size_t)(n_rows > 0 ? n_rows : 1);
        double *rows = (double *)malloc(sizeof(double) * nr * (size_t)dk);
        double *buf = (double *)malloc(sizeof(double) * nr);
        const uint8_t *base = kv8 + (int64_t)q_seq[i] * kv_seq_stride;
        for (int j = 0; j < n_rows; j++) {
            const uint8_t *row = base + (int64_t)idx[(int64_t)i * topk + j] * kv_row_stride;
            float sigma;
            memcpy(&sigma, row + d_lat + 2 * d_rope, sizeof sigma);
            double *dst = rows + (int64_t)j * dk;
            for (int d = 0; d < d_lat; d++) dst[d] = (double)sigma * lut[row[d]];
            for (int d = 0; d < d_rope; d++) {
                uint16_t bits;
                memcpy(&bits, row + d_lat + 2 * d, sizeof bits);
                dst[d_lat + d] = bf16_bits_to_double(bits);
            }
        }
        double l;
        attend_one_head_f64(q + e * dk, rows, n_rows, d_lat, d_rope, scale, buf, out + e * d_lat, &l);
        if (lse) lse[e] = l;
        free(rows);
        free(buf);
    }
}
