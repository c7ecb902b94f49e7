/*
 * qsa_oracle.c -- plain, slow, fp64 CPU oracle for Qwen Sparse Attention (QSA).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call this file:
 * only the test-suite, the package's smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header or constant with the CUDA
 * library and includes nothing but the C standard library and OpenMP.
 *
 * Sources (the page title, then the section or equation):
 *   [notes]  "On the Design of Qwen3.8 Next Architecture: Evaluation,
 *            Efficiency, and Training Stability" (reading notes), section 6
 *            "GDN 连续压缩与 QSA 精确检索": the pooled-key equation for k̄_b,
 *            the indexer equation for I_ib, the budget sentence (K = 2048,
 *            r = 4, at most 512 complete blocks, the trailing causal block always
 *            kept, selected blocks expanded to token indices) and the O(n²/r)
 *            complexity equation.
 *   [table]  same page, "Model Summary" table: QSA 24 query / 2 KV heads, head
 *            dim 256; indexer 4 query heads, 1 key head, dim 128, ratio 4.
 *
 * Readings where the pages are silent:
 *   - RMSNorm in the compressor has unit gain and eps (default 1e-6); the
 *     caller may switch it off (plain mean-pool).
 *   - the indexer score carries a per-(query, head) weight w; w = 1 gives the
 *     [notes] I_ib equation exactly.  No scale inside the indexer.
 *   - the own block b_t = floor(t/r) is always selected; the remaining k-1
 *     slots go to the best strictly earlier blocks, ordered by score
 *     (descending) then block index (ascending).  |Sel_t| = min(k, b_t + 1).
 *   - inside the own block only tokens j <= t are attended.
 *   - plain softmax with scale s (1/sqrt(256) for the model), no sink or cap.
 *   - the partial RoPE of the pooled key (optional): after the pool and the
 *     norm, the first rope_dims dims rotate in pairs (i, i + rope_dims/2) by
 *     (b r) base^(-2i / rope_dims); queries arrive already rotated at t.
 *
 * All inputs that are bf16 on the device are passed here as raw 16-bit
 * patterns and widened exactly to double.  Every accumulation is fp64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* exact bf16 -> double: a bf16 pattern is the top half of an IEEE binary32 */
static double widen_bf16(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------ */
/* [notes] pooled-key equation: k̄_b = RMSNorm(AvgPool(k_{br .. br+r-1})).     */
/* Only complete blocks b < floor(Lk / r) exist.                               */
/* ------------------------------------------------------------------------ */
void qsa_oracle_compress(const uint16_t *k_idx, int64_t Lk, int r, int d,
                         int normalise, double eps, double *kc)
{
    int64_t nb = Lk / r;
#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < nb; ++b) {
        double *out = kc + b * d;
        for (int c = 0; c < d; ++c) {
            double s = 0.0;
            for (int j = 0; j < r; ++j)
                s += widen_bf16(k_idx[(b * r + j) * d + c]);
            out[c] = s / (double)r;
        }
        if (normalise) {
            double ms = 0.0;
            for (int c = 0; c < d; ++c)
                ms += out[c] * out[c];
            ms /= (double)d;
            double inv = 1.0 / sqrt(ms + eps);
            for (int c = 0; c < d; ++c)
                out[c] *= inv;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* [notes] section 6, the sentence before the pooled-key equation: the keys   */
/* are average-pooled first and the partial RoPE is applied afterwards, so     */
/* token representations of different rotation phases are never averaged.     */
/* Readings (the pages give no dims, base or position): the first rope_dims   */
/* dims rotate, in pairs (i, i + rope_dims/2), by the angle pos * base^(-2i /  */
/* rope_dims); a pooled key sits at the position of its block's first token   */
/* (b * r), a query at its own position t.  x is rotated in place:            */
/*   x[i]     <- x[i] cos a - x[i + h] sin a                                   */
/*   x[i + h] <- x[i] sin a + x[i + h] cos a                                   */
/* ------------------------------------------------------------------------ */
void qsa_oracle_rope(double *x, int64_t n, int d, const int64_t *pos, int rope_dims, double base)
{
    int h = rope_dims / 2;
#pragma omp parallel for schedule(static)
    for (int64_t v = 0; v < n; ++v) {
        double *xv = x + v * d;
        for (int i = 0; i < h; ++i) {
            double a = (double)pos[v] * pow(base, -2.0 * (double)i / (double)rope_dims);
            double c = cos(a), s = sin(a);
            double x0 = xv[i], x1 = xv[i + h];
            xv[i] = x0 * c - x1 * s;
            xv[i + h] = x0 * s + x1 * c;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* [notes] indexer equation, weighted: for query position t and every        */
/* complete block b strictly before the own block (b < b_t = floor(t / r)):   */
/*   S[t, b] = sum_h w[t, h] * max(0, <q_idx[t, h, :], kc[b, :]>)             */
/* Entries b >= b_t are not candidates and are set to -inf.                   */
/* Query row i of the sequence sits at t = (Lk - Lq) + i.                      */
/* ------------------------------------------------------------------------ */
void qsa_oracle_index_scores(const uint16_t *q_idx, const float *w, const double *kc,
                             int64_t Lq, int64_t Lk, int r, int H, int d,
                             const int64_t *rows, int64_t nrows,
                             double *out, int64_t ld)
{
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t n = 0; n < nrows; ++n) {
        int64_t i = rows[n];
        int64_t t = (Lk - Lq) + i;
        int64_t bt = t / r;
        double *srow = out + n * ld;
        double q[16][256];
        for (int h = 0; h < H; ++h)
            for (int c = 0; c < d; ++c)
                q[h][c] = widen_bf16(q_idx[(i * H + h) * d + c]);
        for (int64_t b = 0; b < ld; ++b) {
            if (b >= bt) {
                srow[b] = -INFINITY;
                continue;
            }
            double s = 0.0;
            for (int h = 0; h < H; ++h) {
                double dot = 0.0;
                for (int c = 0; c < d; ++c)
                    dot += q[h][c] * kc[b * d + c];
                s += (double)w[i * H + h] * (dot > 0.0 ? dot : 0.0);
            }
            srow[b] = s;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* [notes] budget sentence: own block forced, then the k-1 best candidates.  */
/* Candidates of a row are blocks 0 .. b_t - 1.  Order: score descending,      */
/* block index ascending on ties.  Output sorted ascending, padded with -1.    */
/* ------------------------------------------------------------------------ */
struct cand { double s; int64_t b; };

static int cand_cmp(const void *pa, const void *pb)
{
    const struct cand *a = (const struct cand *)pa, *b = (const struct cand *)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->b < b->b) ? -1 : (a->b > b->b);
}

static int i32_cmp(const void *pa, const void *pb)
{
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

void qsa_oracle_select(const double *scores, int64_t ld, const int64_t *bt,
                       int64_t nrows, int k, int32_t *sel)
{
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t n = 0; n < nrows; ++n) {
        int64_t nc = bt[n];
        int32_t *out = sel + n * k;
        struct cand *c = (struct cand *)malloc((size_t)(nc > 0 ? nc : 1) * sizeof *c);
        for (int64_t b = 0; b < nc; ++b) {
            c[b].s = scores[n * ld + b];
            c[b].b = b;
        }
        qsort(c, (size_t)nc, sizeof *c, cand_cmp);
        int64_t take = nc < (int64_t)(k - 1) ? nc : (int64_t)(k - 1);
        for (int64_t j = 0; j < take; ++j)
            out[j] = (int32_t)c[j].b;
        out[take] = (int32_t)bt[n];
        qsort(out, (size_t)(take + 1), sizeof *out, i32_cmp);
        for (int64_t j = take + 1; j < k; ++j)
            out[j] = -1;
        free(c);
    }
}

/* Decode with multi-token prediction ("结果 2": decode at next_n = 4 with three MTP
 * steps; section 5, step 5: the MTP steps reuse the QSA top-k indices).  Reading
 * taken: ONE selection per sequence serves its next_n queries t = L - next_n ..
 * L - 1, made from the indexer scores of the last query (row n of `scores`, blocks
 * b < floor((L - 1) / r)).  Every query keeps its own trailing causal block (the
 * budget sentence), so the own blocks floor((L - next_n) / r) .. floor((L - 1) / r)
 * are all forced; the other slots, at most k minus their number, go to the best
 * blocks below the first of them (score descending, lower index first on ties).
 * Output ascending, padded with -1.  next_n = 1 is qsa_oracle_select. */
void qsa_oracle_select_shared(const double *scores, int64_t ld, const int64_t *L, int64_t nrows,
                              int next_n, int r, int k, int32_t *sel)
{
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t n = 0; n < nrows; ++n) {
        int32_t *out = sel + n * k;
        int64_t t_last = L[n] - 1, t_first = L[n] - next_n;
        if (t_first < 0) t_first = 0;
        int64_t b_first = t_first / r, b_last = t_last / r;
        int64_t nf = b_last - b_first + 1;
        struct cand *c = (struct cand *)malloc((size_t)(b_first > 0 ? b_first : 1) * sizeof *c);
        for (int64_t b = 0; b < b_first; ++b) {
            c[b].s = scores[n * ld + b];
            c[b].b = b;
        }
        qsort(c, (size_t)b_first, sizeof *c, cand_cmp);
        int64_t room = (int64_t)k - nf;
        if (room < 0) room = 0;
        int64_t take = b_first < room ? b_first : room;
        int64_t m = 0;
        for (int64_t j = 0; j < take; ++j)
            out[m++] = (int32_t)c[j].b;
        for (int64_t b = b_first; b <= b_last && m < k; ++b)
            out[m++] = (int32_t)b;
        qsort(out, (size_t)m, sizeof *out, i32_cmp);
        for (int64_t j = m; j < k; ++j)
            out[j] = -1;
        free(c);
    }
}

/* one query row, one head: softmax attention over an explicit token list */
static void attend_tokens(const double *qh, const uint16_t *k, const uint16_t *v,
                          int Hkv, int D, int g, double scale,
                          const int64_t *tok, int64_t ntok, double *o, double *lse)
{
    double *logit = (double *)malloc((size_t)(ntok > 0 ? ntok : 1) * sizeof *logit);
    double m = -INFINITY;
    for (int64_t n = 0; n < ntok; ++n) {
        const uint16_t *kj = k + (tok[n] * Hkv + g) * D;
        double dot = 0.0;
        for (int c = 0; c < D; ++c)
            dot += qh[c] * widen_bf16(kj[c]);
        logit[n] = dot * scale;
        if (logit[n] > m) m = logit[n];
    }
    double l = 0.0;
    for (int c = 0; c < D; ++c)
        o[c] = 0.0;
    for (int64_t n = 0; n < ntok; ++n) {
        double p = exp(logit[n] - m);
        l += p;
        const uint16_t *vj = v + (tok[n] * Hkv + g) * D;
        for (int c = 0; c < D; ++c)
            o[c] += p * widen_bf16(vj[c]);
    }
    for (int c = 0; c < D; ++c)
        o[c] /= l;
    *lse = m + log(l);
    free(logit);
}

/* ------------------------------------------------------------------------ */
/* [notes] expansion + sparse core attention: the token set of query t is the */
/* union over selected blocks b of [b r, b r + r) cut to j <= t; every head h  */
/* attends with its KV group g = h / (Hq / Hkv) (GQA, [table] 24 / 2 heads).   */
/* sel row n belongs to query row rows[n]; -1 entries are padding; a block    */
/* listed twice counts once (the token set is a set).                         */
/* ------------------------------------------------------------------------ */
void qsa_oracle_attend(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                       const int32_t *sel, int kb, int64_t Lq, int64_t Lk, int r,
                       int Hq, int Hkv, int D, double scale,
                       const int64_t *rows, int64_t nrows, double *o, double *lse)
{
    int grp = Hq / Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t n = 0; n < nrows; ++n) {
        int64_t i = rows[n];
        int64_t t = (Lk - Lq) + i;
        int32_t *blk = (int32_t *)malloc((size_t)kb * sizeof *blk);
        memcpy(blk, sel + n * kb, (size_t)kb * sizeof *blk);
        qsort(blk, (size_t)kb, sizeof *blk, i32_cmp);
        int64_t *tok = (int64_t *)malloc((size_t)kb * (size_t)r * sizeof *tok);
        int64_t ntok = 0;
        for (int j = 0; j < kb; ++j) {
            if (blk[j] < 0) continue;
            if (j > 0 && blk[j] == blk[j - 1]) continue;
            for (int u = 0; u < r; ++u) {
                int64_t tj = (int64_t)blk[j] * r + u;
                if (tj <= t && tj < Lk)
                    tok[ntok++] = tj;
            }
        }
        double qh[1024];
        for (int h = 0; h < Hq; ++h) {
            for (int c = 0; c < D; ++c)
                qh[c] = widen_bf16(q[(i * Hq + h) * D + c]);
            attend_tokens(qh, k, v, Hkv, D, h / grp, scale, tok, ntok,
                          o + (n * Hq + h) * D, lse + n * Hq + h);
        }
        free(tok);
        free(blk);
    }
}

/* ------------------------------------------------------------------------ */
/* Dense causal GQA attention, written as its own triple loop: query t sees   */
/* every key j <= t.  It is the baseline the pages compare QSA against.       */
/* ------------------------------------------------------------------------ */
void qsa_oracle_dense(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                      int64_t Lq, int64_t Lk, int Hq, int Hkv, int D, double scale,
                      const int64_t *rows, int64_t nrows, double *o, double *lse)
{
    int grp = Hq / Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t n = 0; n < nrows; ++n) {
        int64_t i = rows[n];
        int64_t t = (Lk - Lq) + i;
        double *logit = (double *)malloc((size_t)(t + 1) * sizeof *logit);
        for (int h = 0; h < Hq; ++h) {
            int g = h / grp;
            double m = -INFINITY;
            for (int64_t j = 0; j <= t; ++j) {
                double dot = 0.0;
                for (int c = 0; c < D; ++c)
                    dot += widen_bf16(q[(i * Hq + h) * D + c]) * widen_bf16(k[(j * Hkv + g) * D + c]);
                logit[j] = dot * scale;
                if (logit[j] > m) m = logit[j];
            }
            double l = 0.0;
            double *oh = o + (n * Hq + h) * D;
            for (int c = 0; c < D; ++c) oh[c] = 0.0;
            for (int64_t j = 0; j <= t; ++j) {
                double p = exp(logit[j] - m);
                l += p;
                for (int c = 0; c < D; ++c)
                    oh[c] += p * widen_bf16(v[(j * Hkv + g) * D + c]);
            }
            for (int c = 0; c < D; ++c) oh[c] /= l;
            lse[n * Hq + h] = m + log(l);
        }
        free(logit);
    }
}

int qsa_oracle_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
