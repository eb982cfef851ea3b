/*
 * oracle.c -- plain CPU reference for causal sparse attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header or constant with the CUDA
 * library.
 *
 * Every function is the textbook definition written out with plain loops:
 * integer scores in int64, attention in fp64 (bf16 inputs are widened
 * exactly), top-k by a full sort with ties broken towards the lower index.
 * There is no blocking, fusion or reordering beyond what a definition states.
 * OpenMP is used only to run independent query rows in parallel.
 *
 * Sources (page title, section):
 *  - "IndexCache: inferencia 82% mas rapida en ..." (body): a lightweight
 *    indexer scores earlier tokens and each query keeps a small top-scoring
 *    subset; F layers run the indexer, S layers reuse the nearest preceding
 *    F layer's indices.
 *  - "SpatialLM-Mini acelero el entrenamiento ..." (section "Como eligen los
 *    tokens a quien escuchar"): the fixed set is the token itself, a few near
 *    predecessors and positions at distances 1, 2, 4, 8, ...; never a future
 *    position; weights from learnable 3-D query/key coordinates, a smaller
 *    distance giving a larger weight.
 *  - "Xiaomi presenta HySparse2 ..." (sections "Dos niveles para compartir la
 *    cache", "Mas precision con menos memoria"): token-level selection with
 *    the most recent tokens forced into the selected set.
 *  - "NVIDIA AI Research presenta Star Attention ..." (body): per-block
 *    attention results are merged by a distributed softmax.
 *  - "Native Sparse Attention ..." (section "Puntos Clave"): coarse token
 *    compression, fine-grained blockwise selection and a sliding window.
 *
 * Return codes: 0 ok, 1 invalid argument / inconsistent sizes, 2 an index
 * that is out of range or refers to a future position.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>

#define OR_OK 0
#define OR_BAD_ARG 1
#define OR_BAD_INDEX 2

/* bf16 bit pattern -> fp64, exact (bf16 is the upper half of an IEEE float). */
static double bf16_to_f64(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Row list helper: rows == NULL means every flat row 0..n_all-1. */
static int64_t row_at(const int64_t *rows, int64_t i) { return rows ? rows[i] : i; }

/* ------------------------------------------------------------------------ */
/* Indexer score (IndexCache page, body; formula of the tiny DSA workload):  */
/*   I(t, j) = sum_h w[t,h] * max(0, sum_c q[t,h,c] * k[j,c])                */
/* in int64, one indexer key per token shared by every indexer head.         */
/* ------------------------------------------------------------------------ */
static int64_t indexer_score(const int8_t *q_row, const int8_t *k_row,
                             const int32_t *w_row, int64_t Hi, int64_t di)
{
    int64_t total = 0;
    for (int64_t h = 0; h < Hi; ++h) {
        int64_t dot = 0;
        for (int64_t c = 0; c < di; ++c)
            dot += (int64_t)q_row[h * di + c] * (int64_t)k_row[c];
        if (dot > 0)
            total += (int64_t)w_row[h] * dot;
    }
    return total;
}

/*
 * Scores of every key j <= pos(t) for the requested rows; keys after the
 * query position are set to INT64_MIN.  Flat row r = b*Tq + t, pos = q_pos0+t.
 * out: [n_rows, L].
 */
int oracle_indexer_scores(const int8_t *q, const int8_t *k, const int32_t *w,
                          int64_t B, int64_t Tq, int64_t L, int64_t Hi, int64_t di,
                          int64_t q_pos0, const int64_t *rows, int64_t n_rows,
                          int64_t *out)
{
    if (B <= 0 || Tq <= 0 || L <= 0 || Hi <= 0 || di <= 0 || q_pos0 < 0)
        return OR_BAD_ARG;
    if (q_pos0 + Tq - 1 >= L)
        return OR_BAD_ARG;
    if (!rows) n_rows = B * Tq;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < n_rows; ++i) {
        int64_t r = row_at(rows, i);
        if (r < 0 || r >= B * Tq) { bad = 1; continue; }
        int64_t b = r / Tq, t = r % Tq, pos = q_pos0 + t;
        const int8_t *q_row = q + r * Hi * di;
        const int32_t *w_row = w + r * Hi;
        for (int64_t j = 0; j < L; ++j)
            out[i * L + j] = (j <= pos)
                ? indexer_score(q_row, k + (b * L + j) * di, w_row, Hi, di)
                : INT64_MIN;
    }
    return bad ? OR_BAD_ARG : OR_OK;
}

typedef struct { int64_t score; int64_t j; } cand_t;

/* Order: larger score first; equal scores -> lower index first. */
static int cand_cmp(const void *a, const void *b)
{
    const cand_t *x = (const cand_t *)a, *y = (const cand_t *)b;
    if (x->score != y->score) return x->score > y->score ? -1 : 1;
    return (x->j > y->j) - (x->j < y->j);
}

static int i32_cmp(const void *a, const void *b)
{
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/*
 * Causal top-k with a forced recent window.
 * W_t = {max(0, p-window+1) .. p} (empty when window == 0) is always kept
 * (HySparse2 page: the most recent tokens are forced into the selected set);
 * the remaining candidates C_t = {0..p} \ W_t are fully sorted by
 * (score desc, index asc) and the first min(topk, |C_t|) are kept (IndexCache
 * page: a small top-scoring subset).  Output row: ascending positions of
 * W_t u chosen, padded with -1 to topk+window; out_count = valid length.
 */
int oracle_indexer_topk(const int8_t *q, const int8_t *k, const int32_t *w,
                        int64_t B, int64_t Tq, int64_t L, int64_t Hi, int64_t di,
                        int64_t q_pos0, int64_t topk, int64_t window,
                        const int64_t *rows, int64_t n_rows,
                        int32_t *out_idx, int32_t *out_count)
{
    if (B <= 0 || Tq <= 0 || L <= 0 || Hi <= 0 || di <= 0 || q_pos0 < 0 ||
        topk < 0 || window < 0 || topk + window <= 0)
        return OR_BAD_ARG;
    if (q_pos0 + Tq - 1 >= L)
        return OR_BAD_ARG;
    if (!rows) n_rows = B * Tq;
    const int64_t K = topk + window;
    int bad = 0;
#pragma omp parallel
    {
        cand_t *cand = (cand_t *)malloc(sizeof(cand_t) * (size_t)L);
        int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)K);
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < n_rows; ++i) {
            int64_t r = row_at(rows, i);
            if (r < 0 || r >= B * Tq || !cand || !sel) { bad = 1; continue; }
            int64_t b = r / Tq, t = r % Tq, p = q_pos0 + t;
            const int8_t *q_row = q + r * Hi * di;
            const int32_t *w_row = w + r * Hi;
            int64_t w_lo = window > 0 ? (p - window + 1 > 0 ? p - window + 1 : 0) : p + 1;
            /* candidates: 0 .. w_lo-1 */
            int64_t n_c = 0;
            for (int64_t j = 0; j < w_lo; ++j) {
                cand[n_c].score = indexer_score(q_row, k + (b * L + j) * di, w_row, Hi, di);
                cand[n_c].j = j;
                ++n_c;
            }
            qsort(cand, (size_t)n_c, sizeof(cand_t), cand_cmp);
            int64_t n_take = n_c < topk ? n_c : topk;
            int64_t n_sel = 0;
            for (int64_t m = 0; m < n_take; ++m) sel[n_sel++] = (int32_t)cand[m].j;
            for (int64_t j = w_lo; j <= p; ++j) sel[n_sel++] = (int32_t)j;
            qsort(sel, (size_t)n_sel, sizeof(int32_t), i32_cmp);
            for (int64_t m = 0; m < K; ++m)
                out_idx[i * K + m] = m < n_sel ? sel[m] : -1;
            if (out_count) out_count[i] = (int32_t)n_sel;
        }
        free(cand);
        free(sel);
    }
    return bad ? OR_BAD_ARG : OR_OK;
}

/*
 * Fixed graph of the SpatialLM page ("Como eligen los tokens a quien
 * escuchar"): the token itself, its nearest predecessors and the positions at
 * distances 1, 2, 4, 8, ... ; no future position.  With the workload's
 * parameters: S_p = {p-o : 0 <= o < window, p-o >= 0}  u  {p - 2^i : 2^i < p}
 * (the dilated part only when `dilated` is non-zero).  Output ascending,
 * de-duplicated, padded with -1 to `cap`; returns the set size or -1 when
 * `cap` is too small.
 */
int64_t oracle_fixed_graph_row(int64_t p, int64_t window, int dilated,
                               int32_t *out, int64_t cap)
{
    int64_t n = 0;
    /* membership by a plain scan of every earlier position */
    for (int64_t j = 0; j <= p; ++j) {
        int64_t o = p - j;
        int in = (o < window);
        if (!in && dilated) {
            /* is o a power of two with o < p ? */
            if (o > 0 && (o & (o - 1)) == 0 && o < p) in = 1;
        }
        if (in) {
            if (n >= cap) return -1;
            out[n++] = (int32_t)j;
        }
    }
    for (int64_t m = n; m < cap; ++m) out[m] = -1;
    return n;
}

/*
 * Attention over an explicit per-query index list (the operation every page
 * reduces to once the index set is fixed).
 *   q [B,Tq,Hq,d], k/v [B,L,Hkv,d] as bf16 bit patterns.
 *   idx [B,Tq,idx_heads,K] int32, -1 = padding; idx_heads is 1 (one list for
 *   every head) or Hkv (one list per KV head).  Query head h reads KV head
 *   h / (Hq/Hkv).
 *   Optional coordinate bias (SpatialLM page): cq [B,Tq,Hq,3], ck [B,L,Hkv,3],
 *   beta [Hq]; bias = -beta_h * ||cq - ck||^2, added after scaling.
 * For each row r and head h:
 *   z_j = scale * (q . k_j) + bias_j,   lse = log sum_j exp z_j,
 *   o = sum_j exp(z_j - lse) v_j,       psum = sum_j exp(z_j - lse).
 * An empty list gives o = 0, lse = -inf, psum = 0.  maxj[i] is the largest
 * position any head of row i read (-1 if none).
 * Outputs: out [n_rows,Hq,d], lse [n_rows,Hq], psum [n_rows,Hq] (nullable),
 * maxj [n_rows] (nullable).
 */
int oracle_sparse_attn(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                       int64_t B, int64_t Tq, int64_t L, int64_t Hq, int64_t Hkv,
                       int64_t d, int64_t q_pos0,
                       const int32_t *idx, int64_t idx_heads, int64_t K,
                       const float *cq, const float *ck, const float *beta,
                       double scale, const int64_t *rows, int64_t n_rows,
                       double *out, double *lse, double *psum, int64_t *maxj)
{
    if (B <= 0 || Tq <= 0 || L <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || K < 0 ||
        Hq % Hkv != 0 || q_pos0 < 0 || !(idx_heads == 1 || idx_heads == Hkv))
        return OR_BAD_ARG;
    if ((cq || ck || beta) && !(cq && ck && beta))
        return OR_BAD_ARG;
    if (!rows) n_rows = B * Tq;
    const int64_t G = Hq / Hkv;
    int status = OR_OK;
#pragma omp parallel
    {
        double *z = (double *)malloc(sizeof(double) * (size_t)(K > 0 ? K : 1));
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < n_rows; ++i) {
            int64_t r = row_at(rows, i);
            if (r < 0 || r >= B * Tq || !z) { status = OR_BAD_ARG; continue; }
            int64_t b = r / Tq, t = r % Tq, pos = q_pos0 + t;
            int64_t row_max = -1;
            for (int64_t h = 0; h < Hq; ++h) {
                int64_t g = h / G;
                const int32_t *list = idx + (r * idx_heads + (idx_heads == 1 ? 0 : g)) * K;
                const uint16_t *qv = q + (r * Hq + h) * d;
                double m = -INFINITY;
                for (int64_t e = 0; e < K; ++e) {
                    int64_t j = list[e];
                    if (j < 0) { z[e] = -INFINITY; continue; }
                    if (j >= L || j > pos) { status = OR_BAD_INDEX; z[e] = -INFINITY; continue; }
                    if (j > row_max) row_max = j;
                    const uint16_t *kv = k + ((b * L + j) * Hkv + g) * d;
                    double dot = 0.0;
                    for (int64_t c = 0; c < d; ++c)
                        dot += bf16_to_f64(qv[c]) * bf16_to_f64(kv[c]);
                    double zz = scale * dot;
                    if (cq) {
                        const float *a = cq + (r * Hq + h) * 3;
                        const float *bb = ck + ((b * L + j) * Hkv + g) * 3;
                        double dist2 = 0.0;
                        for (int c = 0; c < 3; ++c) {
                            double diff = (double)a[c] - (double)bb[c];
                            dist2 += diff * diff;
                        }
                        zz -= (double)beta[h] * dist2;
                    }
                    z[e] = zz;
                    if (zz > m) m = zz;
                }
                double *o = out + (i * Hq + h) * d;
                for (int64_t c = 0; c < d; ++c) o[c] = 0.0;
                if (m == -INFINITY) {
                    lse[i * Hq + h] = -INFINITY;
                    if (psum) psum[i * Hq + h] = 0.0;
                    continue;
                }
                double s = 0.0;
                for (int64_t e = 0; e < K; ++e)
                    if (z[e] != -INFINITY) s += exp(z[e] - m);
                double l = m + log(s);
                double ps = 0.0;
                for (int64_t e = 0; e < K; ++e) {
                    if (z[e] == -INFINITY) continue;
                    double p = exp(z[e] - l);
                    ps += p;
                    const uint16_t *vv = v + ((b * L + list[e]) * Hkv + g) * d;
                    for (int64_t c = 0; c < d; ++c) o[c] += p * bf16_to_f64(vv[c]);
                }
                lse[i * Hq + h] = l;
                if (psum) psum[i * Hq + h] = ps;
            }
            if (maxj) maxj[i] = row_max;
        }
        free(z);
    }
    return status;
}

/*
 * Backward of attention over explicit index lists (the gradient of the
 * forward above without a bias; the training results of the SpatialLM page,
 * "SpatialLM-Mini acelero el entrenamiento ...", and the backward speed-up of
 * the NSA page, "Puntos Clave", need it).  For each row r and head h with
 * p_j = exp(z_j - lse), z_j = scale * (q . k_j):
 *   dP_j = dO . v_j,   D = sum_j p_j dP_j,   dS_j = p_j (dP_j - D),
 *   dq  = scale * sum_j dS_j k_j,
 *   dk_j += scale * dS_j q,     dv_j += p_j dO
 * (a key listed twice contributes twice).  The forward is recomputed here in
 * fp64; dout is bf16, widened exactly.  Rows run in parallel; dk and dv are
 * accumulated with atomic adds.  dq [B,Tq,Hq,d], dk/dv [B,L,Hkv,d], all fp64.
 */
int oracle_sparse_attn_bwd(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                           const uint16_t *dout, int64_t B, int64_t Tq, int64_t L,
                           int64_t Hq, int64_t Hkv, int64_t d, int64_t q_pos0,
                           const int32_t *idx, int64_t idx_heads, int64_t K, double scale,
                           double *dq, double *dk, double *dv)
{
    if (B <= 0 || Tq <= 0 || L <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || K < 0 ||
        Hq % Hkv != 0 || q_pos0 < 0 || !(idx_heads == 1 || idx_heads == Hkv))
        return OR_BAD_ARG;
    const int64_t G = Hq / Hkv;
    for (int64_t e = 0; e < B * L * Hkv * d; ++e) { dk[e] = 0.0; dv[e] = 0.0; }
    int status = OR_OK;
#pragma omp parallel
    {
        double *z = (double *)malloc(sizeof(double) * (size_t)(K > 0 ? K : 1));
        double *dp = (double *)malloc(sizeof(double) * (size_t)(K > 0 ? K : 1));
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < B * Tq; ++r) {
            if (!z || !dp) { status = OR_BAD_ARG; continue; }
            int64_t b = r / Tq, t = r % Tq, pos = q_pos0 + t;
            for (int64_t h = 0; h < Hq; ++h) {
                int64_t g = h / G;
                const int32_t *list = idx + (r * idx_heads + (idx_heads == 1 ? 0 : g)) * K;
                const uint16_t *qv = q + (r * Hq + h) * d;
                const uint16_t *dov = dout + (r * Hq + h) * d;
                double *dqv = dq + (r * Hq + h) * d;
                for (int64_t c = 0; c < d; ++c) dqv[c] = 0.0;
                /* forward: logits and their log-sum-exp */
                double m = -INFINITY;
                for (int64_t e = 0; e < K; ++e) {
                    int64_t j = list[e];
                    z[e] = -INFINITY;
                    if (j < 0) continue;
                    if (j >= L || j > pos) { status = OR_BAD_INDEX; continue; }
                    const uint16_t *kv = k + ((b * L + j) * Hkv + g) * d;
                    double dot = 0.0;
                    for (int64_t c = 0; c < d; ++c) dot += bf16_to_f64(qv[c]) * bf16_to_f64(kv[c]);
                    z[e] = scale * dot;
                    if (z[e] > m) m = z[e];
                }
                if (m == -INFINITY) continue;              /* empty set: no gradient */
                double s = 0.0;
                for (int64_t e = 0; e < K; ++e)
                    if (z[e] != -INFINITY) s += exp(z[e] - m);
                const double lse = m + log(s);
                /* dP_j and D */
                double D = 0.0;
                for (int64_t e = 0; e < K; ++e) {
                    if (z[e] == -INFINITY) continue;
                    const uint16_t *vv = v + ((b * L + list[e]) * Hkv + g) * d;
                    double x = 0.0;
                    for (int64_t c = 0; c < d; ++c) x += bf16_to_f64(dov[c]) * bf16_to_f64(vv[c]);
                    dp[e] = x;
                    D += exp(z[e] - lse) * x;
                }
                /* dS_j, then dq, dk_j and dv_j */
                for (int64_t e = 0; e < K; ++e) {
                    if (z[e] == -INFINITY) continue;
                    const int64_t j = list[e];
                    const double p = exp(z[e] - lse);
                    const double ds = p * (dp[e] - D);
                    const uint16_t *kv = k + ((b * L + j) * Hkv + g) * d;
                    double *dkv = dk + ((b * L + j) * Hkv + g) * d;
                    double *dvv = dv + ((b * L + j) * Hkv + g) * d;
                    for (int64_t c = 0; c < d; ++c) {
                        dqv[c] += scale * ds * bf16_to_f64(kv[c]);
                        const double a = scale * ds * bf16_to_f64(qv[c]);
                        const double bv = p * bf16_to_f64(dov[c]);
#pragma omp atomic
                        dkv[c] += a;
#pragma omp atomic
                        dvv[c] += bv;
                    }
                }
            }
        }
        free(z);
        free(dp);
    }
    return status;
}

/*
 * Distributed-softmax merge (Star Attention page, body): partial results
 * (O_s, lse_s) over disjoint pieces of one softmax are combined as
 *   lse = log sum_s exp(lse_s),   O = sum_s exp(lse_s - lse) O_s.
 * A piece with lse_s = -inf contributes nothing; all empty -> O = 0,
 * lse = -inf.  part_o [n_split, rows, d], part_lse [n_split, rows].
 */
int oracle_lse_combine(const double *part_o, const double *part_lse,
                       int64_t n_split, int64_t rows, int64_t d,
                       double *out, double *lse)
{
    if (n_split <= 0 || rows < 0 || d <= 0) return OR_BAD_ARG;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        double m = -INFINITY;
        for (int64_t s = 0; s < n_split; ++s)
            if (part_lse[s * rows + r] > m) m = part_lse[s * rows + r];
        double *o = out + r * d;
        for (int64_t c = 0; c < d; ++c) o[c] = 0.0;
        if (m == -INFINITY) { lse[r] = -INFINITY; continue; }
        double acc = 0.0;
        for (int64_t s = 0; s < n_split; ++s)
            if (part_lse[s * rows + r] != -INFINITY) acc += exp(part_lse[s * rows + r] - m);
        double l = m + log(acc);
        for (int64_t s = 0; s < n_split; ++s) {
            double ls = part_lse[s * rows + r];
            if (ls == -INFINITY) continue;
            double f = exp(ls - l);
            for (int64_t c = 0; c < d; ++c) o[c] += f * part_o[(s * rows + r) * d + c];
        }
        lse[r] = l;
    }
    return OR_OK;
}

/* ------------------------------------------------------------------------ */
/* NSA (Native Sparse Attention page, "Puntos Clave" and "Analisis            */
/* Profundo"): coarse compression, blockwise selection, sliding window.       */
/* ------------------------------------------------------------------------ */

/* Number of compressed tokens: windows [i*stride, i*stride+len) inside [0,T). */
static int64_t nsa_n_cmp(int64_t T, int64_t len, int64_t stride)
{
    return T >= len ? (T - len) / stride + 1 : 0;
}

/*
 * Compression: Kc[b,i,g,:] = mean of K[b, i*stride + u, g, :] for u < len
 * (and likewise Vc), computed in fp64.  kc/vc: [B, n_cmp, Hkv, d] fp64.
 */
int oracle_nsa_compress(const uint16_t *k, const uint16_t *v, int64_t B, int64_t T,
                        int64_t Hkv, int64_t d, int64_t len, int64_t stride,
                        double *kc, double *vc)
{
    if (B <= 0 || T <= 0 || Hkv <= 0 || d <= 0 || len <= 0 || stride <= 0) return OR_BAD_ARG;
    int64_t nc = nsa_n_cmp(T, len, stride);
#pragma omp parallel for schedule(static)
    for (int64_t bi = 0; bi < B * nc; ++bi) {
        int64_t b = bi / nc, i = bi % nc;
        for (int64_t g = 0; g < Hkv; ++g)
            for (int64_t c = 0; c < d; ++c) {
                double sk = 0.0, sv = 0.0;
                for (int64_t u = 0; u < len; ++u) {
                    int64_t j = i * stride + u;
                    sk += bf16_to_f64(k[((b * T + j) * Hkv + g) * d + c]);
                    sv += bf16_to_f64(v[((b * T + j) * Hkv + g) * d + c]);
                }
                kc[((b * nc + i) * Hkv + g) * d + c] = sk / (double)len;
                vc[((b * nc + i) * Hkv + g) * d + c] = sv / (double)len;
            }
    }
    return OR_OK;
}

/* softmax attention of one query vector over a list of fp64 key rows */
static void attend_f64(const double *qv, int64_t d, double scale,
                       const double *const *krows, const double *const *vrows,
                       int64_t n, double *z, double *o, double *lse_out)
{
    for (int64_t c = 0; c < d; ++c) o[c] = 0.0;
    if (n == 0) { *lse_out = -INFINITY; return; }
    double m = -INFINITY;
    for (int64_t e = 0; e < n; ++e) {
        double dot = 0.0;
        for (int64_t c = 0; c < d; ++c) dot += qv[c] * krows[e][c];
        z[e] = scale * dot;
        if (z[e] > m) m = z[e];
    }
    double s = 0.0;
    for (int64_t e = 0; e < n; ++e) s += exp(z[e] - m);
    double l = m + log(s);
    for (int64_t e = 0; e < n; ++e) {
        double p = exp(z[e] - l);
        z[e] = p; /* leave probabilities behind for the caller */
        for (int64_t c = 0; c < d; ++c) o[c] += p * vrows[e][c];
    }
    *lse_out = l;
}

/*
 * Full NSA forward for the requested rows (flat r = b*T + t, position t).
 *  1. Compressed branch: keys Kc_i visible iff i*stride + len - 1 <= t.
 *  2. Importance of selection block b for KV group g:
 *       imp[b] = sum_{h in g} sum_{i : b*sel_block <= i*stride < (b+1)*sel_block}
 *                p_cmp[h, i]
 *     (p_cmp = compressed-branch softmax probabilities, 0 for invisible i).
 *  3. Selection: candidates b with b*sel_block <= t, top sel_topk by
 *     (imp desc, b asc); fewer candidates -> all.  Stored ascending, -1 pad.
 *     sel_override (nullable, same layout) replaces the computed choice.
 *  4. Selected branch: keys of the chosen blocks, masked to j <= t.
 *  5. Window branch: keys max(0, t-window+1) .. t.
 *  6. out = g_c * o_cmp + g_s * o_slc + g_w * o_win   (gates already sigmoid).
 * Outputs (all nullable except out): out [n_rows,Hq,d], o_branch [3,n_rows,Hq,d],
 * lse_branch [n_rows,Hq,3], sel_idx [n_rows,Hkv,sel_topk],
 * imp_out [n_rows,Hkv,n_blocks] with n_blocks = ceil(T/sel_block).
 */
int oracle_nsa_fwd(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                   const float *gates, int64_t B, int64_t T, int64_t Hq, int64_t Hkv,
                   int64_t d, int64_t cmp_len, int64_t cmp_stride, int64_t sel_block,
                   int64_t sel_topk, int64_t window, double scale,
                   const int64_t *rows, int64_t n_rows, const int32_t *sel_override,
                   double *out, double *o_branch, double *lse_branch,
                   int32_t *sel_idx, double *imp_out)
{
    if (B <= 0 || T <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || Hq % Hkv != 0 ||
        cmp_len <= 0 || cmp_stride <= 0 || sel_block <= 0 || sel_topk <= 0 || window <= 0)
        return OR_BAD_ARG;
    if (!rows) n_rows = B * T;
    const int64_t G = Hq / Hkv;
    const int64_t nc = nsa_n_cmp(T, cmp_len, cmp_stride);
    const int64_t nb = (T + sel_block - 1) / sel_block;
    double *kc = (double *)malloc(sizeof(double) * (size_t)(B * (nc > 0 ? nc : 1) * Hkv * d));
    double *vc = (double *)malloc(sizeof(double) * (size_t)(B * (nc > 0 ? nc : 1) * Hkv * d));
    if (!kc || !vc) { free(kc); free(vc); return OR_BAD_ARG; }
    if (nc > 0) oracle_nsa_compress(k, v, B, T, Hkv, d, cmp_len, cmp_stride, kc, vc);
    int status = OR_OK;
#pragma omp parallel
    {
        /* key buffers: the selected branch holds at most sel_topk*sel_block
           rows, the window branch at most `window`, the compressed branch nc */
        int64_t nbuf = sel_topk * sel_block > window ? sel_topk * sel_block : window;
        int64_t nmax = (nc > nbuf ? nc : nbuf) + 1;
        double *z = (double *)malloc(sizeof(double) * (size_t)nmax);
        const double **kr = (const double **)malloc(sizeof(double *) * (size_t)nmax);
        const double **vr = (const double **)malloc(sizeof(double *) * (size_t)nmax);
        double *kbuf = (double *)malloc(sizeof(double) * (size_t)((nbuf + 1) * d));
        double *vbuf = (double *)malloc(sizeof(double) * (size_t)((nbuf + 1) * d));
        double *qv = (double *)malloc(sizeof(double) * (size_t)d);
        double *ob = (double *)malloc(sizeof(double) * (size_t)(3 * Hq * d));
        double *lb = (double *)malloc(sizeof(double) * (size_t)(3 * Hq));
        double *imp = (double *)malloc(sizeof(double) * (size_t)(Hkv * nb));
        int64_t *cand = (int64_t *)malloc(sizeof(int64_t) * (size_t)nb);
        int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)(Hkv * sel_topk));
        int ok = z && kr && vr && kbuf && vbuf && qv && ob && lb && imp && cand && sel;
#pragma omp for schedule(dynamic, 1)
        for (int64_t ii = 0; ii < n_rows; ++ii) {
            int64_t r = row_at(rows, ii);
            if (!ok || r < 0 || r >= B * T) { status = OR_BAD_ARG; continue; }
            int64_t b = r / T, t = r % T;
            for (int64_t e = 0; e < Hkv * nb; ++e) imp[e] = 0.0;
            /* 1 + 2: compressed branch and block importance */
            int64_t n_vis = 0;
            while (n_vis < nc && n_vis * cmp_stride + cmp_len - 1 <= t) ++n_vis;
            for (int64_t h = 0; h < Hq; ++h) {
                int64_t g = h / G;
                for (int64_t c = 0; c < d; ++c) qv[c] = bf16_to_f64(q[((r)*Hq + h) * d + c]);
                for (int64_t i = 0; i < n_vis; ++i) {
                    kr[i] = kc + ((b * nc + i) * Hkv + g) * d;
                    vr[i] = vc + ((b * nc + i) * Hkv + g) * d;
                }
                attend_f64(qv, d, scale, kr, vr, n_vis, z, ob + (0 * Hq + h) * d, lb + 0 * Hq + h);
                for (int64_t i = 0; i < n_vis; ++i) {
                    int64_t blk = (i * cmp_stride) / sel_block;
                    imp[g * nb + blk] += z[i];
                }
            }
            /* 3: block selection per KV group */
            for (int64_t g = 0; g < Hkv; ++g) {
                int32_t *sg = sel + g * sel_topk;
                if (sel_override) {
                    for (int64_t m = 0; m < sel_topk; ++m)
                        sg[m] = sel_override[(ii * Hkv + g) * sel_topk + m];
                } else {
                    int64_t n_cand = 0;
                    for (int64_t blk = 0; blk < nb && blk * sel_block <= t; ++blk)
                        cand[n_cand++] = blk;
                    /* selection sort by (imp desc, b asc): plain and exact */
                    int64_t n_take = n_cand < sel_topk ? n_cand : sel_topk;
                    for (int64_t m = 0; m < n_take; ++m) {
                        int64_t best = m;
                        for (int64_t e = m + 1; e < n_cand; ++e) {
                            double ie = imp[g * nb + cand[e]], ib = imp[g * nb + cand[best]];
                            if (ie > ib || (ie == ib && cand[e] < cand[best])) best = e;
                        }
                        int64_t tmp = cand[m]; cand[m] = cand[best]; cand[best] = tmp;
                    }
                    for (int64_t m = 0; m < sel_topk; ++m) sg[m] = m < n_take ? (int32_t)cand[m] : -1;
                    qsort(sg, (size_t)n_take, sizeof(int32_t), i32_cmp);
                }
                if (sel_idx)
                    for (int64_t m = 0; m < sel_topk; ++m) sel_idx[(ii * Hkv + g) * sel_topk + m] = sg[m];
                if (imp_out)
                    for (int64_t blk = 0; blk < nb; ++blk) imp_out[(ii * Hkv + g) * nb + blk] = imp[g * nb + blk];
            }
            /* 4 + 5: selected and window branches over raw keys */
            for (int64_t h = 0; h < Hq; ++h) {
                int64_t g = h / G;
                for (int64_t c = 0; c < d; ++c) qv[c] = bf16_to_f64(q[(r * Hq + h) * d + c]);
                int64_t n = 0;
                const int32_t *sg = sel + g * sel_topk;
                for (int64_t m = 0; m < sel_topk; ++m) {
                    int64_t blk = sg[m];
                    if (blk < 0) continue;
                    if (blk >= nb) { status = OR_BAD_INDEX; continue; }
                    for (int64_t j = blk * sel_block; j < (blk + 1) * sel_block && j <= t && j < T; ++j) {
                        for (int64_t c = 0; c < d; ++c) {
                            kbuf[n * d + c] = bf16_to_f64(k[((b * T + j) * Hkv + g) * d + c]);
                            vbuf[n * d + c] = bf16_to_f64(v[((b * T + j) * Hkv + g) * d + c]);
                        }
                        kr[n] = kbuf + n * d; vr[n] = vbuf + n * d; ++n;
                    }
                }
                attend_f64(qv, d, scale, kr, vr, n, z, ob + (1 * Hq + h) * d, lb + 1 * Hq + h);
                n = 0;
                int64_t lo = t - window + 1 > 0 ? t - window + 1 : 0;
                for (int64_t j = lo; j <= t; ++j) {
                    for (int64_t c = 0; c < d; ++c) {
                        kbuf[n * d + c] = bf16_to_f64(k[((b * T + j) * Hkv + g) * d + c]);
                        vbuf[n * d + c] = bf16_to_f64(v[((b * T + j) * Hkv + g) * d + c]);
                    }
                    kr[n] = kbuf + n * d; vr[n] = vbuf + n * d; ++n;
                }
                attend_f64(qv, d, scale, kr, vr, n, z, ob + (2 * Hq + h) * d, lb + 2 * Hq + h);
            }
            /* 6: gated sum */
            for (int64_t h = 0; h < Hq; ++h) {
                const float *gt = gates + (r * Hq + h) * 3;
                for (int64_t c = 0; c < d; ++c) {
                    double acc = 0.0;
                    for (int br = 0; br < 3; ++br) acc += (double)gt[br] * ob[(br * Hq + h) * d + c];
                    out[(ii * Hq + h) * d + c] = acc;
                }
                if (lse_branch)
                    for (int br = 0; br < 3; ++br) lse_branch[(ii * Hq + h) * 3 + br] = lb[br * Hq + h];
                if (o_branch)
                    for (int br = 0; br < 3; ++br)
                        for (int64_t c = 0; c < d; ++c)
                            o_branch[((br * n_rows + ii) * Hq + h) * d + c] = ob[(br * Hq + h) * d + c];
            }
        }
        free(z); free(kr); free(vr); free(kbuf); free(vbuf); free(qv); free(ob); free(lb);
        free(imp); free(cand); free(sel);
    }
    free(kc);
    free(vc);
    return status;
}

/*
 * Backward of one softmax branch for one query vector (the gradient of
 * attend_f64's output o for an upstream gradient dob):
 *   dP_e = dob . v_e,   D = sum_e p_e dP_e,   dS_e = p_e (dP_e - D)
 *   dq += scale sum_e dS_e k_e,   dk_e += scale dS_e q,   dv_e += p_e dob
 * p holds the branch's probabilities; dk/dv rows are shared between query
 * rows, so their updates are atomic.
 */
static void attend_bwd_f64(const double *qv, const double *dob, int64_t d, double scale,
                           const double *const *krows, const double *const *vrows,
                           const double *p, int64_t n, double *dq,
                           double *const *dkrows, double *const *dvrows)
{
    double D = 0.0;
    for (int64_t e = 0; e < n; ++e) {
        double x = 0.0;
        for (int64_t c = 0; c < d; ++c) x += dob[c] * vrows[e][c];
        D += p[e] * x;
    }
    for (int64_t e = 0; e < n; ++e) {
        double x = 0.0;
        for (int64_t c = 0; c < d; ++c) x += dob[c] * vrows[e][c];
        const double ds = p[e] * (x - D);
        for (int64_t c = 0; c < d; ++c) {
            dq[c] += scale * ds * krows[e][c];
            const double a = scale * ds * qv[c];
            const double bv = p[e] * dob[c];
#pragma omp atomic
            dkrows[e][c] += a;
#pragma omp atomic
            dvrows[e][c] += bv;
        }
    }
}

/*
 * NSA backward (Native Sparse Attention page, "Puntos Clave": the method is
 * trained natively and its backward pass is accelerated).  The gradient of
 * oracle_nsa_fwd's out for an upstream gradient dout, with the block choice
 * sel (the forward's sel_idx, [B*T, Hkv, sel_topk]) held fixed: the choice
 * is piecewise constant in the inputs, so no gradient flows through the
 * importance or the top-k.  Per row and head, for branch br with gate g_br
 * (the post-sigmoid value the forward multiplied by):
 *   dgates[br] = dout . o_br,   the branch's upstream gradient is g_br dout,
 * pushed through that branch's softmax (attend_bwd_f64).  The compressed
 * branch's key gradients land on the compressed rows Kc_i, Vc_i; since
 * Kc_i is the mean of K[i*stride .. i*stride+len-1], each of those rows
 * then receives dKc_i / len (likewise V).
 * Outputs: dq [B*T,Hq,d], dk/dv [B,T,Hkv,d], dgates [B*T,Hq,3], fp64.
 */
int oracle_nsa_bwd(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                   const float *gates, const uint16_t *dout, const int32_t *sel,
                   int64_t B, int64_t T, int64_t Hq, int64_t Hkv, int64_t d,
                   int64_t cmp_len, int64_t cmp_stride, int64_t sel_block,
                   int64_t sel_topk, int64_t window, double scale,
                   double *dq, double *dk, double *dv, double *dgates)
{
    if (B <= 0 || T <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || Hq % Hkv != 0 ||
        cmp_len <= 0 || cmp_stride <= 0 || sel_block <= 0 || sel_topk <= 0 || window <= 0)
        return OR_BAD_ARG;
    const int64_t G = Hq / Hkv;
    const int64_t nc = nsa_n_cmp(T, cmp_len, cmp_stride);
    const int64_t nb = (T + sel_block - 1) / sel_block;
    const int64_t ncs = nc > 0 ? nc : 1;
    double *kc = (double *)malloc(sizeof(double) * (size_t)(B * ncs * Hkv * d));
    double *vc = (double *)malloc(sizeof(double) * (size_t)(B * ncs * Hkv * d));
    double *dkc = (double *)calloc((size_t)(B * ncs * Hkv * d), sizeof(double));
    double *dvc = (double *)calloc((size_t)(B * ncs * Hkv * d), sizeof(double));
    double *kraw = (double *)malloc(sizeof(double) * (size_t)(B * T * Hkv * d));
    double *vraw = (double *)malloc(sizeof(double) * (size_t)(B * T * Hkv * d));
    if (!kc || !vc || !dkc || !dvc || !kraw || !vraw) {
        free(kc); free(vc); free(dkc); free(dvc); free(kraw); free(vraw);
        return OR_BAD_ARG;
    }
    if (nc > 0) oracle_nsa_compress(k, v, B, T, Hkv, d, cmp_len, cmp_stride, kc, vc);
    for (int64_t e = 0; e < B * T * Hkv * d; ++e) {
        kraw[e] = bf16_to_f64(k[e]);
        vraw[e] = bf16_to_f64(v[e]);
        dk[e] = 0.0;
        dv[e] = 0.0;
    }
    int status = OR_OK;
#pragma omp parallel
    {
        int64_t nmax = sel_topk * sel_block;
        if (window > nmax) nmax = window;
        if (nc > nmax) nmax = nc;
        nmax += 1;
        double *p = (double *)malloc(sizeof(double) * (size_t)nmax);
        const double **kr = (const double **)malloc(sizeof(double *) * (size_t)nmax);
        const double **vr = (const double **)malloc(sizeof(double *) * (size_t)nmax);
        double **dkr = (double **)malloc(sizeof(double *) * (size_t)nmax);
        double **dvr = (double **)malloc(sizeof(double *) * (size_t)nmax);
        double *qv = (double *)malloc(sizeof(double) * (size_t)d);
        double *dov = (double *)malloc(sizeof(double) * (size_t)d);
        double *dob = (double *)malloc(sizeof(double) * (size_t)d);
        double *o = (double *)malloc(sizeof(double) * (size_t)d);
        int ok = p && kr && vr && dkr && dvr && qv && dov && dob && o;
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < B * T; ++r) {
            if (!ok) { status = OR_BAD_ARG; continue; }
            const int64_t b = r / T, t = r % T;
            int64_t n_vis = 0;
            while (n_vis < nc && n_vis * cmp_stride + cmp_len - 1 <= t) ++n_vis;
            for (int64_t h = 0; h < Hq; ++h) {
                const int64_t g = h / G;
                for (int64_t c = 0; c < d; ++c) {
                    qv[c] = bf16_to_f64(q[(r * Hq + h) * d + c]);
                    dov[c] = bf16_to_f64(dout[(r * Hq + h) * d + c]);
                }
                double *dqv = dq + (r * Hq + h) * d;
                for (int64_t c = 0; c < d; ++c) dqv[c] = 0.0;
                for (int br = 0; br < 3; ++br) {
                    /* the branch's key set, as in the forward */
                    int64_t n = 0;
                    if (br == 0) {
                        for (int64_t i = 0; i < n_vis; ++i) {
                            const int64_t off = ((b * nc + i) * Hkv + g) * d;
                            kr[n] = kc + off; vr[n] = vc + off;
                            dkr[n] = dkc + off; dvr[n] = dvc + off; ++n;
                        }
                    } else if (br == 1) {
                        const int32_t *sg = sel + (r * Hkv + g) * sel_topk;
                        for (int64_t m = 0; m < sel_topk; ++m) {
                            const int64_t blk = sg[m];
                            if (blk < 0) continue;
                            if (blk >= nb) { status = OR_BAD_INDEX; continue; }
                            for (int64_t j = blk * sel_block; j < (blk + 1) * sel_block && j <= t && j < T; ++j) {
                                const int64_t off = ((b * T + j) * Hkv + g) * d;
                                kr[n] = kraw + off; vr[n] = vraw + off;
                                dkr[n] = dk + off; dvr[n] = dv + off; ++n;
                            }
                        }
                    } else {
                        const int64_t lo = t - window + 1 > 0 ? t - window + 1 : 0;
                        for (int64_t j = lo; j <= t; ++j) {
                            const int64_t off = ((b * T + j) * Hkv + g) * d;
                            kr[n] = kraw + off; vr[n] = vraw + off;
                            dkr[n] = dk + off; dvr[n] = dv + off; ++n;
                        }
                    }
                    double lse;
                    attend_f64(qv, d, scale, kr, vr, n, p, o, &lse);
                    const double gb = (double)gates[(r * Hq + h) * 3 + br];
                    double dg = 0.0;
                    for (int64_t c = 0; c < d; ++c) {
                        dg += dov[c] * o[c];
                        dob[c] = gb * dov[c];
                    }
                    dgates[(r * Hq + h) * 3 + br] = dg;
                    if (n > 0) attend_bwd_f64(qv, dob, d, scale, kr, vr, p, n, dqv, dkr, dvr);
                }
            }
        }
        free(p); free(kr); free(vr); free(dkr); free(dvr); free(qv); free(dov); free(dob); free(o);
    }
    /* compressed rows back to the raw rows they average */
    for (int64_t b = 0; b < B; ++b)
        for (int64_t i = 0; i < nc; ++i)
            for (int64_t u = 0; u < cmp_len; ++u) {
                const int64_t j = i * cmp_stride + u;
                for (int64_t g = 0; g < Hkv; ++g)
                    for (int64_t c = 0; c < d; ++c) {
                        dk[((b * T + j) * Hkv + g) * d + c] += dkc[((b * nc + i) * Hkv + g) * d + c] / (double)cmp_len;
                        dv[((b * T + j) * Hkv + g) * d + c] += dvc[((b * nc + i) * Hkv + g) * d + c] / (double)cmp_len;
                    }
            }
    free(kc); free(vc); free(dkc); free(dvc); free(kraw); free(vraw);
    return status;
}

/* ------------------------------------------------------------------------ */
/* A full-attention layer as an exact indexer (HySparse2 page, "Que         */
/* significa para la evolucion de la IA": a few full-attention layers       */
/* compute exact scores and guide the sparse layers' selection).            */
/* ------------------------------------------------------------------------ */

typedef struct { double score; int64_t j; } dcand_t;

/* Order: larger score first; equal scores -> lower index first. */
static int dcand_cmp(const void *a, const void *b)
{
    const dcand_t *x = (const dcand_t *)a, *y = (const dcand_t *)b;
    if (x->score != y->score) return x->score > y->score ? -1 : 1;
    return (x->j > y->j) - (x->j < y->j);
}

/*
 * For the requested rows (flat r = b*T + t, position t):
 *  1. the full layer itself: causal softmax attention of every head over all
 *     keys j <= t (fp64): out [n_rows,Hq,d], lse [n_rows,Hq];
 *  2. the exact score of key j for query t: the attention probability that
 *     the full layer puts on j, summed over all Hq heads:
 *       score(t, j) = sum_h exp(scale q_{t,h}.k_{j,g(h)} - lse_{t,h});
 *  3. the index set for the sparse layers: the forced window W_t =
 *     {max(0, t-window+1) .. t} plus the top-k of the other keys by
 *     (score desc, j asc), as in oracle_indexer_topk; ascending, -1 padded
 *     to topk+window.
 * scores (nullable) [n_rows, T]: score(t, j) for j <= t, 0 after t.
 */
int oracle_full_attn_topk(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                          int64_t B, int64_t T, int64_t Hq, int64_t Hkv, int64_t d,
                          double scale, int64_t topk, int64_t window,
                          const int64_t *rows, int64_t n_rows,
                          double *out, double *lse, int32_t *out_idx, double *scores)
{
    if (B <= 0 || T <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || Hq % Hkv != 0 ||
        topk < 0 || window < 0 || topk + window <= 0)
        return OR_BAD_ARG;
    if (!rows) n_rows = B * T;
    const int64_t G = Hq / Hkv;
    const int64_t K = topk + window;
    int bad = 0;
#pragma omp parallel
    {
        double *z = (double *)malloc(sizeof(double) * (size_t)T);
        double *sc = (double *)malloc(sizeof(double) * (size_t)T);
        double *qv = (double *)malloc(sizeof(double) * (size_t)d);
        dcand_t *cand = (dcand_t *)malloc(sizeof(dcand_t) * (size_t)T);
        int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)K);
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < n_rows; ++i) {
            int64_t r = row_at(rows, i);
            if (r < 0 || r >= B * T || !z || !sc || !qv || !cand || !sel) { bad = 1; continue; }
            const int64_t b = r / T, t = r % T;
            for (int64_t j = 0; j <= t; ++j) sc[j] = 0.0;
            for (int64_t h = 0; h < Hq; ++h) {
                const int64_t g = h / G;
                for (int64_t c = 0; c < d; ++c) qv[c] = bf16_to_f64(q[(r * Hq + h) * d + c]);
                double m = -INFINITY;
                for (int64_t j = 0; j <= t; ++j) {
                    const uint16_t *kr = k + ((b * T + j) * Hkv + g) * d;
                    double dot = 0.0;
                    for (int64_t c = 0; c < d; ++c) dot += qv[c] * bf16_to_f64(kr[c]);
                    z[j] = scale * dot;
                    if (z[j] > m) m = z[j];
                }
                double s = 0.0;
                for (int64_t j = 0; j <= t; ++j) s += exp(z[j] - m);
                const double l = m + log(s);
                if (lse) lse[i * Hq + h] = l;
                double *o = out ? out + (i * Hq + h) * d : NULL;
                if (o) for (int64_t c = 0; c < d; ++c) o[c] = 0.0;
                for (int64_t j = 0; j <= t; ++j) {
                    const double p = exp(z[j] - l);
                    sc[j] += p;
                    if (o) {
                        const uint16_t *vr = v + ((b * T + j) * Hkv + g) * d;
                        for (int64_t c = 0; c < d; ++c) o[c] += p * bf16_to_f64(vr[c]);
                    }
                }
            }
            if (scores)
                for (int64_t j = 0; j < T; ++j) scores[i * T + j] = j <= t ? sc[j] : 0.0;
            const int64_t w_lo = window > 0 ? (t - window + 1 > 0 ? t - window + 1 : 0) : t + 1;
            for (int64_t j = 0; j < w_lo; ++j) { cand[j].score = sc[j]; cand[j].j = j; }
            qsort(cand, (size_t)w_lo, sizeof(dcand_t), dcand_cmp);
            const int64_t n_take = w_lo < topk ? w_lo : topk;
            int64_t n_sel = 0;
            for (int64_t m2 = 0; m2 < n_take; ++m2) sel[n_sel++] = (int32_t)cand[m2].j;
            for (int64_t j = w_lo; j <= t; ++j) sel[n_sel++] = (int32_t)j;
            qsort(sel, (size_t)n_sel, sizeof(int32_t), i32_cmp);
            for (int64_t m2 = 0; m2 < K; ++m2) out_idx[i * K + m2] = m2 < n_sel ? sel[m2] : -1;
        }
        free(z); free(sc); free(qv); free(cand); free(sel);
    }
    return bad ? OR_BAD_ARG : OR_OK;
}
