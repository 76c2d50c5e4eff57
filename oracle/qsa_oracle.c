/*
 * QSA CPU ORACLE -- TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT PATH.
 *
 * Plain, slow, obviously-correct restatement of the Qwen Sparse Attention
 * (QSA) layer, in fp64 wherever the method leaves the precision open.  Only
 * the test suite, the smoke check and the benchmark's CPU-baseline leg may
 * load this library.  It shares no code, header or constant generator with
 * the CUDA library: both sides are written from the definitions below.
 *
 * Sources (web pages about the Qwen3.8-Flash-Next architecture):
 *   [ART] "用125亿分之6的参数，打平3970亿的旗舰模型", section
 *         "稀疏注意力：给检索建索引，也得先学会省纸" -- micro-block packing,
 *         mean pooling into one representative key, a lightweight MQA indexer
 *         scoring every block, the top blocks expanded back to their tokens
 *         for the real attention; DSA's per-token lightweight indexer as the
 *         predecessor.
 *   [SUM] "On the Design of Qwen3.8-Next Architecture: Evaluation,
 *         Efficiency, and Training Stability", token-mixing paragraph --
 *         indexing cost O(n^2) -> O(n^2/r); deployed token budget 2048 and
 *         compression ratio 4.
 *   [NEWS] "Qwen3.8-Flash发布并开源：6B激活参数背后，是Qwen4架构的第一次公开
 *         亮相", section "二、架构 / 1. 注意力机制" -- only the selected
 *         blocks receive full-precision attention.
 *
 * Readings where the pages are silent (fixed once, here):
 *   - score(t, j) = sum_h w[t,h] * max(0, q_idx[t,h,:] . Kp[j,:]), DSA style,
 *     with per-token weights w supplied by the caller; no extra scale.
 *   - candidates for a query at absolute position p are the complete blocks
 *     j < floor(p / r); the query's own block floor(p / r) is always kept.
 *   - ranking is (score descending, block index ascending); the budget in
 *     blocks kb = budget / r includes the own block.
 *   - the selection is output ascending, padded with -1.
 *   - attention scale = caller-supplied (1/sqrt(D) in every workload).
 *   - an empty token set gives o = 0 and lse = -inf.
 *
 * "Parity unpinned": the scoring form itself.  The pages print no formula or
 * worked example for it; the tests pin it by closed forms, invariants and
 * the r = 1 / Hi = 1 reduction to a plain top-k of ReLU dot products.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -shared -fPIC (see build.py).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- bf16 -- */

/* bf16 bits -> float: the bf16 pattern is the high half of an IEEE binary32. */
static float bf16_bits_to_float(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* float -> bf16 bits, round to nearest, ties to even, on the bit pattern:
 * add half an ulp of the kept part (0x7FFF) plus the kept part's lowest bit,
 * then truncate.  NaN stays NaN (quietened). */
static uint16_t float_to_bf16_bits_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u)
        return (uint16_t)((u >> 16) | 0x0040u);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

uint16_t qsa_oracle_float_to_bf16(float f) { return float_to_bf16_bits_rne(f); }

/* -------------------------------------------------------------- step 1 -- */

/*
 * Micro-block mean pooling [ART]: the r consecutive indexer keys of block j
 * are averaged into one pooled key.  For r = 4 the fp32 sum is taken as
 * ((k0 + k1) + (k2 + k3)); in general (r a power of two) adjacent pairs are
 * summed level by level.  The sum is scaled by 1/r (exact: a power of two)
 * and rounded to bf16, nearest-even.
 *
 * k_idx [B, T, Di] bf16; kp [B, T/r, Di] bf16; only blocks [j0, j1) written.
 * Returns 0, or -1 on bad arguments.
 */
int qsa_oracle_pool(const uint16_t *k_idx, int B, int64_t T, int Di, int r,
                    int64_t j0, int64_t j1, uint16_t *kp)
{
    if (r < 1 || r > 64 || (r & (r - 1)) != 0 || B < 0 || T < 0 || Di < 1)
        return -1;
    const int64_t N = T / r;
    if (j0 < 0 || j1 > N || j0 > j1)
        return -1;
    const float inv_r = 1.0f / (float)r;
    for (int b = 0; b < B; ++b) {
        for (int64_t j = j0; j < j1; ++j) {
            for (int d = 0; d < Di; ++d) {
                float buf[64];
                for (int i = 0; i < r; ++i)
                    buf[i] = bf16_bits_to_float(
                        k_idx[((int64_t)b * T + j * r + i) * Di + d]);
                for (int width = r; width > 1; width /= 2)
                    for (int i = 0; i < width / 2; ++i)
                        buf[i] = buf[2 * i] + buf[2 * i + 1];
                kp[((int64_t)b * N + j) * Di + d] =
                    float_to_bf16_bits_rne(buf[0] * inv_r);
            }
        }
    }
    return 0;
}

/* -------------------------------------------------------------- step 2 -- */

/*
 * Lightweight MQA indexer score [ART]: several indexer query heads share one
 * pooled key head.  DSA-style form: sum over heads of w_h * ReLU(q_h . Kp_j),
 * every product and sum in fp64.
 */
static double index_score(const uint16_t *q_row, const float *w_row,
                          const uint16_t *kp_row, int Hi, int Di)
{
    double s = 0.0;
    for (int h = 0; h < Hi; ++h) {
        double dot = 0.0;
        for (int d = 0; d < Di; ++d)
            dot += (double)bf16_bits_to_float(q_row[h * Di + d]) *
                   (double)bf16_bits_to_float(kp_row[d]);
        s += (double)w_row[h] * (dot > 0.0 ? dot : 0.0);
    }
    return s;
}

/*
 * Dense scores for chosen query rows (test use, small inputs).
 * rows[i] = b * Tq + t; pos[i] = absolute position p of that query.
 * out [nrows, n_cols] fp64; -inf where j >= floor(p / r) (not a candidate)
 * or j >= n_blocks.
 */
int qsa_oracle_index_scores_rows(const uint16_t *q_idx, const float *w,
                                 const uint16_t *kp, int B, int64_t Tq,
                                 int64_t n_blocks, int Hi, int Di, int r,
                                 const int64_t *rows, const int64_t *pos,
                                 int64_t nrows, int64_t n_cols, double *out)
{
    if (r < 1 || Hi < 1 || Di < 1 || B < 1)
        return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; ++i) {
        const int64_t b = rows[i] / Tq;
        const int64_t c = pos[i] / r;
        const uint16_t *q_row = q_idx + rows[i] * Hi * Di;
        const float *w_row = w + rows[i] * Hi;
        for (int64_t j = 0; j < n_cols; ++j) {
            if (j < c && j < n_blocks)
                out[i * n_cols + j] = index_score(
                    q_row, w_row, kp + (b * n_blocks + j) * Di, Hi, Di);
            else
                out[i * n_cols + j] = -INFINITY;
        }
    }
    return 0;
}

/* Scores of given (row, block) pairs: out[i] = score(rows[i], blocks[i]). */
int qsa_oracle_score_pairs(const uint16_t *q_idx, const float *w,
                           const uint16_t *kp, int64_t Tq, int64_t n_blocks,
                           int Hi, int Di, const int64_t *rows,
                           const int64_t *blocks, int64_t npairs, double *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < npairs; ++i) {
        const int64_t b = rows[i] / Tq;
        out[i] = index_score(q_idx + rows[i] * Hi * Di, w + rows[i] * Hi,
                             kp + (b * n_blocks + blocks[i]) * Di, Hi, Di);
    }
    return 0;
}

/* -------------------------------------------------------------- step 3 -- */

typedef struct {
    double s;
    int64_t j;
} cand_t;

/* score descending, then block index ascending */
static int cand_rank_cmp(const void *a, const void *b)
{
    const cand_t *x = (const cand_t *)a, *y = (const cand_t *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->j < y->j) ? -1 : (x->j > y->j);
}

static int int32_asc_cmp(const void *a, const void *b)
{
    const int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/*
 * Block selection [ART, SUM]: the highest-scoring candidate blocks are kept
 * up to the token budget (kb = budget / r blocks, own block included).
 *
 * For each requested row: score all candidates j < c = floor(p / r), rank
 * them (score desc, j asc), keep the first kb - 1, add the own block c,
 * sort ascending, pad with -1 to kb entries.
 *   sel       [nrows, kb] int32
 *   sel_score [nrows, kb] fp32 (own block +inf, padding -inf)  (nullable)
 *   margin    [nrows] fp64: s_(kb-1) - s_(kb) in rank order, +inf when at
 *             most kb - 1 candidates exist                       (nullable)
 *   s_cut     [nrows] fp64: score of the last kept candidate, +inf when
 *             there is none (c == 0)                             (nullable)
 * Returns 0, -1 on bad arguments, -2 on allocation failure.
 */
int qsa_oracle_index_topk_rows(const uint16_t *q_idx, const float *w,
                               const uint16_t *kp, int B, int64_t Tq,
                               int64_t n_blocks, int Hi, int Di, int r,
                               int budget, const int64_t *rows,
                               const int64_t *pos, int64_t nrows, int32_t *sel,
                               float *sel_score, double *margin, double *s_cut)
{
    if (r < 1 || budget < r || budget % r != 0 || Hi < 1 || Di < 1 || B < 1)
        return -1;
    const int kb = budget / r;
    for (int64_t i = 0; i < nrows; ++i)
        if (pos[i] < 0 || pos[i] / r > n_blocks)
            return -1;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; ++i) {
        const int64_t b = rows[i] / Tq;
        const int64_t c = pos[i] / r;
        cand_t *cand = (cand_t *)malloc((size_t)(c > 0 ? c : 1) * sizeof(cand_t));
        int32_t *ids = (int32_t *)malloc((size_t)kb * sizeof(int32_t));
        if (!cand || !ids) {
            free(cand);
            free(ids);
#pragma omp atomic write
            failed = 1;
            continue;
        }
        for (int64_t j = 0; j < c; ++j) {
            cand[j].s = index_score(q_idx + rows[i] * Hi * Di, w + rows[i] * Hi,
                                    kp + (b * n_blocks + j) * Di, Hi, Di);
            cand[j].j = j;
        }
        qsort(cand, (size_t)c, sizeof(cand_t), cand_rank_cmp);
        const int64_t keep = c < kb - 1 ? c : kb - 1;
        for (int64_t m = 0; m < keep; ++m)
            ids[m] = (int32_t)cand[m].j;
        ids[keep] = (int32_t)c;
        const int64_t n_sel = keep + 1;
        qsort(ids, (size_t)n_sel, sizeof(int32_t), int32_asc_cmp);
        for (int64_t m = 0; m < kb; ++m) {
            const int32_t id = m < n_sel ? ids[m] : -1;
            sel[i * kb + m] = id;
            if (sel_score) {
                float sc;
                if (id < 0)
                    sc = -INFINITY;
                else if (id == c)
                    sc = INFINITY;
                else
                    sc = (float)index_score(q_idx + rows[i] * Hi * Di,
                                            w + rows[i] * Hi,
                                            kp + (b * n_blocks + id) * Di, Hi, Di);
                sel_score[i * kb + m] = sc;
            }
        }
        if (margin)
            margin[i] = (kb >= 2 && c > kb - 1) ? cand[kb - 2].s - cand[kb - 1].s
                                                : INFINITY;
        if (s_cut)
            s_cut[i] = keep > 0 ? cand[keep - 1].s : INFINITY;
        free(cand);
        free(ids);
    }
    return failed ? -2 : 0;
}

/* -------------------------------------------------------------- step 4 -- */

/*
 * Exact softmax attention over a token set, per query head [ART, NEWS]:
 * o[h] = sum_u softmax_u(scale * q[h] . k[u, g]) v[u, g], g = h / (Hq/Hkv);
 * lse[h] = natural log of sum_u exp(scale * q[h] . k[u, g]).
 * Every product, exponential and sum in fp64.
 */
static void attend_token_set(const uint16_t *q_row, const uint16_t *k_b,
                             const uint16_t *v_b, const int64_t *keys,
                             int64_t n_keys, int Hq, int Hkv, int D,
                             double scale, double *o_row, double *lse_row,
                             double *logit)
{
    const int G = Hq / Hkv;
    if (n_keys == 0) {
        /* Empty token set (only reachable with a caller-supplied selection
         * that names no attendable token): the sum over no tokens, o = 0,
         * and lse = ln 0 = -inf. */
        for (int i = 0; i < Hq * D; ++i) o_row[i] = 0.0;
        if (lse_row)
            for (int h = 0; h < Hq; ++h) lse_row[h] = -INFINITY;
        return;
    }
    for (int h = 0; h < Hq; ++h) {
        const int g = h / G;
        double mx = -INFINITY;
        for (int64_t n = 0; n < n_keys; ++n) {
            const uint16_t *kr = k_b + (keys[n] * Hkv + g) * D;
            double dot = 0.0;
            for (int d = 0; d < D; ++d)
                dot += (double)bf16_bits_to_float(q_row[h * D + d]) *
                       (double)bf16_bits_to_float(kr[d]);
            logit[n] = scale * dot;
            if (logit[n] > mx) mx = logit[n];
        }
        double l = 0.0;
        for (int d = 0; d < D; ++d) o_row[h * D + d] = 0.0;
        for (int64_t n = 0; n < n_keys; ++n) {
            const double e = exp(logit[n] - mx);
            l += e;
            const uint16_t *vr = v_b + (keys[n] * Hkv + g) * D;
            for (int d = 0; d < D; ++d)
                o_row[h * D + d] += e * (double)bf16_bits_to_float(vr[d]);
        }
        for (int d = 0; d < D; ++d) o_row[h * D + d] /= l;
        if (lse_row) lse_row[h] = mx + log(l);
    }
}

/*
 * Attention rows.  q [B, Tq, Hq, D]; k, v [B, Tk, Hkv, D]; all bf16.
 * rows[i] = b * Tq + t, pos[i] = absolute position p of that query.
 * sel == NULL: dense causal attention over tokens 0..p.
 * sel != NULL ([nrows, kb] int32): the expanded token set
 *   { r*j + i : j in sel, j >= 0, 0 <= i < r, r*j + i <= p }  [ART].
 * o [nrows, Hq, D] fp64; lse [nrows, Hq] fp64 (nullable).
 */
int qsa_oracle_attn_rows(const uint16_t *q, const uint16_t *k,
                         const uint16_t *v, int B, int64_t Tq, int64_t Tk,
                         int Hq, int Hkv, int D, int r, int kb, double scale,
                         const int32_t *sel, const int64_t *rows,
                         const int64_t *pos, int64_t nrows, double *o,
                         double *lse)
{
    if (Hkv < 1 || Hq % Hkv != 0 || D < 1 || r < 1 || B < 1)
        return -1;
    for (int64_t i = 0; i < nrows; ++i)
        if (pos[i] < 0 || pos[i] >= Tk)
            return -1;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; ++i) {
        const int64_t b = rows[i] / Tq;
        const int64_t p = pos[i];
        const int64_t cap = sel ? (int64_t)kb * r : p + 1;
        int64_t *keys = (int64_t *)malloc((size_t)cap * sizeof(int64_t));
        double *logit = (double *)malloc((size_t)cap * sizeof(double));
        if (!keys || !logit) {
            free(keys);
            free(logit);
#pragma omp atomic write
            failed = 1;
            continue;
        }
        int64_t n_keys = 0;
        if (sel) {
            for (int m = 0; m < kb; ++m) {
                const int32_t j = sel[i * kb + m];
                if (j < 0) continue;
                for (int u = 0; u < r; ++u) {
                    const int64_t tok = (int64_t)j * r + u;
                    if (tok <= p) keys[n_keys++] = tok;
                }
            }
        } else {
            for (int64_t tok = 0; tok <= p; ++tok) keys[n_keys++] = tok;
        }
        attend_token_set(q + rows[i] * Hq * D, k + b * Tk * Hkv * D,
                         v + b * Tk * Hkv * D, keys, n_keys, Hq, Hkv, D, scale,
                         o + i * Hq * D, lse ? lse + i * Hq : NULL, logit);
        free(keys);
        free(logit);
    }
    return failed ? -2 : 0;
}

int qsa_oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void qsa_oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
