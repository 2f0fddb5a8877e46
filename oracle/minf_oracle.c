/*
 * minf_oracle.c -- fp64 CPU oracle for MInference-style dynamic sparse prefill
 * attention.  TEST INFRASTRUCTURE ONLY: the test suite, the package smoke check
 * and the benchmark's CPU-baseline leg are the only code that may load it.  The
 * product path (libminf.so) never links, loads or calls anything here, and this
 * file shares no code, header, table or helper with it.
 *
 * What it computes, step by step and in the order the sources give:
 *
 *   [NEWS] = news article "单卡A100实现百万token推理，速度快10倍，这是微软官方的大模型推理加速"
 *            (yntaolf.cn), sections 方法介绍 (method) and 延迟和内核中的稀疏模式 (Figure 4).
 *   [TALK] = transcript of the AICon 2025 talk "以 KV 缓存为中心的高效长文本方法" (dify360.com),
 *            section of the same name (the three observations and the MInference 1.0 description).
 *
 *   1. Vertical-Slash estimation ([NEWS] 方法介绍): attention of the last queries
 *      against all keys; the column sums rank the vertical lines (key positions),
 *      the diagonal sums rank the slash lines (offsets o = q - k); top-k of each.
 *   2. Block-Sparse estimation ([NEWS] 方法介绍): mean-pool Q and K over blocks of
 *      `block` tokens, multiply the pooled matrices (mean pooling commutes with
 *      the matrix product), keep the top-k key blocks of each query block.
 *   3. A-shape ([TALK] second observation; [NEWS] 方法介绍): a static mask of the
 *      first tokens plus a local window.  Tri-shape ([TALK], SCBench part, named
 *      only as an A-shape variant): read here as the A-shape mask plus dense
 *      rows for the last queries.
 *   4. Masked-softmax attention over the key set each pattern selects, causal.
 *      Vertical-Slash has two key sets: token-exact (a key enters row i if it
 *      is a vertical or i - k is a selected offset) and whole slash tiles
 *      ([NEWS] Figure 4 computes slashes as dense blocks: every key an offset
 *      reaches from some row of the query tile is attended by all its rows).
 *
 * Readings where the pages are silent (each is listed with its reason in the
 * design notes): logits are scale * q.k, softmax over keys k <= i (causal) in the
 * estimate, slash offset 0 is forced into the slash set (it takes one slot), the
 * Block-Sparse diagonal block is forced (it takes one slot), ties in any top-k go
 * to the lower index, budgets clamp to the number of candidates, a key enters a
 * Vertical-Slash row at most once, the A-shape window counts the query itself,
 * GQA maps q-head h to kv-head h / (hq / hkv).  An empty key set gives o = 0 and
 * lse = -inf.
 *
 * Inputs are bf16 values widened exactly to fp32 ([heads][n][d] row-major);
 * all arithmetic is fp64.  OpenMP spreads independent (head, row) work.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_ERR (-1)

/* Planted-mistake switches: only the mutation tests build with these, to show
 * that the pins catch each plausible slip.  The default build defines none. */
#ifndef ORC_MUTANT
#define ORC_MUTANT 0
#endif

static int kv_of(int h, int hq, int hkv) { return h / (hq / hkv); }

static int head_at(const int *head_ids, int pos) { return head_ids ? head_ids[pos] : pos; }

static double dot(const float *a, const float *b, int d) {
    double s = 0.0;
    for (int t = 0; t < d; ++t) s += (double)a[t] * (double)b[t];
    return s;
}

/* ---- top-k by (score desc, index asc) -------------------------------------- */

typedef struct { double s; int i; } scored_t;

static int by_score_desc_index_asc(const void *pa, const void *pb) {
    const scored_t *a = (const scored_t *)pa, *b = (const scored_t *)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->i > b->i) - (a->i < b->i);
}

static int int_asc(const void *pa, const void *pb) {
    int a = *(const int *)pa, b = *(const int *)pb;
    return (a > b) - (a < b);
}

/* Picks the kk best of the m candidates and writes their indices ascending to
 * out[0..kk), then -1 up to out[cap). */
static void topk_ascending(scored_t *cand, int m, int kk, int *out, int cap) {
    qsort(cand, (size_t)m, sizeof(scored_t), by_score_desc_index_asc);
    if (kk > m) kk = m;
    for (int j = 0; j < kk; ++j) out[j] = cand[j].i;
    qsort(out, (size_t)kk, sizeof(int), int_asc);
    for (int j = kk; j < cap; ++j) out[j] = -1;
}

/* ---- 1. Vertical-Slash estimation -------------------------------------------- */

/* Column sums vert[k] and diagonal sums slash[o] of the row-softmax weights of
 * the last L queries of one head (Q, K [n][d]); z is scratch of n doubles. */
static void vs_scores(const float *Q, const float *K, int n, int d, int L, double scale, double *z,
                      double *vert, double *slash) {
    for (int i = n - L; i < n; ++i) {
        /* logits of query i against keys 0..i (causal) */
        double m = -INFINITY;
#if ORC_MUTANT == 1 /* planted: no causal limit inside the last block */
        const int kend = n - 1;
#else
        const int kend = i;
#endif
        for (int kk = 0; kk <= kend; ++kk) {
            z[kk] = scale * dot(Q + (size_t)i * d, K + (size_t)kk * d, d);
            if (z[kk] > m) m = z[kk];
        }
        double den = 0.0;
        for (int kk = 0; kk <= kend; ++kk) den += exp(z[kk] - m);
        for (int kk = 0; kk <= kend; ++kk) {
            const double a = exp(z[kk] - m) / den; /* softmax weight A_ik */
            vert[kk] += a;                          /* column sum */
#if ORC_MUTANT == 2 /* planted: diagonal offset off by one */
            slash[(i - kk + 1) % n] += a;
#else
            if (kk <= i) slash[i - kk] += a;        /* diagonal sum, o = i - k */
#endif
        }
    }
}

int orc_vs_estimate(const float *q, const float *k, int hq, int hkv, int n, int d,
                    int last_q, int n_vertical, int n_slash, double scale,
                    const int *head_ids, int n_heads,
                    int *v_idx, int *s_idx, double *vert_out, double *slash_out) {
    if (!q || !k || !v_idx || !s_idx || hq <= 0 || hkv <= 0 || hq % hkv || n <= 0 ||
        d <= 0 || last_q <= 0 || n_vertical <= 0 || n_slash <= 0)
        return ORC_ERR;
    const int L = last_q < n ? last_q : n;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int hp = 0; hp < n_heads; ++hp) {
        const int h = head_at(head_ids, hp), g = kv_of(h, hq, hkv);
        const float *Q = q + (size_t)h * n * d, *K = k + (size_t)g * n * d;
        double *z = (double *)malloc(sizeof(double) * (size_t)n);
        double *vert = (double *)calloc((size_t)n, sizeof(double));
        double *slash = (double *)calloc((size_t)n, sizeof(double));
        scored_t *cand = (scored_t *)malloc(sizeof(scored_t) * (size_t)n);
        if (!z || !vert || !slash || !cand) {
            failed = 1;
        } else {
            vs_scores(Q, K, n, d, L, scale, z, vert, slash);
#if ORC_MUTANT != 3 /* planted (3): the main diagonal is not forced */
            slash[0] = INFINITY;
#endif
            for (int t = 0; t < n; ++t) { cand[t].s = vert[t]; cand[t].i = t; }
            topk_ascending(cand, n, n_vertical, v_idx + (size_t)hp * n_vertical, n_vertical);
            for (int t = 0; t < n; ++t) { cand[t].s = slash[t]; cand[t].i = t; }
            topk_ascending(cand, n, n_slash, s_idx + (size_t)hp * n_slash, n_slash);
            if (vert_out) memcpy(vert_out + (size_t)hp * n, vert, sizeof(double) * (size_t)n);
            if (slash_out) memcpy(slash_out + (size_t)hp * n, slash, sizeof(double) * (size_t)n);
        }
        free(z); free(vert); free(slash); free(cand);
    }
    return failed ? ORC_ERR : ORC_OK;
}

/* Top-p selection: the shortest prefix of the (score desc, index asc) order of
 * cand[first..m) whose score mass, added to `acc`, reaches `target`; at most
 * cap - first entries.  cand must be sorted from `first` on.  Returns the
 * number of entries taken. */
static int topp_take(const scored_t *cand, int first, int m, double acc, double target, int cap) {
    int c = first;
    while (c < m && c < cap && acc < target) acc += cand[c++].s;
    return c - first;
}

/* Vertical-Slash estimation with top-p budgets ([TALK], the part on the work
 * that followed MInference: a top-p of the attention weights instead of a
 * fixed top-k, with column-level estimation).  The scores are those of
 * orc_vs_estimate.  Verticals: the fewest keys, best first (ties to the lower
 * index), whose column sums reach p_vertical of the total column mass.
 * Slashes: offset 0 first (forced, with its own mass), then the fewest further
 * offsets, best first, until the diagonal mass reaches p_slash of the total.
 * n_vertical and n_slash cap the counts and size the rows (-1 padded);
 * v_cnt/s_cnt (nullable) get the counts; vert_out/slash_out (nullable) get the
 * scores, slash_out[0] the true diagonal mass. */
int orc_vs_estimate_topp(const float *q, const float *k, int hq, int hkv, int n, int d, int last_q,
                         int n_vertical, int n_slash, double p_vertical, double p_slash, double scale,
                         const int *head_ids, int n_heads, int *v_idx, int *s_idx, int *v_cnt,
                         int *s_cnt, double *vert_out, double *slash_out) {
    if (!q || !k || !v_idx || !s_idx || hq <= 0 || hkv <= 0 || hq % hkv || n <= 0 || d <= 0 ||
        last_q <= 0 || n_vertical <= 0 || n_slash <= 0 || !(p_vertical > 0.0 && p_vertical <= 1.0) ||
        !(p_slash > 0.0 && p_slash <= 1.0))
        return ORC_ERR;
    const int L = last_q < n ? last_q : n;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int hp = 0; hp < n_heads; ++hp) {
        const int h = head_at(head_ids, hp), g = kv_of(h, hq, hkv);
        const float *Q = q + (size_t)h * n * d, *K = k + (size_t)g * n * d;
        double *z = (double *)malloc(sizeof(double) * (size_t)n);
        double *vert = (double *)calloc((size_t)n, sizeof(double));
        double *slash = (double *)calloc((size_t)n, sizeof(double));
        scored_t *cand = (scored_t *)malloc(sizeof(scored_t) * (size_t)n);
        if (!z || !vert || !slash || !cand) {
            failed = 1;
        } else {
            vs_scores(Q, K, n, d, L, scale, z, vert, slash);
            double tv = 0.0, ts = 0.0;
            for (int t = 0; t < n; ++t) { tv += vert[t]; ts += slash[t]; }
            int *vr = v_idx + (size_t)hp * n_vertical, *sr = s_idx + (size_t)hp * n_slash;
            /* verticals */
            for (int t = 0; t < n; ++t) { cand[t].s = vert[t]; cand[t].i = t; }
            qsort(cand, (size_t)n, sizeof(scored_t), by_score_desc_index_asc);
            const int cv = topp_take(cand, 0, n, 0.0, p_vertical * tv, n_vertical);
            for (int j = 0; j < cv; ++j) vr[j] = cand[j].i;
            qsort(vr, (size_t)cv, sizeof(int), int_asc);
            for (int j = cv; j < n_vertical; ++j) vr[j] = -1;
            /* slashes: offset 0, then the others best first */
            for (int t = 1; t < n; ++t) { cand[t - 1].s = slash[t]; cand[t - 1].i = t; }
            qsort(cand, (size_t)(n - 1), sizeof(scored_t), by_score_desc_index_asc);
#if ORC_MUTANT == 9 /* planted: the forced diagonal's mass not counted */
            const double acc0 = 0.0;
#else
            const double acc0 = slash[0];
#endif
            const int cs = topp_take(cand, 0, n - 1, acc0, p_slash * ts, n_slash - 1);
            sr[0] = 0;
            for (int j = 0; j < cs; ++j) sr[1 + j] = cand[j].i;
            qsort(sr, (size_t)(cs + 1), sizeof(int), int_asc);
            for (int j = cs + 1; j < n_slash; ++j) sr[j] = -1;
            if (v_cnt) v_cnt[hp] = cv;
            if (s_cnt) s_cnt[hp] = cs + 1;
            if (vert_out) memcpy(vert_out + (size_t)hp * n, vert, sizeof(double) * (size_t)n);
            if (slash_out) memcpy(slash_out + (size_t)hp * n, slash, sizeof(double) * (size_t)n);
        }
        free(z); free(vert); free(slash); free(cand);
    }
    return failed ? ORC_ERR : ORC_OK;
}

/* ---- 2. Block-Sparse estimation ------------------------------------------------ */

/* Mean of `block` consecutive rows of x ([n][d]) for block b. */
static void mean_pool(const float *x, int d, int block, int b, double *out) {
    for (int t = 0; t < d; ++t) out[t] = 0.0;
    for (int r = 0; r < block; ++r)
        for (int t = 0; t < d; ++t) out[t] += (double)x[((size_t)b * block + r) * d + t];
    for (int t = 0; t < d; ++t) out[t] /= (double)block;
}

int orc_block_estimate(const float *q, const float *k, int hq, int hkv, int n, int d,
                       int block, int topk, const int *head_ids, int n_heads,
                       int *blk_idx, int *blk_cnt, double *pooled_q, double *pooled_k,
                       double *scores) {
    if (!q || !k || !blk_idx || !blk_cnt || hq <= 0 || hkv <= 0 || hq % hkv || n <= 0 ||
        d <= 0 || block <= 0 || n % block || topk <= 0)
        return ORC_ERR;
    const int nb = n / block;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int hp = 0; hp < n_heads; ++hp) {
        const int h = head_at(head_ids, hp), g = kv_of(h, hq, hkv);
        double *qp = (double *)malloc(sizeof(double) * (size_t)nb * d);
        double *kp = (double *)malloc(sizeof(double) * (size_t)nb * d);
        scored_t *cand = (scored_t *)malloc(sizeof(scored_t) * (size_t)nb);
        if (!qp || !kp || !cand) {
            failed = 1;
        } else {
            for (int b = 0; b < nb; ++b) {
                mean_pool(q + (size_t)h * n * d, d, block, b, qp + (size_t)b * d);
                mean_pool(k + (size_t)g * n * d, d, block, b, kp + (size_t)b * d);
            }
            if (pooled_q) memcpy(pooled_q + (size_t)hp * nb * d, qp, sizeof(double) * (size_t)nb * d);
            if (pooled_k) memcpy(pooled_k + (size_t)hp * nb * d, kp, sizeof(double) * (size_t)nb * d);
            for (int i = 0; i < nb; ++i) {
                int *row = blk_idx + ((size_t)hp * nb + i) * topk;
                /* pooled score s_ij = Qp_i . Kp_j for j <= i */
                for (int j = 0; j <= i; ++j) {
                    double s = 0.0;
                    for (int t = 0; t < d; ++t) s += qp[(size_t)i * d + t] * kp[(size_t)j * d + t];
                    if (scores) scores[((size_t)hp * nb + i) * nb + j] = s;
                    cand[j].s = s;
                    cand[j].i = j;
                }
                if (scores)
                    for (int j = i + 1; j < nb; ++j) scores[((size_t)hp * nb + i) * nb + j] = -INFINITY;
#if ORC_MUTANT == 4 /* planted: diagonal block not forced */
                topk_ascending(cand, i + 1, topk, row, topk);
                int c = 0;
                while (c < topk && row[c] >= 0) ++c;
                blk_cnt[(size_t)hp * nb + i] = c;
#else
                /* the diagonal block is always taken; the best topk-1 of j < i join it */
                int c = 0;
                if (topk > 1 && i > 0) {
                    topk_ascending(cand, i, topk - 1, row, topk);
                    while (c < topk && row[c] >= 0) ++c;
                }
                row[c] = i; /* i is larger than every j < i, so the row stays ascending */
                ++c;
                for (int j = c; j < topk; ++j) row[j] = -1;
                blk_cnt[(size_t)hp * nb + i] = c;
#endif
            }
        }
        free(qp); free(kp); free(cand);
    }
    return failed ? ORC_ERR : ORC_OK;
}

/* ---- 4. masked-softmax attention over an explicit key set ------------------- */

/* o = sum_k softmax(z)_k v_k over the listed keys; lse = log sum_k exp(z_k). */
static void attend_keys(const float *qi, const float *K, const float *V, int d, double scale,
                        const int *keys, int nk, double *z, double *o, double *lse) {
    for (int t = 0; t < d; ++t) o[t] = 0.0;
    if (nk == 0) { *lse = -INFINITY; return; }
    double m = -INFINITY;
    for (int j = 0; j < nk; ++j) {
        z[j] = scale * dot(qi, K + (size_t)keys[j] * d, d);
        if (z[j] > m) m = z[j];
    }
    double den = 0.0;
    for (int j = 0; j < nk; ++j) den += exp(z[j] - m);
    for (int j = 0; j < nk; ++j) {
        const double p = exp(z[j] - m) / den;
        const float *vk = V + (size_t)keys[j] * d;
        for (int t = 0; t < d; ++t) o[t] += p * (double)vk[t];
    }
    *lse = m + log(den);
}

enum { PAT_DENSE = 0, PAT_ASHAPE = 1, PAT_BLOCK = 2, PAT_VS = 3, PAT_TRISHAPE = 4, PAT_VS_TILES = 5 };

typedef struct {
    int pattern;
    int n_sink, window;                               /* A-shape, Tri-shape */
    int n_last;                                       /* Tri-shape: dense last rows */
    const int *blk_idx, *blk_cnt; int topk, block;    /* Block-Sparse */
    const int *v_idx; int n_v; const int *s_idx; int n_s; /* Vertical-Slash */
    int tile_rows;                                    /* Vertical-Slash, whole slash tiles */
} mask_spec_t;

/* Builds the key list of query row i of head position hp, ascending, each key
 * once.  mark[] is scratch of n bytes, all zero on entry and on exit. */
static int key_list(const mask_spec_t *ms, int hp, int i, int n, int *keys, unsigned char *mark) {
    int nk = 0;
    switch (ms->pattern) {
    case PAT_DENSE:
        for (int kk = 0; kk <= i; ++kk) keys[nk++] = kk;
        break;
    case PAT_ASHAPE:
        /* first n_sink tokens, plus the window of `window` keys ending at i */
        for (int kk = 0; kk <= i; ++kk)
#if ORC_MUTANT == 5 /* planted: window excludes the query itself */
            if (kk < ms->n_sink || i - kk < ms->window - 1) keys[nk++] = kk;
#else
            if (kk < ms->n_sink || i - kk < ms->window) keys[nk++] = kk;
#endif
        break;
    case PAT_TRISHAPE:
        /* the A-shape lines, plus every key for the last n_last queries */
        for (int kk = 0; kk <= i; ++kk)
#if ORC_MUTANT == 7 /* planted: the dense tail one row short */
            if (kk < ms->n_sink || i - kk < ms->window || i > n - ms->n_last) keys[nk++] = kk;
#else
            if (kk < ms->n_sink || i - kk < ms->window || i >= n - ms->n_last) keys[nk++] = kk;
#endif
        break;
    case PAT_BLOCK: {
        const int nb = n / ms->block, bq = i / ms->block;
        const int *row = ms->blk_idx + ((size_t)hp * nb + bq) * ms->topk;
        const int cnt = ms->blk_cnt[(size_t)hp * nb + bq];
        for (int j = 0; j < cnt; ++j) {
            const int bk = row[j];
            if (bk < 0) continue;
            for (int kk = bk * ms->block; kk < (bk + 1) * ms->block && kk <= i; ++kk) mark[kk] = 1;
        }
        for (int kk = 0; kk <= i; ++kk)
            if (mark[kk]) { keys[nk++] = kk; mark[kk] = 0; }
        break;
    }
    case PAT_VS: {
        const int *vr = ms->v_idx + (size_t)hp * ms->n_v, *sr = ms->s_idx + (size_t)hp * ms->n_s;
        for (int j = 0; j < ms->n_v; ++j)              /* vertical lines: key positions */
            if (vr[j] >= 0 && vr[j] <= i) mark[vr[j]] = 1;
        for (int j = 0; j < ms->n_s; ++j)              /* slash lines: offsets o = i - k */
            if (sr[j] >= 0 && sr[j] <= i) mark[i - sr[j]] = 1;
        for (int kk = 0; kk <= i; ++kk)
            if (mark[kk]) {
#if ORC_MUTANT == 6 /* planted: a key in both a vertical and a slash counted twice */
                int both = 0;
                for (int j = 0; j < ms->n_v; ++j) both |= vr[j] == kk;
                int on_slash = 0;
                for (int j = 0; j < ms->n_s; ++j) on_slash |= sr[j] == i - kk;
                keys[nk++] = kk;
                if (both && on_slash) keys[nk++] = kk;
#else
                keys[nk++] = kk;
#endif
                mark[kk] = 0;
            }
        break;
    }
    case PAT_VS_TILES: {
        /* Slash ranges attended whole: row i of the tile_rows-row query tile that
         * starts at r0 takes, for every selected offset o, the keys r0 - o ..
         * r0 + tile_rows - 1 - o (the keys that o reaches from any row of its
         * tile), plus the verticals; then only the causal bound k <= i. */
        const int *vr = ms->v_idx + (size_t)hp * ms->n_v, *sr = ms->s_idx + (size_t)hp * ms->n_s;
        const int r0 = i - i % ms->tile_rows;
#if ORC_MUTANT == 8 /* planted: the range one key too wide */
        const int span = ms->tile_rows;
#else
        const int span = ms->tile_rows - 1;
#endif
        for (int j = 0; j < ms->n_v; ++j)
            if (vr[j] >= 0 && vr[j] <= i) mark[vr[j]] = 1;
        for (int j = 0; j < ms->n_s; ++j) {
            const int o = sr[j];
            if (o < 0 || o >= n) continue;
            const int lo = r0 - o < 0 ? 0 : r0 - o, hi = r0 + span - o < i ? r0 + span - o : i;
            for (int kk = lo; kk <= hi; ++kk) mark[kk] = 1;
        }
        for (int kk = 0; kk <= i; ++kk)
            if (mark[kk]) { keys[nk++] = kk; mark[kk] = 0; }
        break;
    }
    }
    return nk;
}

static int attend(const float *q, const float *k, const float *v, int hq, int hkv, int n, int d,
                  double scale, const int *head_ids, int n_heads, const mask_spec_t *ms,
                  const int *rows, int n_rows, double *out, double *lse) {
    if (!q || !k || !v || !out || hq <= 0 || hkv <= 0 || hq % hkv || n <= 0 || d <= 0)
        return ORC_ERR;
    const int nr = rows ? n_rows : n;
    int failed = 0;
#pragma omp parallel
    {
        int *keys = (int *)malloc(sizeof(int) * 2 * (size_t)n);
        double *z = (double *)malloc(sizeof(double) * 2 * (size_t)n);
        unsigned char *mark = (unsigned char *)calloc((size_t)n, 1);
        if (!keys || !z || !mark) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 4) collapse(2)
            for (int hp = 0; hp < n_heads; ++hp)
                for (int r = 0; r < nr; ++r) {
                    const int h = head_at(head_ids, hp), g = kv_of(h, hq, hkv);
                    const int i = rows ? rows[r] : r;
                    const size_t slot = (size_t)hp * nr + r;
                    double l;
                    if (i < 0 || i >= n) { l = NAN; for (int t = 0; t < d; ++t) out[slot * d + t] = NAN; }
                    else {
                        const int nk = key_list(ms, hp, i, n, keys, mark);
                        attend_keys(q + ((size_t)h * n + i) * d, k + (size_t)g * n * d,
                                    v + (size_t)g * n * d, d, scale, keys, nk, z, out + slot * d, &l);
                    }
                    if (lse) lse[slot] = l;
                }
        }
        free(keys); free(z); free(mark);
    }
    return failed ? ORC_ERR : ORC_OK;
}

int orc_dense_attention(const float *q, const float *k, const float *v, int hq, int hkv, int n,
                        int d, double scale, const int *head_ids, int n_heads, const int *rows,
                        int n_rows, double *out, double *lse) {
    mask_spec_t ms = {0};
    ms.pattern = PAT_DENSE;
    return attend(q, k, v, hq, hkv, n, d, scale, head_ids, n_heads, &ms, rows, n_rows, out, lse);
}

int orc_ashape_attention(const float *q, const float *k, const float *v, int hq, int hkv, int n,
                         int d, double scale, const int *head_ids, int n_heads, int n_sink,
                         int window, const int *rows, int n_rows, double *out, double *lse) {
    if (n_sink < 0 || window < 1) return ORC_ERR;
    mask_spec_t ms = {0};
    ms.pattern = PAT_ASHAPE;
    ms.n_sink = n_sink;
    ms.window = window;
    return attend(q, k, v, hq, hkv, n, d, scale, head_ids, n_heads, &ms, rows, n_rows, out, lse);
}

/* Tri-shape: A-shape plus dense rows for the last n_last queries (the reading
 * taken here of the Tri-shape named in the AICon talk transcript
 * "以 KV 缓存为中心的高效长文本方法", SCBench part, as an A-shape variant). */
int orc_trishape_attention(const float *q, const float *k, const float *v, int hq, int hkv, int n,
                           int d, double scale, const int *head_ids, int n_heads, int n_sink,
                           int window, int n_last, const int *rows, int n_rows, double *out,
                           double *lse) {
    if (n_sink < 0 || window < 1 || n_last < 0) return ORC_ERR;
    mask_spec_t ms = {0};
    ms.pattern = PAT_TRISHAPE;
    ms.n_sink = n_sink;
    ms.window = window;
    ms.n_last = n_last;
    return attend(q, k, v, hq, hkv, n, d, scale, head_ids, n_heads, &ms, rows, n_rows, out, lse);
}

int orc_block_attention(const float *q, const float *k, const float *v, int hq, int hkv, int n,
                        int d, double scale, const int *head_ids, int n_heads, int block,
                        const int *blk_idx, const int *blk_cnt, int topk, const int *rows,
                        int n_rows, double *out, double *lse) {
    if (!blk_idx || !blk_cnt || block <= 0 || n % block || topk <= 0) return ORC_ERR;
    mask_spec_t ms = {0};
    ms.pattern = PAT_BLOCK;
    ms.blk_idx = blk_idx;
    ms.blk_cnt = blk_cnt;
    ms.topk = topk;
    ms.block = block;
    return attend(q, k, v, hq, hkv, n, d, scale, head_ids, n_heads, &ms, rows, n_rows, out, lse);
}

int orc_vs_attention(const float *q, const float *k, const float *v, int hq, int hkv, int n, int d,
                     double scale, const int *head_ids, int n_heads, const int *v_idx,
                     int n_vertical, const int *s_idx, int n_slash, const int *rows, int n_rows,
                     double *out, double *lse) {
    if (!v_idx || !s_idx || n_vertical <= 0 || n_slash <= 0) return ORC_ERR;
    mask_spec_t ms = {0};
    ms.pattern = PAT_VS;
    ms.v_idx = v_idx;
    ms.n_v = n_vertical;
    ms.s_idx = s_idx;
    ms.n_s = n_slash;
    return attend(q, k, v, hq, hkv, n, d, scale, head_ids, n_heads, &ms, rows, n_rows, out, lse);
}

/* Vertical-Slash with every computed slash range attended whole by the rows of
 * its query tile (the pages' kernel computes slashes as dense blocks: news
 * article "单卡A100实现百万token推理…", Figure 4); tile_rows is the query tile height. */
int orc_vs_tiles_attention(const float *q, const float *k, const float *v, int hq, int hkv, int n,
                           int d, double scale, const int *head_ids, int n_heads, const int *v_idx,
                           int n_vertical, const int *s_idx, int n_slash, int tile_rows,
                           const int *rows, int n_rows, double *out, double *lse) {
    if (!v_idx || !s_idx || n_vertical <= 0 || n_slash <= 0 || tile_rows <= 0) return ORC_ERR;
    mask_spec_t ms = {0};
    ms.pattern = PAT_VS_TILES;
    ms.v_idx = v_idx;
    ms.n_v = n_vertical;
    ms.s_idx = s_idx;
    ms.n_s = n_slash;
    ms.tile_rows = tile_rows;
    return attend(q, k, v, hq, hkv, n, d, scale, head_ids, n_heads, &ms, rows, n_rows, out, lse);
}

int orc_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

int orc_mutant(void) { return ORC_MUTANT; }
