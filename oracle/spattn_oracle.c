/*
 * spattn_oracle.c -- float64 CPU oracle for block-sparse decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously-correct
 * definition that the CUDA library is checked against.  Only the tests, the
 * smoke check and the CPU-baseline leg of the benchmark load it.  It shares
 * no source, header, table or helper with the CUDA library and must never be
 * used as a fallback for it.
 *
 * What it computes, step by step, in float64 (sources are the pages this
 * library restates; titles are given as printed on the pages):
 *
 *  1. Dequantise the stored cache.  bf16 is the upper half of an IEEE
 *     binary32; fp8 e4m3fn is 1 sign / 4 exponent (bias 7) / 3 mantissa bits
 *     with no infinities, times a per-(page, head) fp32 scale
 *     ("Claude Code 1M 上下文", §2(3) "FP8量化与无损压缩": FP8 KV storage).
 *  2. Block compression by mean pooling: one entry per 64-token block, the
 *     mean of the keys of the tokens the block holds
 *     ("Claude Code压缩上下文窗口的底层原理与性能优化实践", 算法流程, the
 *     均值池化合并 node; "CSA + HCA 混合注意力机制" §4.1, where plain
 *     averaging is named as the parameter-free compression).
 *  3. Block scores: the query of each KV-head group, averaged over the group,
 *     dotted with each compressed key and scaled by 1/sqrt(d)
 *     ("CSA + HCA 混合注意力机制" §4.2 Lightning Indexer, steps 3-4, and
 *     §4.4 step 1: score every compressed entry against the query).
 *  4. Selection: the sink block and the local-window blocks are always kept;
 *     the middle blocks are ranked by (score desc, index asc) and the top-k,
 *     or the minimal top-p prefix of their softmax probabilities capped at
 *     k_max, are kept ("Claude Opus 长上下文 KV Cache 稀疏注意力",
 *     §稀疏注意力与 KV Cache 压缩的工程实现: block-level management,
 *     attention sink, local context, Top-P selection; the configuration
 *     table of §可落地的配置参数与监控要点; "CSA + HCA 混合注意力机制" §4.4
 *     step 3 argsort/top-k).  For a chunk of query tokens the kept middle set
 *     is the union over the tokens.
 *  5. Exact softmax attention of every query head over every token of the
 *     kept blocks, causal inside the chunk, scale 1/sqrt(d)
 *     ("CSA + HCA 混合注意力机制" §2.1 scaled dot-product attention, §4.4
 *     step 4).
 *
 * Where the pages are silent the reading taken is stated beside the code.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Keep in step with oracle/__init__.py (ctypes mirror). */
typedef struct {
    int batch;          /* B */
    int q_tokens;       /* Tq: query tokens per request (1 = decode) */
    int num_q_heads;    /* Hq */
    int num_kv_heads;   /* Hkv; query head i reads KV head i / (Hq/Hkv) */
    int head_dim;       /* d */
    int block_size;     /* P: tokens per block (= per page) */
    int num_pages;      /* pages in the cache pool */
    int max_blocks;     /* columns of the block table */
    int max_sel;        /* columns of the selection output */
    int kv_fp8;         /* 0: bf16 cache, 1: fp8 e4m3fn cache + fp32 scales */
} spo_dims;

typedef struct {
    int sink_blocks;    /* S */
    int local_blocks;   /* W */
    int mode;           /* 0: top-k, 1: top-p, 2: top-p with the anchor-adaptive cap */
    int top_k;          /* top-k: fixed k when > 0 */
    double top_p;       /* top-p: mass threshold in (0, 1] */
    double max_ratio;   /* cap k_max = floor(max_ratio * n_mid); <= 0: no cap */
    double sm_scale;    /* 0: 1/sqrt(d) */
    double min_ratio;   /* mode 2: the cap ratio when the anchors dominate */
} spo_params;

/* ---------------------------------------------------------------- decoding */

/*
 * The bf16 value nearest to x, ties to even: bf16 keeps the top 16 bits of a
 * binary32, i.e. 8 significant bits with binary32's exponent range (smallest
 * normal 2^-126, subnormal spacing 2^-133, largest finite (2 - 2^-7) 2^127).
 * One rounding from binary64 (low-precision scoring: "CSA + HCA 混合注意力机制"
 * §4.2, the indexer's QK path at reduced precision).
 */
double spo_round_bf16(double x)
{
    if (!isfinite(x) || x == 0.0)
        return x;
    int e;
    (void)frexp(x, &e);                 /* |x| = m 2^e, m in [0.5, 1) */
    int q = e - 8;                      /* spacing of 8-bit significands in this binade */
    if (q < -133) q = -133;             /* subnormal: fixed spacing */
    double y = ldexp(nearbyint(ldexp(x, -q)), q);   /* exact scalings; nearbyint ties to even */
    if (fabs(y) >= 0x1p128)
        y = copysign(INFINITY, x);
    return y;
}

void spo_round_bf16_array(double *x, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        x[i] = spo_round_bf16(x[i]);
}

/* bf16 is the high 16 bits of a binary32: widening is exact. */
double spo_bf16_to_f64(uint16_t bits)
{
    uint32_t w = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return (double)f;
}

/* e4m3fn: exponent bias 7, subnormals at exponent 0, S.1111.111 is NaN,
 * no infinities. */
double spo_e4m3_to_f64(uint8_t bits)
{
    int sign = (bits >> 7) & 1;
    int e = (bits >> 3) & 0xF;
    int m = bits & 0x7;
    double v;
    if (e == 0xF && m == 0x7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* Element (page, h, t, c) of a cache, dequantised. */
static double cache_at(const spo_dims *dm, const void *cache, const float *scale,
                       int64_t page, int h, int t, int c)
{
    int64_t off = (((page * dm->num_kv_heads + h) * dm->block_size) + t) * dm->head_dim + c;
    if (dm->kv_fp8)
        return spo_e4m3_to_f64(((const uint8_t *)cache)[off]) *
               (double)scale[page * dm->num_kv_heads + h];
    return spo_bf16_to_f64(((const uint16_t *)cache)[off]);
}

static int num_blocks(const spo_dims *dm, int len)
{
    return (len + dm->block_size - 1) / dm->block_size;
}

static double softmax_scale(const spo_dims *dm, const spo_params *pr)
{
    return pr->sm_scale > 0.0 ? pr->sm_scale : 1.0 / sqrt((double)dm->head_dim);
}

/* --------------------------------------------------------- 2. compression */

/*
 * kbar[page][h][c] = mean over the filled tokens of block j of K, for every
 * block j of every request.  A block holds min(P, L - j*P) tokens; the tail
 * block of a request is partly filled.  Pages not referenced are untouched.
 */
int spo_compress_keys(const spo_dims *dm, const void *k_cache, const float *k_scale,
                      const int32_t *block_table, const int32_t *seq_lens,
                      double *kbar)
{
    const int P = dm->block_size, D = dm->head_dim, H = dm->num_kv_heads;
    for (int b = 0; b < dm->batch; ++b) {
        int L = seq_lens[b];
        int nb = num_blocks(dm, L);
        if (nb > dm->max_blocks)
            return -1;
        #pragma omp parallel for schedule(dynamic)
        for (int j = 0; j < nb; ++j) {
            int64_t page = block_table[(int64_t)b * dm->max_blocks + j];
            int filled = L - j * P < P ? L - j * P : P;
            for (int h = 0; h < H; ++h)
                for (int c = 0; c < D; ++c) {
                    double s = 0.0;
                    for (int t = 0; t < filled; ++t)
                        s += cache_at(dm, k_cache, k_scale, page, h, t, c);
                    kbar[(page * H + h) * D + c] = s / (double)filled;
                }
        }
    }
    return 0;
}

/* ------------------------------------------------------------- 3. scores */

/*
 * scores[b][t][h][j] = scale * (qbar . kbar[page(b, j)][h]) for middle
 * blocks j in [S, nb - W); -inf for every other column.  qbar is the mean of
 * the G query rows that share KV head h (reading: the indexer aggregates
 * over heads; with no learned indexer the group's mean query gives the mean
 * of the group's per-head logits against the compressed key).
 */
int spo_block_scores(const spo_dims *dm, const spo_params *pr, const uint16_t *q,
                     const double *kbar, const int32_t *block_table,
                     const int32_t *seq_lens, double *scores)
{
    const int D = dm->head_dim, H = dm->num_kv_heads, Tq = dm->q_tokens;
    const int G = dm->num_q_heads / H;
    const double scale = softmax_scale(dm, pr);
    const int64_t nrows = (int64_t)dm->batch * Tq * H;
    #pragma omp parallel for schedule(dynamic)
    for (int64_t row = 0; row < nrows; ++row) {
        int h = (int)(row % H);
        int t = (int)((row / H) % Tq);
        int b = (int)(row / ((int64_t)H * Tq));
        int nb = num_blocks(dm, seq_lens[b]);
        double *out = scores + row * dm->max_blocks;
        double *qbar = (double *)calloc((size_t)D, sizeof(double));
        for (int g = 0; g < G; ++g)
            for (int c = 0; c < D; ++c)
                qbar[c] += spo_bf16_to_f64(
                    q[(((int64_t)b * Tq + t) * dm->num_q_heads + h * G + g) * D + c]);
        for (int c = 0; c < D; ++c)
            qbar[c] /= (double)G;
        for (int j = 0; j < dm->max_blocks; ++j) {
            /* mode 2 also scores the anchors (sink and local blocks) */
            const int anchor = j < pr->sink_blocks || j >= nb - pr->local_blocks;
            if (j >= nb || (anchor && pr->mode != 2)) {
                out[j] = -INFINITY;
                continue;
            }
            int64_t page = block_table[(int64_t)b * dm->max_blocks + j];
            double s = 0.0;
            for (int c = 0; c < D; ++c)
                s += qbar[c] * kbar[(page * H + h) * D + c];
            out[j] = s * scale;
        }
        free(qbar);
    }
    return 0;
}

/* ---------------------------------------------------------- 4. selection */

typedef struct {
    double s;
    int j;
} ranked;

/* Rank order: higher score first; equal scores, lower block index first. */
static int rank_cmp(const void *a, const void *b)
{
    const ranked *x = (const ranked *)a, *y = (const ranked *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->j > y->j) - (x->j < y->j);
}

/*
 * Mode 2 cap ("Claude Opus 长上下文 KV Cache 稀疏注意力", §多上下文场景下的跨文档注意力
 * 恢复: the sink and local blocks are anchors; the maximum and minimum of the
 * scores set the Top-P ratio, higher when the maximum stands well above the
 * anchors).  Reading: a = the anchors' best score, hi / lo the middle's best
 * and worst; r = clamp((hi - a) / (hi - lo), 0, 1) (0 when hi <= lo);
 * ratio = min_ratio + r (max_ratio - min_ratio); k_max = floor(ratio n_mid).
 * *margin_k: how far (in score units) the inputs may move before k_max
 * changes.
 */
static int anchor_k_max(const spo_params *pr, double a, double hi, double lo, int n_mid, double *margin_k)
{
    double r = hi > lo ? (hi - a) / (hi - lo) : 0.0;
    if (r < 0.0) r = 0.0;
    if (r > 1.0) r = 1.0;
    const double span = pr->max_ratio - pr->min_ratio;
    const double ratio = pr->min_ratio + r * span;
    const double x = ratio * (double)n_mid;
    int k = (int)floor(x);
    if (k > n_mid) k = n_mid;
    if (!(hi > lo))
        *margin_k = 0.0;                       /* degenerate: any change moves r */
    else if (a >= hi)
        *margin_k = a - hi;                    /* r pinned at 0 */
    else if (a <= lo)
        *margin_k = lo - a;                    /* r pinned at 1 */
    else if (span <= 0.0)
        *margin_k = INFINITY;
    else {
        double d = x - floor(x);
        if (ceil(x) - x < d) d = ceil(x) - x;
        *margin_k = d * (hi - lo) / (span * (double)n_mid);
    }
    return k;
}

/* Number of middle blocks kept for one query row, and the decision margin.
 * a: the anchors' best score (mode 2 only).
 *
 * The decision margin is the distance from the inputs to the nearest point
 * where the kept set would change, measured on each quantity the decision
 * is taken on: the score gap across the cut (the worst kept block against
 * the best dropped one; score units) and, for top-p, the distance of the
 * threshold p to the nearest prefix mass at which the kept set changes
 * (probability units).  Top-p keeps the minimal ranked prefix m* with
 * C_{m*} >= p (C_i: mass of the i best blocks), capped at k_max:
 *   uncapped (m* <= k_max): p - C_{m*-1} (a lower p reaching C_{m*-1} keeps
 *     m* - 1 blocks; no such point when m* = 1) and C_{m*} - p (a higher p
 *     keeps m* + 1; none when m* = n_mid or m* = k_max, where the cap holds
 *     the set);
 *   capped (m* > k_max): p - C_{k_max-1} (only a p at or below C_{k_max-1}
 *     keeps fewer than k_max; none when k_max <= 1); a higher p changes
 *     nothing.
 * Mode 2 adds how far the anchor score may move before k_max changes. */
static int row_keep_count(const spo_params *pr, const ranked *r, int n_mid, double a,
                          double *margin)
{
    int k_max = pr->max_ratio > 0.0 ? (int)floor(pr->max_ratio * (double)n_mid) : n_mid;
    if (k_max > n_mid) k_max = n_mid;
    double gap_inf = INFINITY;
    *margin = gap_inf;
    if (n_mid == 0)
        return 0;
    double margin_k = INFINITY;
    if (pr->mode == 2)
        k_max = anchor_k_max(pr, a, r[0].s, r[n_mid - 1].s, n_mid, &margin_k);
    if (pr->mode == 0) {
        /* top-k: k = top_k if given, else the ratio's k_max; never above the
         * cap or the middle count. */
        int k = pr->top_k > 0 ? pr->top_k : k_max;
        if (k > k_max) k = k_max;
        if (k > 0 && k < n_mid)
            *margin = r[k - 1].s - r[k].s;
        return k;
    }
    /* top-p: probabilities are the softmax of the middle scores; keep the
     * minimal prefix of the ranked order whose mass reaches top_p
     * (inclusive), then apply the cap. */
    double mx = r[0].s, z = 0.0;
    for (int i = 0; i < n_mid; ++i)
        z += exp(r[i].s - mx);
    double c = 0.0, c_prev = 0.0;
    int m = n_mid;
    for (int i = 0; i < n_mid; ++i) {
        c_prev = c;
        c += exp(r[i].s - mx) / z;
        if (c >= pr->top_p) {
            m = i + 1;
            break;
        }
    }
    if (m > k_max) {
        /* the cap binds: the set is the top k_max; it would change only if
         * the rank order at the cut changed or p fell to the mass of the
         * k_max - 1 best blocks */
        double cum = 0.0;
        for (int i = 0; i + 1 < k_max; ++i)
            cum += exp(r[i].s - mx) / z;
        double mg = k_max >= 2 ? pr->top_p - cum : INFINITY;
        if (k_max > 0 && k_max < n_mid && r[k_max - 1].s - r[k_max].s < mg)
            mg = r[k_max - 1].s - r[k_max].s;
        *margin = mg < margin_k ? mg : margin_k;
        return k_max;
    }
    double mg = m >= 2 ? pr->top_p - c_prev : INFINITY;
    if (m < n_mid && c - pr->top_p < mg && m < k_max)
        mg = c - pr->top_p;
    if (m < n_mid && r[m - 1].s - r[m].s < mg)
        mg = r[m - 1].s - r[m].s;
    /* (k_max only matters when it binds, but a moved k_max could bind) */
    if (pr->mode == 2 && m >= k_max - 1 && margin_k < mg)
        mg = margin_k;
    *margin = mg;
    return m;
}

/*
 * Selection for every (b, h): sink blocks [0, S), local blocks [nb - W, nb)
 * and, per query token t, the kept middle set M_t; the union over t is
 * written ascending to sel_idx[b][h][*], its size to sel_count[b][h].
 * margin[b][h] (optional) receives the smallest decision margin over t.
 * Returns -2 if max_sel is too small for a row.
 */
int spo_select(const spo_dims *dm, const spo_params *pr, const double *scores,
               const int32_t *seq_lens, int32_t *sel_idx, int32_t *sel_count,
               double *margin)
{
    const int H = dm->num_kv_heads, Tq = dm->q_tokens;
    int err = 0;
    #pragma omp parallel for schedule(dynamic)
    for (int64_t bh = 0; bh < (int64_t)dm->batch * H; ++bh) {
        int b = (int)(bh / H), h = (int)(bh % H);
        int nb = num_blocks(dm, seq_lens[b]);
        int S = pr->sink_blocks, W = pr->local_blocks;
        int n_mid = nb - S - W > 0 ? nb - S - W : 0;
        char *keep = (char *)calloc((size_t)(nb > 0 ? nb : 1), 1);
        ranked *r = (ranked *)malloc(sizeof(ranked) * (size_t)(n_mid > 0 ? n_mid : 1));
        double mg_row = INFINITY;
        for (int j = 0; j < nb; ++j)
            if (j < S || j >= nb - W)
                keep[j] = 1;
        for (int t = 0; t < Tq; ++t) {
            const double *s = scores + (((int64_t)b * Tq + t) * H + h) * dm->max_blocks;
            for (int i = 0; i < n_mid; ++i) {
                r[i].s = s[S + i];
                r[i].j = S + i;
            }
            qsort(r, (size_t)n_mid, sizeof(ranked), rank_cmp);
            double a = -INFINITY;   /* the anchors' best score (mode 2) */
            if (pr->mode == 2)
                for (int j = 0; j < nb; ++j)
                    if ((j < S || j >= nb - W) && s[j] > a) a = s[j];
            double mg;
            int m = row_keep_count(pr, r, n_mid, a, &mg);
            if (mg < mg_row) mg_row = mg;
            for (int i = 0; i < m; ++i)
                keep[r[i].j] = 1;
        }
        int cnt = 0;
        for (int j = 0; j < nb; ++j)
            if (keep[j]) {
                if (cnt >= dm->max_sel) {
                    #pragma omp atomic write
                    err = -2;
                    break;
                }
                sel_idx[bh * dm->max_sel + cnt++] = j;
            }
        sel_count[bh] = cnt;
        if (margin) margin[bh] = mg_row;
        free(keep);
        free(r);
    }
    return err;
}

/* ---------------------------------------------------------- 5. attention */

/*
 * out[b][t][i][c] for the (b, h) units listed in `units` (pairs b, h; NULL
 * means all units): softmax attention of query head i (i / G == h) over
 * every token of the kept blocks of (b, h) that exists (position < L) and is
 * not in the future of query token t (query t sits at position L - Tq + t;
 * the chunk's own keys are already in the cache).  A row with no visible
 * token is all zeros.
 */
int spo_attend(const spo_dims *dm, const spo_params *pr, const uint16_t *q,
               const void *k_cache, const void *v_cache, const float *k_scale,
               const float *v_scale, const int32_t *block_table,
               const int32_t *seq_lens, const int32_t *sel_idx,
               const int32_t *sel_count, const int32_t *units, int n_units,
               double *out, double *lse)
{
    const int D = dm->head_dim, H = dm->num_kv_heads, Tq = dm->q_tokens;
    const int P = dm->block_size, Hq = dm->num_q_heads, G = Hq / H;
    const double scale = softmax_scale(dm, pr);
    int total = units ? n_units : dm->batch * H;
    #pragma omp parallel for schedule(dynamic)
    for (int u = 0; u < total; ++u) {
        int b = units ? units[2 * u] : u / H;
        int h = units ? units[2 * u + 1] : u % H;
        int L = seq_lens[b];
        int64_t bh = (int64_t)b * H + h;
        int cnt = sel_count[bh];
        int ntok_max = cnt * P;
        double *logit = (double *)malloc(sizeof(double) * (size_t)(ntok_max > 0 ? ntok_max : 1));
        int64_t *tpage = (int64_t *)malloc(sizeof(int64_t) * (size_t)(ntok_max > 0 ? ntok_max : 1));
        int *tslot = (int *)malloc(sizeof(int) * (size_t)(ntok_max > 0 ? ntok_max : 1));
        for (int t = 0; t < Tq; ++t) {
            int64_t qpos = (int64_t)L - Tq + t;
            for (int g = 0; g < G; ++g) {
                int i = h * G + g;
                const uint16_t *qr = q + (((int64_t)b * Tq + t) * Hq + i) * D;
                double *o = out + (((int64_t)b * Tq + t) * Hq + i) * D;
                int n = 0;
                for (int s = 0; s < cnt; ++s) {
                    int j = sel_idx[bh * dm->max_sel + s];
                    int64_t page = block_table[(int64_t)b * dm->max_blocks + j];
                    for (int tt = 0; tt < P; ++tt) {
                        int64_t pos = (int64_t)j * P + tt;
                        if (pos >= L || pos > qpos)
                            continue;
                        double dot = 0.0;
                        for (int c = 0; c < D; ++c)
                            dot += spo_bf16_to_f64(qr[c]) *
                                   cache_at(dm, k_cache, k_scale, page, h, tt, c);
                        logit[n] = dot * scale;
                        tpage[n] = page;
                        tslot[n] = tt;
                        ++n;
                    }
                }
                for (int c = 0; c < D; ++c)
                    o[c] = 0.0;
                double *ls = lse ? lse + (((int64_t)b * Tq + t) * Hq + i) : NULL;
                if (ls) *ls = -INFINITY;
                if (n == 0)
                    continue;
                double mx = logit[0];
                for (int k = 1; k < n; ++k)
                    if (logit[k] > mx) mx = logit[k];
                double z = 0.0;
                for (int k = 0; k < n; ++k)
                    z += exp(logit[k] - mx);
                if (ls) *ls = mx + log(z);   /* ln of the sum of exp(logit) */
                for (int k = 0; k < n; ++k) {
                    double p = exp(logit[k] - mx) / z;
                    for (int c = 0; c < D; ++c)
                        o[c] += p * cache_at(dm, v_cache, v_scale, tpage[k], h, tslot[k], c);
                }
            }
        }
        free(logit);
        free(tpage);
        free(tslot);
    }
    return 0;
}

/* ------------------------------------------------- 6. HCA branch (weight-free) */

/*
 * "CSA + HCA 混合注意力机制" §5.1-5.2: every m' consecutive tokens are pooled
 * into one entry and a query attends densely over all entries.  Reading: the
 * pooling is the mean (the page's learned attention pooling needs weights);
 * a group is group_blocks consecutive logical blocks (m' = group_blocks * P).
 * khat/vhat[b][g][h][c] = mean over the group's filled tokens of K / V;
 * groups past a request's end are 0.  Layout [B][G_max][H][D],
 * G_max = ceil(max_blocks / group_blocks).
 */
int spo_hca_pool(const spo_dims *dm, const void *k_cache, const void *v_cache,
                 const float *k_scale, const float *v_scale, const int32_t *block_table,
                 const int32_t *seq_lens, int group_blocks, double *khat, double *vhat)
{
    const int D = dm->head_dim, H = dm->num_kv_heads, P = dm->block_size;
    const int Gmax = (dm->max_blocks + group_blocks - 1) / group_blocks;
    #pragma omp parallel for schedule(dynamic)
    for (int64_t bg = 0; bg < (int64_t)dm->batch * Gmax; ++bg) {
        int b = (int)(bg / Gmax), g = (int)(bg % Gmax);
        int64_t L = seq_lens[b], t0 = (int64_t)g * group_blocks * P;
        int64_t t1 = t0 + (int64_t)group_blocks * P < L ? t0 + (int64_t)group_blocks * P : L;
        for (int h = 0; h < H; ++h) {
            double *kh = khat + ((bg * H) + h) * D, *vh = vhat + ((bg * H) + h) * D;
            for (int c = 0; c < D; ++c)
                kh[c] = vh[c] = 0.0;
            if (t1 <= t0)
                continue;
            for (int64_t tok = t0; tok < t1; ++tok) {
                int64_t page = block_table[(int64_t)b * dm->max_blocks + tok / P];
                for (int c = 0; c < D; ++c) {
                    kh[c] += cache_at(dm, k_cache, k_scale, page, h, (int)(tok % P), c);
                    vh[c] += cache_at(dm, v_cache, v_scale, page, h, (int)(tok % P), c);
                }
            }
            for (int c = 0; c < D; ++c) {
                kh[c] /= (double)(t1 - t0);
                vh[c] /= (double)(t1 - t0);
            }
        }
    }
    return 0;
}

/*
 * Dense attention of every query row over the pooled entries (§5.2: no
 * selection).  Reading: entry g is visible to query token t when all its
 * tokens are at or before the query's position L - Tq + t (no future token
 * inside an entry); scale as the sparse branch; no position tag or sink logit
 * (both need learned values).  out = softmax(q khat^T * scale) vhat; lse = ln
 * of the sum of exp(logit) (-inf with no visible entry, out 0).
 */
int spo_hca_attend(const spo_dims *dm, const spo_params *pr, const uint16_t *q,
                   const double *khat, const double *vhat, const int32_t *seq_lens,
                   int group_blocks, double *out, double *lse)
{
    const int D = dm->head_dim, H = dm->num_kv_heads, Tq = dm->q_tokens;
    const int P = dm->block_size, Hq = dm->num_q_heads, Gq = Hq / H;
    const int Gmax = (dm->max_blocks + group_blocks - 1) / group_blocks;
    const double scale = softmax_scale(dm, pr);
    #pragma omp parallel for schedule(dynamic)
    for (int64_t row = 0; row < (int64_t)dm->batch * Tq * Hq; ++row) {
        int i = (int)(row % Hq), t = (int)((row / Hq) % Tq), b = (int)(row / ((int64_t)Hq * Tq));
        int h = i / Gq;
        int64_t L = seq_lens[b], qpos = L - Tq + t;
        double *o = out + row * D;
        const uint16_t *qr = q + row * D;
        double *logit = (double *)malloc(sizeof(double) * (size_t)Gmax);
        int n = 0;
        for (int g = 0; g < Gmax; ++g) {
            int64_t t0 = (int64_t)g * group_blocks * P;
            int64_t last = t0 + (int64_t)group_blocks * P < L ? t0 + (int64_t)group_blocks * P - 1 : L - 1;
            if (t0 >= L || last > qpos) break;
            const double *kh = khat + (((int64_t)b * Gmax + g) * H + h) * D;
            double dot = 0.0;
            for (int c = 0; c < D; ++c)
                dot += spo_bf16_to_f64(qr[c]) * kh[c];
            logit[n++] = dot * scale;
        }
        for (int c = 0; c < D; ++c)
            o[c] = 0.0;
        lse[row] = -INFINITY;
        if (n > 0) {
            double mx = logit[0], z = 0.0;
            for (int k = 1; k < n; ++k)
                if (logit[k] > mx) mx = logit[k];
            for (int k = 0; k < n; ++k)
                z += exp(logit[k] - mx);
            for (int k = 0; k < n; ++k) {
                double p = exp(logit[k] - mx) / z;
                const double *vh = vhat + (((int64_t)b * Gmax + k) * H + h) * D;
                for (int c = 0; c < D; ++c)
                    o[c] += p * vh[c];
            }
            lse[row] = mx + log(z);
        }
        free(logit);
    }
    return 0;
}

/* Threads the OpenMP runtime will use (1 when built without OpenMP). */
int spo_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Set the number of OpenMP threads later calls use (no effect without
 * OpenMP); the timing of a one-core run of the oracle uses it. */
void spo_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
