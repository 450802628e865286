/*
 * fvattn_oracle.c -- plain, slow fp64 CPU oracle of the adaptive block-sparse
 * attention hot path.
 *
 * TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load this library. The product path
 * (the CUDA library and its Python binding) never calls it, shares no code
 * with it, and fails loudly when its own extension is missing.
 *
 * What it computes, step by step, in the order the pages give it:
 *
 *  1. Video-aware blocks. The latent grid (T,H,W) is cut into (bt,bh,bw)
 *     spatio-temporal blocks; the block count is the product of the per-axis
 *     ceilings, and edge blocks hold fewer ("valid") tokens.
 *     [zskr.cn FastVideo VSA guide, sections 1 and 3 (num_blocks =
 *      ceil(31/4)*ceil(22/8)*ceil(40/8) = 120); section 6 (variable-length edge
 *      blocks, pad rows never act as keys); ai-feeds.com FVAttn summary,
 *      "Key modules" 1 (video-aware block organisation).]
 *     Token n sits at (t,y,x) with n = (t*H + y)*W + x (raster order, T slowest).
 *  2. Block-level scores. Q and K are mean-pooled over the valid tokens of each
 *     block; the score of query block i against key block j is
 *     s[i][j] = scale * dot(Qbar_i, Kbar_j), scale = softmax scale (1/sqrt(D)
 *     by default). [zskr.cn guide, section 1: block-level scoring per query
 *     block; pooling operator = mean over valid tokens (reading).]
 *  3. Softmax of each score row: P[j] = exp(s[j]-max)/sum.
 *  4. Top-p with a Top-k safety floor. Blocks are ranked by P descending
 *     (softmax is strictly increasing in s, so this is the order of s
 *     descending); equal scores rank the lower block index first. The Top-p
 *     count m_p is the smallest m whose inclusive cumulative probability
 *     reaches p (p >= 1 keeps every block); the floor raises it to
 *     m = min(nb, max(m_p, k_min)). [ai-feeds.com summary, "Key modules" 1
 *     (cumulative-probability threshold, Top-k safety lower bound);
 *     hotpaper.ai abstract (Top-p routing, Top-k safety floor).]
 *  5. Mask repair. The diagonal block i is always kept (added as a union).
 *     A row whose scores are not all finite keeps every block and is flagged.
 *     [hotpaper.ai abstract: the materialized mask is repaired at runtime;
 *      ai-feeds.com summary: anomalous patterns are repaired so the mask stays
 *      valid. The diagonal rule and the non-finite rule are readings.]
 *  6. The kept set is emitted as an ascending list of block indices.
 *  7. Attention. Every valid query token r of block i attends to every valid
 *     token of the kept blocks: o_r = sum_k softmax_k(scale*q_r.k_k) v_k.
 *     [ai-feeds.com summary, "Key modules" 1 and the 4.41x result: attention
 *      is computed only over the kept blocks; zskr.cn guide, section 1.]
 *
 * All arithmetic is fp64 on the 16-bit inputs widened exactly: bfloat16
 * (fp16 == 0) or IEEE 754 binary16 (fp16 == 1; the FastVideo VSA backend
 * accepts both, zskr.cn guide, section 5). Loops are parallel over
 * independent (head, block) or (head, token) items only; the arithmetic
 * inside each item runs in the plain order of its definition.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int32_t B, H, T, Hg, W, D, bt, bh, bw;
    int32_t fp16; /* element type of Q, K, V: 0 = bfloat16, 1 = IEEE binary16 */
} oracle_geom;

/* bfloat16: the upper half of an IEEE binary32. */
static double bf16_to_f64(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* IEEE 754 binary16: sign, 5-bit exponent (bias 15), 10-bit fraction.
 * Normal: (1024 + fraction) * 2^(exponent - 25); subnormal (exponent 0):
 * fraction * 2^-24; exponent 31: infinity or NaN. */
static double f16_to_f64(uint16_t h)
{
    const int sign = h >> 15, e = (h >> 10) & 0x1F, m = h & 0x3FF;
    double v;
    if (e == 0) v = ldexp((double)m, -24);
    else if (e == 31) v = m ? NAN : INFINITY;
    else v = ldexp((double)(1024 + m), e - 25);
    return sign ? -v : v;
}

static double elem_to_f64(const oracle_geom *g, uint16_t h)
{
    return g->fp16 ? f16_to_f64(h) : bf16_to_f64(h);
}

/* Widen n raw 16-bit elements of the given type (for the checks of the decode). */
void oracle_widen(int32_t fp16, const uint16_t *x, double *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = fp16 ? f16_to_f64(x[i]) : bf16_to_f64(x[i]);
}

static int ceil_div(int a, int b) { return (a + b - 1) / b; }

int32_t oracle_num_blocks(const oracle_geom *g)
{
    return ceil_div(g->T, g->bt) * ceil_div(g->Hg, g->bh) * ceil_div(g->W, g->bw);
}

/* Valid extent of block j along each axis and its valid token count. */
static void block_extent(const oracle_geom *g, int j, int *t0, int *y0, int *x0,
                         int *tv, int *yv, int *xv)
{
    int nbh = ceil_div(g->Hg, g->bh), nbw = ceil_div(g->W, g->bw);
    int jt = j / (nbh * nbw), jy = (j / nbw) % nbh, jx = j % nbw;
    *t0 = jt * g->bt;
    *y0 = jy * g->bh;
    *x0 = jx * g->bw;
    *tv = (g->T - *t0 < g->bt) ? g->T - *t0 : g->bt;
    *yv = (g->Hg - *y0 < g->bh) ? g->Hg - *y0 : g->bh;
    *xv = (g->W - *x0 < g->bw) ? g->W - *x0 : g->bw;
}

void oracle_block_sizes(const oracle_geom *g, int32_t *valid)
{
    int nb = oracle_num_blocks(g);
    for (int j = 0; j < nb; ++j) {
        int t0, y0, x0, tv, yv, xv;
        block_extent(g, j, &t0, &y0, &x0, &tv, &yv, &xv);
        valid[j] = tv * yv * xv;
    }
}

/* Block index of token n (raster order). */
static int token_block(const oracle_geom *g, int64_t n)
{
    int x = (int)(n % g->W);
    int y = (int)((n / g->W) % g->Hg);
    int t = (int)(n / ((int64_t)g->W * g->Hg));
    int nbh = ceil_div(g->Hg, g->bh), nbw = ceil_div(g->W, g->bw);
    return ((t / g->bt) * nbh + (y / g->bh)) * nbw + (x / g->bw);
}

/* Step 2, first half: out[b,h,j,:] = mean of x[b,h,n,:] over the valid tokens n of block j. */
void oracle_pool(const oracle_geom *g, const uint16_t *x, double *out)
{
    const int nb = oracle_num_blocks(g);
    const int64_t N = (int64_t)g->T * g->Hg * g->W;
    const int D = g->D;
    const int64_t items = (int64_t)g->B * g->H * nb;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t it = 0; it < items; ++it) {
        const int64_t bh = it / nb;
        const int j = (int)(it % nb);
        int t0, y0, x0, tv, yv, xv;
        block_extent(g, j, &t0, &y0, &x0, &tv, &yv, &xv);
        double *o = out + it * D;
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        for (int t = t0; t < t0 + tv; ++t)
            for (int y = y0; y < y0 + yv; ++y)
                for (int xx = x0; xx < x0 + xv; ++xx) {
                    const int64_t n = ((int64_t)t * g->Hg + y) * g->W + xx;
                    const uint16_t *row = x + (bh * N + n) * D;
                    for (int d = 0; d < D; ++d) o[d] += elem_to_f64(g, row[d]);
                }
        const double cnt = (double)(tv * yv * xv);
        for (int d = 0; d < D; ++d) o[d] /= cnt;
    }
}

typedef struct {
    double s;
    int32_t j;
} ranked;

/* Rank by score descending, equal scores by lower block index first. */
static int rank_cmp(const void *a, const void *b)
{
    const ranked *x = (const ranked *)a, *y = (const ranked *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->j < y->j) ? -1 : (x->j > y->j);
}

/*
 * Steps 2 (scores) to 6 for every row (b,h,i).
 *   qbar, kbar : [B,H,nb,D] pooled means (fp64)
 *   kv_cnt     : [B,H,nb]     number of kept blocks per row
 *   kv_idx     : [B,H,nb,nb]  ascending kept block indices (first kv_cnt entries)
 * Optional (NULL to skip), per row of nb entries:
 *   probs      : P[j] in block-index order
 *   order      : the ranking o_0, o_1, ... (step 4)
 *   cum        : inclusive cumulative probability C_r = sum_{q<=r} P[o_q]
 *   nonfinite  : [B,H,nb] 1 where the row's scores were not all finite
 */
void oracle_route(const oracle_geom *g, const double *qbar, const double *kbar,
                  double scale, double p, int32_t k_min,
                  int32_t *kv_cnt, int32_t *kv_idx,
                  double *probs, int32_t *order, double *cum, uint8_t *nonfinite)
{
    const int nb = oracle_num_blocks(g);
    const int D = g->D;
    const int64_t rows = (int64_t)g->B * g->H * nb;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * nb);
        double *P = (double *)malloc(sizeof(double) * nb);
        ranked *rk = (ranked *)malloc(sizeof(ranked) * nb);
        uint8_t *keep = (uint8_t *)malloc(nb);
#pragma omp for schedule(dynamic, 8)
        for (int64_t r = 0; r < rows; ++r) {
            const int64_t bh = r / nb;
            const int i = (int)(r % nb);
            const double *qi = qbar + r * D;
            /* scores */
            int finite = 1;
            for (int j = 0; j < nb; ++j) {
                const double *kj = kbar + (bh * nb + j) * D;
                double acc = 0.0;
                for (int d = 0; d < D; ++d) acc += qi[d] * kj[d];
                s[j] = scale * acc;
                if (!isfinite(s[j])) finite = 0;
            }
            if (nonfinite) nonfinite[r] = (uint8_t)(!finite);
            int32_t *out = kv_idx + r * (int64_t)nb;
            if (!finite) {
                /* repair: an unusable score row keeps every block */
                for (int j = 0; j < nb; ++j) out[j] = j;
                kv_cnt[r] = nb;
                if (probs) for (int j = 0; j < nb; ++j) probs[r * (int64_t)nb + j] = NAN;
                if (order) for (int j = 0; j < nb; ++j) order[r * (int64_t)nb + j] = j;
                if (cum) for (int j = 0; j < nb; ++j) cum[r * (int64_t)nb + j] = NAN;
                continue;
            }
            /* softmax over the row */
            double mx = s[0];
            for (int j = 1; j < nb; ++j) if (s[j] > mx) mx = s[j];
            double z = 0.0;
            for (int j = 0; j < nb; ++j) { P[j] = exp(s[j] - mx); z += P[j]; }
            for (int j = 0; j < nb; ++j) P[j] /= z;
            /* ranking */
            for (int j = 0; j < nb; ++j) { rk[j].s = s[j]; rk[j].j = j; }
            qsort(rk, (size_t)nb, sizeof(ranked), rank_cmp);
            /* Top-p count: smallest m with inclusive cumulative probability >= p */
            int m_p = nb;
            double c = 0.0;
            int found = 0;
            for (int q = 0; q < nb; ++q) {
                c += P[rk[q].j];
                if (cum) cum[r * (int64_t)nb + q] = c;
                if (order) order[r * (int64_t)nb + q] = rk[q].j;
                if (!found && p < 1.0 && c >= p) { m_p = q + 1; found = 1; }
            }
            /* Top-k safety floor, capped at nb */
            int m = m_p > k_min ? m_p : k_min;
            if (m > nb) m = nb;
            memset(keep, 0, (size_t)nb);
            for (int q = 0; q < m; ++q) keep[rk[q].j] = 1;
            keep[i] = 1; /* repair: the diagonal block is always kept */
            int cnt = 0;
            for (int j = 0; j < nb; ++j) if (keep[j]) out[cnt++] = j;
            kv_cnt[r] = cnt;
            if (probs) for (int j = 0; j < nb; ++j) probs[r * (int64_t)nb + j] = P[j];
        }
        free(s);
        free(P);
        free(rk);
        free(keep);
    }
}

/*
 * Step 7 for a list of query tokens.
 *   rows[k] = (b*H + h)*N + n   flat index of the query token
 *   kv_cnt/kv_idx: the kept lists of every (b,h,i) row; NULL for all blocks.
 *   out  : [n_rows, D] attention output
 *   wsum : [n_rows] sum of the normalised attention weights (nullable)
 *   vmin, vmax : [n_rows, D] per-coordinate min/max of the attended V rows
 *                (nullable; used for the convex-combination invariant)
 */
void oracle_attn_rows(const oracle_geom *g, const uint16_t *q, const uint16_t *k,
                      const uint16_t *v, double scale,
                      const int32_t *kv_cnt, const int32_t *kv_idx,
                      int64_t n_rows, const int64_t *rows,
                      double *out, double *wsum, double *vmin, double *vmax)
{
    const int nb = oracle_num_blocks(g);
    const int64_t N = (int64_t)g->T * g->Hg * g->W;
    const int D = g->D;
#pragma omp parallel
    {
        double *qd = (double *)malloc(sizeof(double) * D);
        double *acc = (double *)malloc(sizeof(double) * D);
        /* logits of every attended key, kept so the weights are exp(l - max) */
        double *logit = (double *)malloc(sizeof(double) * (size_t)N);
        int64_t *key = (int64_t *)malloc(sizeof(int64_t) * (size_t)N);
#pragma omp for schedule(dynamic, 1)
        for (int64_t it = 0; it < n_rows; ++it) {
            const int64_t flat = rows[it];
            const int64_t bh = flat / N;
            const int64_t n = flat % N;
            const int i = token_block(g, n);
            const uint16_t *qr = q + (bh * N + n) * D;
            for (int d = 0; d < D; ++d) qd[d] = elem_to_f64(g, qr[d]);
            int cnt = nb;
            const int32_t *lst = NULL;
            if (kv_cnt) {
                cnt = kv_cnt[bh * nb + i];
                lst = kv_idx + (bh * nb + i) * (int64_t)nb;
            }
            int64_t nk = 0;
            double mx = -INFINITY;
            for (int e = 0; e < cnt; ++e) {
                const int j = lst ? lst[e] : e;
                int t0, y0, x0, tv, yv, xv;
                block_extent(g, j, &t0, &y0, &x0, &tv, &yv, &xv);
                for (int t = t0; t < t0 + tv; ++t)
                    for (int y = y0; y < y0 + yv; ++y)
                        for (int x = x0; x < x0 + xv; ++x) {
                            const int64_t m = ((int64_t)t * g->Hg + y) * g->W + x;
                            const uint16_t *kr = k + (bh * N + m) * D;
                            double dot = 0.0;
                            for (int d = 0; d < D; ++d) dot += qd[d] * elem_to_f64(g, kr[d]);
                            logit[nk] = scale * dot;
                            key[nk] = m;
                            if (logit[nk] > mx) mx = logit[nk];
                            ++nk;
                        }
            }
            double z = 0.0;
            for (int64_t e = 0; e < nk; ++e) z += exp(logit[e] - mx);
            for (int d = 0; d < D; ++d) acc[d] = 0.0;
            double ws = 0.0;
            double *lo = vmin ? vmin + it * D : NULL;
            double *hi = vmax ? vmax + it * D : NULL;
            if (lo) for (int d = 0; d < D; ++d) { lo[d] = INFINITY; hi[d] = -INFINITY; }
            for (int64_t e = 0; e < nk; ++e) {
                const double w = exp(logit[e] - mx) / z;
                ws += w;
                const uint16_t *vr = v + (bh * N + key[e]) * D;
                for (int d = 0; d < D; ++d) {
                    const double vv = elem_to_f64(g, vr[d]);
                    acc[d] += w * vv;
                    if (lo) {
                        if (vv < lo[d]) lo[d] = vv;
                        if (vv > hi[d]) hi[d] = vv;
                    }
                }
            }
            for (int d = 0; d < D; ++d) out[it * D + d] = acc[d];
            if (wsum) wsum[it] = ws;
        }
        free(qd);
        free(acc);
        free(logit);
        free(key);
    }
}

/*
 * Slack-aware sparse augmentation (SASA) of one problem's kept lists.
 * [ai-feeds.com FVAttn summary, "Key modules" 3: after load balancing, ranks
 *  below the critical path spend their spare compute on extra high-value
 *  attention blocks, chosen by attention score, without lengthening the
 *  critical path; hotpaper.ai summary, SASA bullet.]
 * Reading taken: a candidate is a (row, block j) pair whose block the row
 * does not keep; its value is the block probability P[row][j] and its cost
 * the token pairs it adds, |i| * |j|. Candidates are taken in the order of
 * value (P descending; equal values by row, then block, ascending) for as
 * long as the total cost stays within the budget (the rank's slack): the
 * first candidate that does not fit ends the augmentation.
 *   probs          [B,H,nb,nb] block probabilities (oracle_route)
 *   kv_cnt/kv_idx  in/out: the lists, ascending
 *   added_pairs    out: token pairs added
 *   added_mass     out: sum of the added candidates' P
 */
typedef struct {
    double p;
    int64_t row;
    int32_t j;
} candidate;

static int candidate_cmp(const void *a, const void *b)
{
    const candidate *x = (const candidate *)a, *y = (const candidate *)b;
    if (x->p > y->p) return -1;
    if (x->p < y->p) return 1;
    if (x->row != y->row) return x->row < y->row ? -1 : 1;
    return (x->j < y->j) ? -1 : (x->j > y->j);
}

void oracle_augment(const oracle_geom *g, const double *probs, int64_t budget,
                    int32_t *kv_cnt, int32_t *kv_idx, int64_t *added_pairs, double *added_mass)
{
    const int nb = oracle_num_blocks(g);
    const int64_t rows = (int64_t)g->B * g->H * nb;
    int32_t *size = (int32_t *)malloc(sizeof(int32_t) * nb);
    uint8_t *keep = (uint8_t *)calloc((size_t)(rows * nb), 1);
    oracle_block_sizes(g, size);
    for (int64_t r = 0; r < rows; ++r)
        for (int e = 0; e < kv_cnt[r]; ++e) keep[r * nb + kv_idx[r * (int64_t)nb + e]] = 1;
    int64_t n = 0;
    for (int64_t x = 0; x < rows * nb; ++x) n += !keep[x];
    candidate *c = (candidate *)malloc(sizeof(candidate) * (size_t)(n > 0 ? n : 1));
    n = 0;
    for (int64_t r = 0; r < rows; ++r)
        for (int j = 0; j < nb; ++j)
            if (!keep[r * nb + j]) {
                c[n].p = probs[r * (int64_t)nb + j];
                c[n].row = r;
                c[n].j = j;
                ++n;
            }
    qsort(c, (size_t)n, sizeof(candidate), candidate_cmp);
    int64_t spent = 0;
    double mass = 0.0;
    for (int64_t x = 0; x < n; ++x) {
        const int i = (int)(c[x].row % nb);
        const int64_t cost = (int64_t)size[i] * size[c[x].j];
        if (spent + cost > budget) break;
        spent += cost;
        mass += c[x].p;
        keep[c[x].row * nb + c[x].j] = 1;
    }
    for (int64_t r = 0; r < rows; ++r) {
        int cnt = 0;
        for (int j = 0; j < nb; ++j)
            if (keep[r * nb + j]) kv_idx[r * (int64_t)nb + cnt++] = j;
        kv_cnt[r] = cnt;
    }
    if (added_pairs) *added_pairs = spent;
    if (added_mass) *added_mass = mass;
    free(c);
    free(keep);
    free(size);
}
