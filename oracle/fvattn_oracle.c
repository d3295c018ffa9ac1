/*
 * fvattn_oracle.c -- TEST INFRASTRUCTURE, not part of the product.
 *
 * A plain, slow, fp64 CPU statement of what top-p routed block-sparse attention
 * computes.  Only the test suite, the smoke check and the benchmark's CPU
 * baseline leg load this library.  It shares no code, header, table or helper
 * with the CUDA library; the two meet only in the seeded input generators.
 *
 * Sources (page title, then section):
 *  [FVAttn]  "[논문리뷰] FVAttn: Adaptive Sparse Attention with Runtime Load
 *            Balancing for Video Generation", §1 Key Terms (Top-p routing):
 *            for every query block, key blocks are taken in order of an
 *            importance score until their cumulative probability reaches p.
 *            §1 (RLB) and §2: the per-head amount of work is what is balanced.
 *  [FA]      "FlashAttention - Fast and Memory-Efficient Exact Attention with
 *            IO-Awareness" review, §Background [3] Motivation: S = QK^T,
 *            P = softmax(S), O = PV; §Model "Tiling Softmax": the row softmax
 *            is computed block by block and the partial results are combined
 *            exactly.
 *
 * The pages name the routing score but never define it.  This library fixes
 * it as: mean-pool every block of `bs` tokens of Q and of K (over the tokens
 * that exist), score = qbar . kbar / sqrt(d), softmax over all key blocks,
 * and keep the shortest prefix of key blocks -- sorted by descending score,
 * equal scores by ascending index -- whose probability mass is >= p
 * (p >= 1 keeps every block).
 *
 * Precision: bf16 inputs are widened to fp64 exactly; every sum runs in fp64
 * in index order.  Compile with -ffp-contract=off so that a*b+c is two
 * roundings, exactly as written.
 *
 * Parity pins (what this file is checked against, in tests/):
 *   pool        closed forms (constant and ramp blocks, ragged last block)
 *   route       top-p invariants, K = 0 uniform closed form (tie-break),
 *               one-hot block, p -> 0+ argmax, p = 1 all blocks, monotone in p,
 *               exhaustive subset search on tiny rows
 *   attn_rows   high-precision Decimal brute force on tiny inputs, closed
 *               forms (single key, K = 0 mean of V, constant V)
 *   attn_tiled  equals attn_rows (the "exact" tiling identity of [FA])
 *   attn_bwd    central finite differences of a numpy fp64 brute-force forward,
 *               fp64 torch autograd of dense attention, and the dense-case
 *               identities sum_u dK_u = 0 and sum_u dV_u = sum_t dO_t
 *   attn_bwd_sampled  equal, value for value, to attn_bwd at the sampled
 *               tokens, and to fp64 torch autograd of dense attention
 *   lpt_order   brute-force sort on small inputs
 *   head_order  brute-force sort on small inputs
 *   pair_items  a hand-worked example (odd nb, empty rows, shared and single
 *               blocks); on random rows, set unions and each row recovered from
 *               its bits
 *   route candidates  the blocks right after the cut in the routing order:
 *               exhaustive comparison with the selected set's complement
 *   sasa        Graham's list-scheduling bound, loads within the makespan,
 *               slack used up unless candidates run out, hand-worked examples
 *   rlb_plan    hand-worked plans, every move lowers the sum of squared loads,
 *               the final state admits no improving move, exhaustive optimum
 *               never beaten on tiny instances
 *   e4m3 / quant_e4m3  the format's own values (known codes, ties to even,
 *               saturation, NaN), round trip of every finite code, monotone
 *               encoding, block scales putting the block maximum in (224, 448],
 *               the half-ulp error bound, exact bf16 representability
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- helpers */

static double bf16_bits_to_double(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f; /* float -> double is exact */
}

static int64_t num_blocks(int N, int bs) { return ((int64_t)N + bs - 1) / bs; }

/* Simple parallel-for over [0, n) with a fixed number of threads. */
typedef void (*range_fn)(void *ctx, int64_t begin, int64_t end);
typedef struct {
    range_fn fn;
    void *ctx;
    int64_t begin, end;
} range_job;

static void *range_trampoline(void *arg) {
    range_job *j = (range_job *)arg;
    j->fn(j->ctx, j->begin, j->end);
    return NULL;
}

static void parallel_for(int64_t n, int nthreads, range_fn fn, void *ctx) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (n < nthreads) nthreads = (int)(n > 0 ? n : 1);
    if (nthreads == 1) {
        fn(ctx, 0, n);
        return;
    }
    pthread_t th[256];
    range_job jobs[256];
    int started[256];
    int64_t chunk = (n + nthreads - 1) / nthreads;
    for (int i = 0; i < nthreads; ++i) {
        jobs[i].fn = fn;
        jobs[i].ctx = ctx;
        jobs[i].begin = i * chunk < n ? i * chunk : n;
        jobs[i].end = (i + 1) * chunk < n ? (i + 1) * chunk : n;
        started[i] = pthread_create(&th[i], NULL, range_trampoline, &jobs[i]) == 0;
        if (!started[i]) fn(ctx, jobs[i].begin, jobs[i].end);
    }
    for (int i = 0; i < nthreads; ++i)
        if (started[i]) pthread_join(th[i], NULL);
}

/* ------------------------------------------------------------ mean pooling */
/*
 * out[bh, i, c] = (1/n_i) * sum_{t in block i, t < N} X[bh, t, c]
 * n_i counts only the tokens that exist (the last block may be ragged).
 */
typedef struct {
    const uint16_t *X;
    int N, d, bs;
    int64_t nb;
    double *out;
} pool_ctx;

static void pool_range(void *vctx, int64_t begin, int64_t end) {
    pool_ctx *c = (pool_ctx *)vctx;
    for (int64_t u = begin; u < end; ++u) { /* u = bh * nb + i */
        int64_t bh = u / c->nb, i = u % c->nb;
        int64_t t0 = i * c->bs, t1 = t0 + c->bs;
        if (t1 > c->N) t1 = c->N;
        double *o = c->out + u * c->d;
        for (int ch = 0; ch < c->d; ++ch) {
            double s = 0.0;
            for (int64_t t = t0; t < t1; ++t)
                s = s + bf16_bits_to_double(c->X[(bh * c->N + t) * c->d + ch]);
            o[ch] = s / (double)(t1 - t0);
        }
    }
}

int oracle_pool(const uint16_t *X, int64_t BH, int N, int d, int bs, double *out, int nthreads) {
    if (!X || !out || BH < 0 || N < 1 || d < 1 || bs < 1) return -1;
    pool_ctx c = {X, N, d, bs, num_blocks(N, bs), out};
    parallel_for(BH * c.nb, nthreads, pool_range, &c);
    return 0;
}

/* ------------------------------------------------------------ top-p routing */

typedef struct {
    double s; /* score */
    int j;    /* key-block index */
} scored_block;

/* Descending score; equal scores by ascending index. */
static int by_score_desc_index_asc(const void *a, const void *b) {
    const scored_block *x = (const scored_block *)a, *y = (const scored_block *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->j > y->j) - (x->j < y->j);
}

typedef struct {
    const double *qbar, *kbar; /* [BH, nb, d] */
    int d;
    int64_t nb;
    double p, scale;
    int32_t *counts;  /* [rows] */
    uint8_t *chosen;  /* [rows, nb] 0/1 */
    double *diag;     /* [rows, 6] or NULL */
    int32_t *cand;    /* [rows, kc] or NULL: the next key blocks after the cut, in routing order */
    double *cand_p;   /* [rows, kc] or NULL: their probabilities */
    int kc;
} route_ctx;

/*
 * One row = one (b, h, query block i).  Steps in the order of [FVAttn] §1:
 * importance score per key block, probability by softmax, then key blocks in
 * descending order until the cumulative probability reaches p.
 */
static void route_range(void *vctx, int64_t begin, int64_t end) {
    route_ctx *c = (route_ctx *)vctx;
    int64_t nb = c->nb;
    scored_block *sb = (scored_block *)malloc(sizeof(scored_block) * nb);
    double *prob = (double *)malloc(sizeof(double) * nb);
    if (!sb || !prob) {
        free(sb);
        free(prob);
        return;
    }
    for (int64_t row = begin; row < end; ++row) {
        int64_t bh = row / nb;
        const double *q = c->qbar + row * c->d;
        /* scores s_j = (qbar_i . kbar_j) * (1/sqrt(d)) */
        double smax = -INFINITY;
        for (int64_t j = 0; j < nb; ++j) {
            const double *k = c->kbar + (bh * nb + j) * c->d;
            double dot = 0.0;
            for (int ch = 0; ch < c->d; ++ch) dot = dot + q[ch] * k[ch];
            sb[j].s = dot * c->scale;
            sb[j].j = (int)j;
            if (sb[j].s > smax) smax = sb[j].s;
        }
        /* softmax over key blocks */
        double z = 0.0;
        for (int64_t j = 0; j < nb; ++j) {
            prob[j] = exp(sb[j].s - smax);
            z = z + prob[j];
        }
        for (int64_t j = 0; j < nb; ++j) prob[j] = prob[j] / z;
        /* order by score, cut where the cumulative mass first reaches p */
        qsort(sb, (size_t)nb, sizeof(scored_block), by_score_desc_index_asc);
        int64_t k = nb - 1; /* p >= 1, or mass never reaches p: all blocks */
        double cum = 0.0, cum_prev = 0.0, cum_at_k = 0.0;
        if (c->p < 1.0) {
            for (int64_t r = 0; r < nb; ++r) {
                cum_prev = cum;
                cum = cum + prob[sb[r].j];
                if (cum >= c->p) {
                    k = r;
                    break;
                }
            }
            cum_at_k = cum;
        } else {
            for (int64_t r = 0; r < nb; ++r) {
                cum_prev = cum;
                cum = cum + prob[sb[r].j];
            }
            cum_at_k = cum;
        }
        uint8_t *ch = c->chosen + row * nb;
        for (int64_t j = 0; j < nb; ++j) ch[j] = 0;
        for (int64_t r = 0; r <= k; ++r) ch[sb[r].j] = 1;
        c->counts[row] = (int32_t)(k + 1);
        if (c->cand) {
            for (int e = 0; e < c->kc; ++e) {
                int64_t r = k + 1 + e;
                c->cand[row * c->kc + e] = (r < nb) ? (int32_t)sb[r].j : -1;
                if (c->cand_p) c->cand_p[row * c->kc + e] = (r < nb) ? prob[sb[r].j] : 0.0;
            }
        }
        if (c->diag) {
            double *g = c->diag + row * 6;
            g[0] = cum_at_k;                                     /* mass kept */
            g[1] = cum_prev;                                     /* mass without the last kept block */
            g[2] = sb[k].s;                                      /* last kept score */
            g[3] = (k + 1 < nb) ? sb[k + 1].s : -INFINITY;       /* first dropped score */
            g[4] = prob[sb[k].j];                                /* last kept probability */
            g[5] = (k + 1 < nb) ? prob[sb[k + 1].j] : 0.0;       /* first dropped probability */
        }
    }
    free(sb);
    free(prob);
}

/*
 * Full routing: pooled Q and K, scores, softmax, top-p selection, CSR with
 * ascending column indices inside each row, and per-head selected-block counts.
 * Returns 0, -1 on bad arguments, -4 when col_capacity is too small.
 */
int oracle_route_cand(const uint16_t *Q, const uint16_t *K, int B, int H, int N, int d, int bs, double p,
                      int32_t *row_ptr, int32_t *col_idx, int64_t col_capacity, int32_t *head_counts,
                      double *diag, int32_t *cand, double *cand_p, int kc, int nthreads) {
    if (!Q || !K || !row_ptr || !head_counts || B < 1 || H < 1 || N < 1 || d < 1 || bs < 1) return -1;
    if (!(p > 0.0) || p > 1.0) return -1;
    int64_t BH = (int64_t)B * H, nb = num_blocks(N, bs), rows = BH * nb;
    double *qbar = (double *)malloc(sizeof(double) * rows * d);
    double *kbar = (double *)malloc(sizeof(double) * rows * d);
    int32_t *counts = (int32_t *)malloc(sizeof(int32_t) * rows);
    uint8_t *chosen = (uint8_t *)malloc((size_t)(rows * nb));
    int rc = 0;
    if (!qbar || !kbar || !counts || !chosen) {
        rc = -1;
        goto done;
    }
    oracle_pool(Q, BH, N, d, bs, qbar, nthreads);
    oracle_pool(K, BH, N, d, bs, kbar, nthreads);
    route_ctx c = {qbar, kbar, d, nb, p, 1.0 / sqrt((double)d), counts, chosen, diag, cand, cand_p, kc};
    parallel_for(rows, nthreads, route_range, &c);
    /* CSR: exclusive prefix sum of the row counts, columns ascending */
    int64_t total = 0;
    for (int64_t r = 0; r < rows; ++r) {
        row_ptr[r] = (int32_t)total;
        total += counts[r];
    }
    row_ptr[rows] = (int32_t)total;
    if (total > col_capacity || !col_idx) {
        rc = -4;
    } else {
        for (int64_t r = 0; r < rows; ++r) {
            int64_t w = row_ptr[r];
            for (int64_t j = 0; j < nb; ++j)
                if (chosen[r * nb + j]) col_idx[w++] = (int32_t)j;
        }
    }
    for (int64_t bh = 0; bh < BH; ++bh) {
        int64_t s = 0;
        for (int64_t i = 0; i < nb; ++i) s += counts[bh * nb + i];
        head_counts[bh] = (int32_t)s;
    }
done:
    free(qbar);
    free(kbar);
    free(counts);
    free(chosen);
    return rc;
}

int oracle_route(const uint16_t *Q, const uint16_t *K, int B, int H, int N, int d, int bs, double p,
                 int32_t *row_ptr, int32_t *col_idx, int64_t col_capacity, int32_t *head_counts,
                 double *diag, int nthreads) {
    return oracle_route_cand(Q, K, B, H, N, d, bs, p, row_ptr, col_idx, col_capacity, head_counts, diag, NULL,
                             NULL, 0, nthreads);
}

/* ------------------------------------------------- attention, row by row */

typedef struct {
    const uint16_t *Q, *K, *V;
    int H, N, d, bs, causal;
    int64_t nb;
    const int32_t *row_ptr, *col_idx;
    const int64_t *tokens; /* global token index bh*N + t */
    double *O, *LSE;
    double scale;
} attn_ctx;

/*
 * The textbook definition of [FA] §Motivation, restricted to the key tokens
 * of the blocks listed in the query token's CSR row (and u <= t if causal):
 *   s_u = q_t . k_u / sqrt(d),  O_t = sum_u softmax(s)_u v_u,
 *   LSE_t = ln sum_u exp(s_u).
 * An empty key set gives O = 0 and LSE = -inf.
 */
static void attn_rows_range(void *vctx, int64_t begin, int64_t end) {
    attn_ctx *c = (attn_ctx *)vctx;
    int d = c->d;
    double *q = (double *)malloc(sizeof(double) * d);
    double *acc = (double *)malloc(sizeof(double) * d);
    int64_t cap = c->nb * c->bs;
    double *s = (double *)malloc(sizeof(double) * cap);
    int64_t *u_of = (int64_t *)malloc(sizeof(int64_t) * cap);
    if (!q || !acc || !s || !u_of) goto out;
    for (int64_t it = begin; it < end; ++it) {
        int64_t g = c->tokens[it], bh = g / c->N, t = g % c->N;
        int64_t row = bh * c->nb + t / c->bs;
        for (int ch = 0; ch < d; ++ch) q[ch] = bf16_bits_to_double(c->Q[g * d + ch]);
        int64_t n = 0;
        double m = -INFINITY;
        for (int32_t e = c->row_ptr[row]; e < c->row_ptr[row + 1]; ++e) {
            int64_t kb = c->col_idx[e];
            for (int64_t u = kb * c->bs; u < (kb + 1) * c->bs && u < c->N; ++u) {
                if (c->causal && u > t) continue;
                const uint16_t *k = c->K + (bh * c->N + u) * d;
                double dot = 0.0;
                for (int ch = 0; ch < d; ++ch) dot = dot + q[ch] * bf16_bits_to_double(k[ch]);
                s[n] = dot * c->scale;
                u_of[n] = u;
                if (s[n] > m) m = s[n];
                ++n;
            }
        }
        double *o = c->O + it * d;
        if (n == 0) {
            for (int ch = 0; ch < d; ++ch) o[ch] = 0.0;
            c->LSE[it] = -INFINITY;
            continue;
        }
        double z = 0.0;
        for (int ch = 0; ch < d; ++ch) acc[ch] = 0.0;
        for (int64_t a = 0; a < n; ++a) {
            double w = exp(s[a] - m);
            z = z + w;
            const uint16_t *v = c->V + (bh * c->N + u_of[a]) * d;
            for (int ch = 0; ch < d; ++ch) acc[ch] = acc[ch] + w * bf16_bits_to_double(v[ch]);
        }
        for (int ch = 0; ch < d; ++ch) o[ch] = acc[ch] / z;
        c->LSE[it] = m + log(z);
    }
out:
    free(q);
    free(acc);
    free(s);
    free(u_of);
}

int oracle_attn_rows(const uint16_t *Q, const uint16_t *K, const uint16_t *V, int B, int H, int N, int d, int bs,
                     int causal, const int32_t *row_ptr, const int32_t *col_idx, const int64_t *tokens,
                     int64_t ntok, double *O, double *LSE, int nthreads) {
    if (!Q || !K || !V || !row_ptr || !col_idx || !tokens || !O || !LSE) return -1;
    if (B < 1 || H < 1 || N < 1 || d < 1 || bs < 1) return -1;
    int64_t total = (int64_t)B * H * N;
    for (int64_t i = 0; i < ntok; ++i)
        if (tokens[i] < 0 || tokens[i] >= total) return -1;
    attn_ctx c = {Q, K, V, H, N, d, bs, causal ? 1 : 0, num_blocks(N, bs), row_ptr, col_idx, tokens, O, LSE,
                  1.0 / sqrt((double)d)};
    parallel_for(ntok, nthreads, attn_rows_range, &c);
    return 0;
}

/* -------------------------------------- attention, tiled online softmax */

/*
 * The same quantity, computed the way [FA] §Model "Tiling Softmax" describes:
 * one key block at a time, keeping a running maximum m, a running sum l and
 * an unnormalised output; when the maximum grows from m to m', the old sum
 * and output are scaled by exp(m - m').  In exact arithmetic this equals
 * attn_rows; the tests pin the two against each other.
 */
static void attn_tiled_range(void *vctx, int64_t begin, int64_t end) {
    attn_ctx *c = (attn_ctx *)vctx;
    int d = c->d;
    double *q = (double *)malloc(sizeof(double) * d);
    double *acc = (double *)malloc(sizeof(double) * d);
    double *s = (double *)malloc(sizeof(double) * c->bs);
    int64_t *u_of = (int64_t *)malloc(sizeof(int64_t) * c->bs);
    if (!q || !acc || !s || !u_of) goto out;
    for (int64_t it = begin; it < end; ++it) {
        int64_t g = c->tokens[it], bh = g / c->N, t = g % c->N;
        int64_t row = bh * c->nb + t / c->bs;
        for (int ch = 0; ch < d; ++ch) {
            q[ch] = bf16_bits_to_double(c->Q[g * d + ch]);
            acc[ch] = 0.0;
        }
        double m = -INFINITY, l = 0.0;
        for (int32_t e = c->row_ptr[row]; e < c->row_ptr[row + 1]; ++e) {
            int64_t kb = c->col_idx[e];
            int n = 0;
            double mt = -INFINITY;
            for (int64_t u = kb * c->bs; u < (kb + 1) * c->bs && u < c->N; ++u) {
                if (c->causal && u > t) continue;
                const uint16_t *k = c->K + (bh * c->N + u) * d;
                double dot = 0.0;
                for (int ch = 0; ch < d; ++ch) dot = dot + q[ch] * bf16_bits_to_double(k[ch]);
                s[n] = dot * c->scale;
                u_of[n] = u;
                if (s[n] > mt) mt = s[n];
                ++n;
            }
            if (n == 0) continue;
            double mn = mt > m ? mt : m;
            double alpha = (m == -INFINITY) ? 0.0 : exp(m - mn);
            l = l * alpha;
            for (int ch = 0; ch < d; ++ch) acc[ch] = acc[ch] * alpha;
            for (int a = 0; a < n; ++a) {
                double w = exp(s[a] - mn);
                l = l + w;
                const uint16_t *v = c->V + (bh * c->N + u_of[a]) * d;
                for (int ch = 0; ch < d; ++ch) acc[ch] = acc[ch] + w * bf16_bits_to_double(v[ch]);
            }
            m = mn;
        }
        double *o = c->O + it * d;
        if (l == 0.0) {
            for (int ch = 0; ch < d; ++ch) o[ch] = 0.0;
            c->LSE[it] = -INFINITY;
        } else {
            for (int ch = 0; ch < d; ++ch) o[ch] = acc[ch] / l;
            c->LSE[it] = m + log(l);
        }
    }
out:
    free(q);
    free(acc);
    free(s);
    free(u_of);
}

int oracle_attn_tiled(const uint16_t *Q, const uint16_t *K, const uint16_t *V, int B, int H, int N, int d, int bs,
                      int causal, const int32_t *row_ptr, const int32_t *col_idx, const int64_t *tokens,
                      int64_t ntok, double *O, double *LSE, int nthreads) {
    if (!Q || !K || !V || !row_ptr || !col_idx || !tokens || !O || !LSE) return -1;
    if (B < 1 || H < 1 || N < 1 || d < 1 || bs < 1) return -1;
    int64_t total = (int64_t)B * H * N;
    for (int64_t i = 0; i < ntok; ++i)
        if (tokens[i] < 0 || tokens[i] >= total) return -1;
    attn_ctx c = {Q, K, V, H, N, d, bs, causal ? 1 : 0, num_blocks(N, bs), row_ptr, col_idx, tokens, O, LSE,
                  1.0 / sqrt((double)d)};
    parallel_for(ntok, nthreads, attn_tiled_range, &c);
    return 0;
}

/* ----------------------------------------------- longest-first work order */

typedef struct {
    int64_t count;
    int64_t id;
} work_item;

static int by_count_desc_id_asc(const void *a, const void *b) {
    const work_item *x = (const work_item *)a, *y = (const work_item *)b;
    if (x->count != y->count) return x->count > y->count ? -1 : 1;
    return (x->id > y->id) - (x->id < y->id);
}

/*
 * Work items are the CSR rows (one query block of one head).  The order is
 * longest first -- descending selected-block count, equal counts by ascending
 * row id -- the single-GPU counterpart of balancing per-head work after the
 * mask is known ([FVAttn] §1 RLB, §3).
 */
int oracle_lpt_order(const int32_t *row_ptr, int64_t rows, int32_t *order) {
    if (!row_ptr || !order || rows < 0) return -1;
    work_item *w = (work_item *)malloc(sizeof(work_item) * (rows > 0 ? rows : 1));
    if (!w) return -1;
    for (int64_t r = 0; r < rows; ++r) {
        w[r].count = (int64_t)row_ptr[r + 1] - row_ptr[r];
        w[r].id = r;
    }
    qsort(w, (size_t)rows, sizeof(work_item), by_count_desc_id_asc);
    for (int64_t r = 0; r < rows; ++r) order[r] = (int32_t)w[r].id;
    free(w);
    return 0;
}

/* ---------------------------------------- attention gradients, row by row */
/*
 * Gradients of the loss L = sum_t dO_t . O_t for the attention of attn_rows
 * (the training use the [FA] review measures in §Experiments 1 "Training
 * Efficiency" needs them; the pages print no formulas, so these are the plain
 * derivatives of the definition above).  Per query token t with allowed keys
 * u (its CSR row's blocks, u < N, u <= t if causal), s_u = q_t . k_u / sqrt(d),
 * P_u = softmax(s)_u, O_t = sum_u P_u v_u:
 *   dV_u += P_u dO_t
 *   dP_u  = dO_t . v_u,   D_t = dO_t . O_t,   dS_u = P_u (dP_u - D_t)
 *   dQ_t  = sum_u dS_u k_u / sqrt(d)
 *   dK_u += dS_u q_t / sqrt(d)
 * One thread owns one (batch, head): all its accumulations are private, and
 * every sum runs over t and u in index order.  A token with no allowed key
 * contributes nothing (its O is 0).
 */
typedef struct {
    const uint16_t *Q, *K, *V, *dO;
    int N, d, bs, causal;
    int64_t nb;
    const int32_t *row_ptr, *col_idx;
    double *dQ, *dK, *dV;
    double scale;
} bwd_ctx;

static void attn_bwd_range(void *vctx, int64_t begin, int64_t end) {
    bwd_ctx *c = (bwd_ctx *)vctx;
    int d = c->d;
    int64_t cap = c->nb * c->bs;
    double *q = (double *)malloc(sizeof(double) * d);
    double *go = (double *)malloc(sizeof(double) * d);
    double *o = (double *)malloc(sizeof(double) * d);
    double *p = (double *)malloc(sizeof(double) * cap);
    int64_t *u_of = (int64_t *)malloc(sizeof(int64_t) * cap);
    if (!q || !go || !o || !p || !u_of) goto out;
    for (int64_t bh = begin; bh < end; ++bh) {
        const int64_t base = bh * c->N * d;
        for (int64_t i = 0; i < (int64_t)c->N * d; ++i) {
            c->dQ[base + i] = 0.0;
            c->dK[base + i] = 0.0;
            c->dV[base + i] = 0.0;
        }
        for (int64_t t = 0; t < c->N; ++t) {
            int64_t row = bh * c->nb + t / c->bs;
            for (int ch = 0; ch < d; ++ch) {
                q[ch] = bf16_bits_to_double(c->Q[base + t * d + ch]);
                go[ch] = bf16_bits_to_double(c->dO[base + t * d + ch]);
            }
            /* scores and softmax over the allowed keys */
            int64_t n = 0;
            double m = -INFINITY;
            for (int32_t e = c->row_ptr[row]; e < c->row_ptr[row + 1]; ++e) {
                int64_t kb = c->col_idx[e];
                for (int64_t u = kb * c->bs; u < (kb + 1) * c->bs && u < c->N; ++u) {
                    if (c->causal && u > t) continue;
                    double dot = 0.0;
                    for (int ch = 0; ch < d; ++ch) dot = dot + q[ch] * bf16_bits_to_double(c->K[base + u * d + ch]);
                    p[n] = dot * c->scale;
                    u_of[n] = u;
                    if (p[n] > m) m = p[n];
                    ++n;
                }
            }
            if (n == 0) continue;
            double z = 0.0;
            for (int64_t a = 0; a < n; ++a) {
                p[a] = exp(p[a] - m);
                z = z + p[a];
            }
            for (int64_t a = 0; a < n; ++a) p[a] = p[a] / z;
            /* O_t and D_t */
            for (int ch = 0; ch < d; ++ch) o[ch] = 0.0;
            for (int64_t a = 0; a < n; ++a)
                for (int ch = 0; ch < d; ++ch) o[ch] = o[ch] + p[a] * bf16_bits_to_double(c->V[base + u_of[a] * d + ch]);
            double D = 0.0;
            for (int ch = 0; ch < d; ++ch) D = D + go[ch] * o[ch];
            /* the gradients */
            double *dq = c->dQ + base + t * d;
            for (int64_t a = 0; a < n; ++a) {
                const int64_t u = u_of[a];
                double dp = 0.0;
                for (int ch = 0; ch < d; ++ch) dp = dp + go[ch] * bf16_bits_to_double(c->V[base + u * d + ch]);
                const double ds = p[a] * (dp - D);
                double *dv = c->dV + base + u * d, *dk = c->dK + base + u * d;
                for (int ch = 0; ch < d; ++ch) {
                    dv[ch] = dv[ch] + p[a] * go[ch];
                    dq[ch] = dq[ch] + ds * bf16_bits_to_double(c->K[base + u * d + ch]) * c->scale;
                    dk[ch] = dk[ch] + ds * q[ch] * c->scale;
                }
            }
        }
    }
out:
    free(q);
    free(go);
    free(o);
    free(p);
    free(u_of);
}

int oracle_attn_bwd(const uint16_t *Q, const uint16_t *K, const uint16_t *V, const uint16_t *dO, int B, int H, int N,
                    int d, int bs, int causal, const int32_t *row_ptr, const int32_t *col_idx, double *dQ, double *dK,
                    double *dV, int nthreads) {
    if (!Q || !K || !V || !dO || !row_ptr || !col_idx || !dQ || !dK || !dV) return -1;
    if (B < 1 || H < 1 || N < 1 || d < 1 || bs < 1) return -1;
    bwd_ctx c = {Q, K, V, dO, N, d, bs, causal, num_blocks(N, bs), row_ptr, col_idx, dQ, dK, dV,
                 1.0 / sqrt((double)d)};
    parallel_for((int64_t)B * H, nthreads, attn_bwd_range, &c);
    return 0;
}

/* ------------------------------ gradients of sampled query and key tokens */

/*
 * The same derivatives as oracle_attn_bwd, evaluated only where asked, so that
 * the gradients of full-size problems can be checked on samples:
 *   dQ_t for the listed query tokens (one row's softmax each), and
 *   dK_u, dV_u for the listed key tokens, summed over every query token t whose
 *   CSR row lists u's block (u <= t if causal), t in index order.
 * Key tokens come grouped by (batch*head, key block) through group_ptr: one
 * query row's softmax serves every key of its group.  Per row the operations
 * and their order are those of oracle_attn_bwd, so both give identical values.
 */
typedef struct {
    const uint16_t *Q, *K, *V, *dO;
    int N, d, bs, causal;
    int64_t nb;
    const int32_t *row_ptr, *col_idx;
    double scale;
    int64_t nq;
    const int64_t *q_tok;
    double *dQ;
    const int64_t *k_tok, *group_ptr;
    double *dK, *dV;
} bwd_sample_ctx;

/* Softmax row of query token t of head bh: fills p (probabilities), u_of, o, and
 * returns the number of allowed keys and D_t = dO_t . O_t (q and go filled). */
static int64_t bwd_row(const bwd_sample_ctx *c, int64_t bh, int64_t t, double *q, double *go, double *o,
                       double *p, int64_t *u_of, double *D_out) {
    const int d = c->d;
    const int64_t base = bh * c->N * d;
    const int64_t row = bh * c->nb + t / c->bs;
    for (int ch = 0; ch < d; ++ch) {
        q[ch] = bf16_bits_to_double(c->Q[base + t * d + ch]);
        go[ch] = bf16_bits_to_double(c->dO[base + t * d + ch]);
    }
    int64_t n = 0;
    double m = -INFINITY;
    for (int32_t e = c->row_ptr[row]; e < c->row_ptr[row + 1]; ++e) {
        int64_t kb = c->col_idx[e];
        for (int64_t u = kb * c->bs; u < (kb + 1) * c->bs && u < c->N; ++u) {
            if (c->causal && u > t) continue;
            double dot = 0.0;
            for (int ch = 0; ch < d; ++ch) dot = dot + q[ch] * bf16_bits_to_double(c->K[base + u * d + ch]);
            p[n] = dot * c->scale;
            u_of[n] = u;
            if (p[n] > m) m = p[n];
            ++n;
        }
    }
    if (n == 0) return 0;
    double z = 0.0;
    for (int64_t a = 0; a < n; ++a) {
        p[a] = exp(p[a] - m);
        z = z + p[a];
    }
    for (int64_t a = 0; a < n; ++a) p[a] = p[a] / z;
    for (int ch = 0; ch < d; ++ch) o[ch] = 0.0;
    for (int64_t a = 0; a < n; ++a)
        for (int ch = 0; ch < d; ++ch) o[ch] = o[ch] + p[a] * bf16_bits_to_double(c->V[base + u_of[a] * d + ch]);
    double D = 0.0;
    for (int ch = 0; ch < d; ++ch) D = D + go[ch] * o[ch];
    *D_out = D;
    return n;
}

static void bwd_sample_range(void *vctx, int64_t begin, int64_t end) {
    bwd_sample_ctx *c = (bwd_sample_ctx *)vctx;
    const int d = c->d;
    const int64_t cap = c->nb * c->bs;
    double *q = (double *)malloc(sizeof(double) * d);
    double *go = (double *)malloc(sizeof(double) * d);
    double *o = (double *)malloc(sizeof(double) * d);
    double *p = (double *)malloc(sizeof(double) * cap);
    int64_t *u_of = (int64_t *)malloc(sizeof(int64_t) * cap);
    if (!q || !go || !o || !p || !u_of) goto out;
    for (int64_t it = begin; it < end; ++it) {
        if (it < c->nq) { /* dQ of one query token */
            const int64_t g = c->q_tok[it], bh = g / c->N, t = g % c->N;
            const int64_t base = bh * c->N * d;
            double *dq = c->dQ + it * d;
            for (int ch = 0; ch < d; ++ch) dq[ch] = 0.0;
            double D = 0.0;
            const int64_t n = bwd_row(c, bh, t, q, go, o, p, u_of, &D);
            for (int64_t a = 0; a < n; ++a) {
                const int64_t u = u_of[a];
                double dp = 0.0;
                for (int ch = 0; ch < d; ++ch) dp = dp + go[ch] * bf16_bits_to_double(c->V[base + u * d + ch]);
                const double ds = p[a] * (dp - D);
                for (int ch = 0; ch < d; ++ch)
                    dq[ch] = dq[ch] + ds * bf16_bits_to_double(c->K[base + u * d + ch]) * c->scale;
            }
            continue;
        }
        /* dK, dV of one group of key tokens (same head, same key block) */
        const int64_t gi = it - c->nq;
        const int64_t k0 = c->group_ptr[gi], k1 = c->group_ptr[gi + 1];
        if (k1 <= k0) continue;
        const int64_t bh = c->k_tok[k0] / c->N, kb = (c->k_tok[k0] % c->N) / c->bs;
        const int64_t base = bh * c->N * d;
        for (int64_t k = k0; k < k1; ++k)
            for (int ch = 0; ch < d; ++ch) {
                c->dK[k * d + ch] = 0.0;
                c->dV[k * d + ch] = 0.0;
            }
        for (int64_t qb = 0; qb < c->nb; ++qb) {
            const int64_t row = bh * c->nb + qb;
            int listed = 0;
            for (int32_t e = c->row_ptr[row]; e < c->row_ptr[row + 1]; ++e)
                if (c->col_idx[e] == kb) listed = 1;
            if (!listed) continue;
            for (int64_t t = qb * c->bs; t < (qb + 1) * c->bs && t < c->N; ++t) {
                double D = 0.0;
                const int64_t n = bwd_row(c, bh, t, q, go, o, p, u_of, &D);
                for (int64_t a = 0; a < n; ++a) {
                    const int64_t u = u_of[a];
                    for (int64_t k = k0; k < k1; ++k) {
                        if (c->k_tok[k] % c->N != u) continue;
                        double dp = 0.0;
                        for (int ch = 0; ch < d; ++ch)
                            dp = dp + go[ch] * bf16_bits_to_double(c->V[base + u * d + ch]);
                        const double ds = p[a] * (dp - D);
                        double *dv = c->dV + k * d, *dk = c->dK + k * d;
                        for (int ch = 0; ch < d; ++ch) {
                            dv[ch] = dv[ch] + p[a] * go[ch];
                            dk[ch] = dk[ch] + ds * q[ch] * c->scale;
                        }
                    }
                }
            }
        }
    }
out:
    free(q);
    free(go);
    free(o);
    free(p);
    free(u_of);
}

int oracle_attn_bwd_sampled(const uint16_t *Q, const uint16_t *K, const uint16_t *V, const uint16_t *dO, int B,
                            int H, int N, int d, int bs, int causal, const int32_t *row_ptr, const int32_t *col_idx,
                            const int64_t *q_tok, int64_t nq, double *dQ, const int64_t *k_tok,
                            const int64_t *group_ptr, int64_t ngroups, double *dK, double *dV, int nthreads) {
    if (!Q || !K || !V || !dO || !row_ptr || !col_idx) return -1;
    if (B < 1 || H < 1 || N < 1 || d < 1 || bs < 1 || nq < 0 || ngroups < 0) return -1;
    if ((nq > 0 && (!q_tok || !dQ)) || (ngroups > 0 && (!k_tok || !group_ptr || !dK || !dV))) return -1;
    const int64_t total = (int64_t)B * H * N;
    for (int64_t i = 0; i < nq; ++i)
        if (q_tok[i] < 0 || q_tok[i] >= total) return -1;
    for (int64_t gi = 0; gi < ngroups; ++gi) {
        if (group_ptr[gi + 1] < group_ptr[gi]) return -1;
        for (int64_t k = group_ptr[gi]; k < group_ptr[gi + 1]; ++k) {
            if (k_tok[k] < 0 || k_tok[k] >= total) return -1;
            if (k_tok[k] / N != k_tok[group_ptr[gi]] / N ||
                (k_tok[k] % N) / bs != (k_tok[group_ptr[gi]] % N) / bs)
                return -1; /* a group spans one head and one key block */
        }
    }
    bwd_sample_ctx c = {Q, K, V, dO, N, d, bs, causal ? 1 : 0, num_blocks(N, bs), row_ptr, col_idx,
                        1.0 / sqrt((double)d), nq, q_tok, dQ, k_tok, group_ptr, dK, dV};
    parallel_for(nq + ngroups, nthreads, bwd_sample_range, &c);
    return 0;
}

/* --------------------------------------------- FP8 (e4m3) block quantization */

/*
 * For the FP8 attention variant (e4m3 Q, K, V).  "Accelerating HunyuanVideo
 * inference with ParaAttention" (WaveSpeed), § "FP8 dynamic quantization",
 * quantizes activations to FP8 at run time but names no format or scaling, so
 * the reading here is the plainest exact one:
 *   - e4m3 as in the OCP FP8 E4M3FN format: 1 sign bit, 4 exponent bits (bias
 *     7), 3 mantissa bits, subnormals m * 2^-9, largest finite 448, no
 *     infinities (0x7F / 0xFF are NaN);
 *   - one power-of-two scale 2^e per (batch*head, block of bs tokens), the
 *     smallest e with absmax * 2^-e <= 448 (e = 0 for an all-zero block), so
 *     that dividing by the scale is exact in any precision (a block holding
 *     inf keeps 2^0; NaN does not count toward the maximum);
 *   - each value x * 2^-e rounded to the nearest e4m3 value, ties to the even
 *     code, magnitudes above 448 saturated to 448.
 * Dequantized value = e4m3 value * 2^e.
 */
double oracle_e4m3_to_double(uint8_t b) {
    const int sign = b >> 7, ex = (b >> 3) & 15, man = b & 7;
    if (ex == 15 && man == 7) return NAN;
    const double mag = (ex == 0) ? ldexp((double)man, -9) : ldexp(1.0 + man / 8.0, ex - 7);
    return sign ? -mag : mag;
}

uint8_t oracle_e4m3_from_double(double x) {
    if (isnan(x)) return 0x7F;
    const uint8_t sign = (x < 0.0 || (x == 0.0 && signbit(x))) ? 0x80 : 0x00;
    const double a = fabs(x);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    /* the finite non-negative codes 0x00..0x7E are in increasing order of value:
       find the two neighbours of a and take the nearer one, ties to the even code */
    int lo = 0, hi = 0x7E;
    while (hi - lo > 1) {
        const int mid = (lo + hi) / 2;
        if (oracle_e4m3_to_double((uint8_t)mid) <= a) lo = mid;
        else hi = mid;
    }
    const double vlo = oracle_e4m3_to_double((uint8_t)lo), vhi = oracle_e4m3_to_double((uint8_t)hi);
    int code;
    if (a - vlo < vhi - a) code = lo;
    else if (a - vlo > vhi - a) code = hi;
    else code = (lo % 2 == 0) ? lo : hi;
    if (a <= vlo) code = lo;
    return (uint8_t)(sign | code);
}

/* X: bf16 bit patterns [BH, N, d].  out: e4m3 codes [BH, N, d]; scale_exp: int32
 * [BH, nb] (the e of each block's scale 2^e).  Rows past N do not exist. */
int oracle_quant_e4m3(const uint16_t *X, int64_t BH, int N, int d, int bs, uint8_t *out, int32_t *scale_exp) {
    if (!X || !out || !scale_exp || BH < 1 || N < 1 || d < 1 || bs < 1) return -1;
    const int64_t nb = num_blocks(N, bs);
    for (int64_t bh = 0; bh < BH; ++bh) {
        for (int64_t b = 0; b < nb; ++b) {
            const int64_t t0 = b * bs, t1 = (b + 1) * bs < N ? (b + 1) * bs : N;
            double amax = 0.0;
            for (int64_t t = t0; t < t1; ++t)
                for (int ch = 0; ch < d; ++ch) {
                    const double v = fabs(bf16_bits_to_double(X[(bh * N + t) * d + ch]));
                    if (v > amax) amax = v;
                }
            int e = 0;
            if (amax > 0.0 && isfinite(amax)) { /* a block holding inf keeps the scale 2^0 */
                e = -200;
                while (ldexp(amax, -e) > 448.0) ++e;
            }
            scale_exp[bh * nb + b] = e;
            for (int64_t t = t0; t < t1; ++t)
                for (int ch = 0; ch < d; ++ch) {
                    const int64_t i = (bh * N + t) * d + ch;
                    out[i] = oracle_e4m3_from_double(ldexp(bf16_bits_to_double(X[i]), -e));
                }
        }
    }
    return 0;
}

/* ------------------------------------------------ head-major work order */

typedef struct {
    int64_t key; /* selected blocks */
    int64_t id;
} keyed_id;

static int by_key_desc_id_asc(const void *a, const void *b) {
    const keyed_id *x = (const keyed_id *)a, *y = (const keyed_id *)b;
    if (x->key != y->key) return (x->key < y->key) - (x->key > y->key);
    return (x->id > y->id) - (x->id < y->id);
}

/*
 * The order the attention kernel takes its work items in ([FVAttn] §1 RLB:
 * per-head work balanced at run time; here over the SMs of one GPU): heads by
 * their total selected blocks (descending, equal totals by lower head), then the
 * rows of each head by block count (descending, equal counts by lower row).
 */
int oracle_head_order(const int32_t *row_ptr, int64_t BH, int64_t nb, int32_t *order) {
    if (!row_ptr || !order || BH < 1 || nb < 1) return -1;
    keyed_id *h = (keyed_id *)malloc(sizeof(keyed_id) * BH);
    keyed_id *r = (keyed_id *)malloc(sizeof(keyed_id) * nb);
    if (!h || !r) {
        free(h);
        free(r);
        return -1;
    }
    for (int64_t b = 0; b < BH; ++b) {
        h[b].key = (int64_t)row_ptr[(b + 1) * nb] - row_ptr[b * nb];
        h[b].id = b;
    }
    qsort(h, (size_t)BH, sizeof(keyed_id), by_key_desc_id_asc);
    int64_t w = 0;
    for (int64_t x = 0; x < BH; ++x) {
        int64_t b = h[x].id;
        for (int64_t i = 0; i < nb; ++i) {
            r[i].key = (int64_t)row_ptr[b * nb + i + 1] - row_ptr[b * nb + i];
            r[i].id = b * nb + i;
        }
        qsort(r, (size_t)nb, sizeof(keyed_id), by_key_desc_id_asc);
        for (int64_t i = 0; i < nb; ++i) order[w++] = (int32_t)r[i].id;
    }
    free(h);
    free(r);
    return 0;
}

/*
 * The attention's work items at a block of 64 tokens.  A tensor-core tile holds
 * 128 query rows, two query blocks; the kernel gives it query blocks 2i and
 * 2i+1 of one head (the last one alone when the head has an odd number of
 * blocks), and the tile visits every key block either of the two selected
 * ([FVAttn] §1 Key Terms, top-p routing: each query block keeps its own set).
 * For pair i of head b (np = ceil(nb / 2) pairs per head, item id b * np + i)
 * this writes the union of the two rows' key blocks, ascending, as a CSR
 * (pair_ptr [BH*np + 1], pair_col), and pair_bits[e] = 1 if row 2i selected
 * block pair_col[e], + 2 if row 2i+1 did.  The rows must hold ascending, in-range
 * indices; the union is their two-way merge.  The work of an item (what the
 * queue of oracle_head_order sorts by) is its union size.
 */
int oracle_pair_items(const int32_t *row_ptr, const int32_t *col_idx, int64_t BH, int64_t nb, int32_t *pair_ptr,
                      int32_t *pair_col, int32_t *pair_bits) {
    if (!row_ptr || !pair_ptr || BH < 1 || nb < 1) return -1;
    const int64_t np = (nb + 1) / 2;
    int64_t w = 0;
    pair_ptr[0] = 0;
    for (int64_t b = 0; b < BH; ++b) {
        for (int64_t i = 0; i < np; ++i) {
            const int64_t ra = b * nb + 2 * i;
            int64_t ia = row_ptr[ra], ea = row_ptr[ra + 1];
            int64_t ib = 0, eb = 0;
            if (2 * i + 1 < nb) {
                ib = row_ptr[ra + 1];
                eb = row_ptr[ra + 2];
            }
            while (ia < ea || ib < eb) {
                if (ib >= eb || (ia < ea && col_idx[ia] < col_idx[ib])) {
                    pair_col[w] = col_idx[ia++];
                    pair_bits[w] = 1;
                } else if (ia >= ea || col_idx[ib] < col_idx[ia]) {
                    pair_col[w] = col_idx[ib++];
                    pair_bits[w] = 2;
                } else {
                    pair_col[w] = col_idx[ia];
                    pair_bits[w] = 3;
                    ++ia;
                    ++ib;
                }
                ++w;
            }
            pair_ptr[b * np + i + 1] = (int32_t)w;
        }
    }
    return 0;
}

/* ------------------------------------------- slack-aware augmentation (SASA) */

/*
 * [FVAttn] §1 Key Terms (SASA) and §3: after the work has been balanced, the
 * ranks that still have idle time (slack) before the slowest one finishes
 * compute additional high-value key blocks, raising quality at no cost in time.
 * On one GPU the ranks are the `machines` SMs of the persistent attention grid:
 *   1. schedule: the rows, taken in the attention's queue order `order`, each go
 *      to the machine with the least load so far (equal loads: the lowest
 *      machine), a row's load being its selected-block count; the makespan T is
 *      the largest load;
 *   2. augmentation: each machine m, with slack T - load_m, walks its rows in
 *      the order they were assigned, round after round, giving each row its next
 *      candidate block (the rows' unselected blocks in routing order, at most kc
 *      of them, cand[row, e] < 0 marks the end) at a cost of one block each,
 *      until the slack is used up or no row of m has a candidate left;
 *   3. the augmented mask: each row's selected blocks plus its added ones, in
 *      ascending order.
 * added[row] receives the number of blocks added, added_mass[row] their
 * probability (the sum of cand_p over them, in the order added).
 * Returns 0, -1 on bad arguments, -4 when col_capacity is too small.
 */
int oracle_sasa(const int32_t *row_ptr, const int32_t *col_idx, int64_t rows, const int32_t *cand,
                const double *cand_p, int kc, const int32_t *order, int machines, int32_t *added,
                double *added_mass, int32_t *row_ptr_out, int32_t *col_idx_out, int64_t col_capacity) {
    if (!row_ptr || !col_idx || !cand || !order || !added || !row_ptr_out || machines < 1 || kc < 0 ||
        rows < 0)
        return -1;
    int64_t *load = (int64_t *)calloc((size_t)machines, sizeof(int64_t));
    int32_t *mach = (int32_t *)malloc(sizeof(int32_t) * (rows > 0 ? rows : 1));
    int64_t *seq = (int64_t *)malloc(sizeof(int64_t) * (rows > 0 ? rows : 1)); /* rows in assignment order */
    if (!load || !mach || !seq) {
        free(load);
        free(mach);
        free(seq);
        return -1;
    }
    /* 1. list schedule in queue order */
    for (int64_t x = 0; x < rows; ++x) {
        int64_t row = order[x];
        int best = 0;
        for (int m = 1; m < machines; ++m)
            if (load[m] < load[best]) best = m;
        mach[row] = best;
        load[best] += (int64_t)row_ptr[row + 1] - row_ptr[row];
        seq[x] = row;
    }
    int64_t T = 0;
    for (int m = 0; m < machines; ++m)
        if (load[m] > T) T = load[m];
    /* 2. fill each machine's slack with its rows' next candidates, round robin */
    for (int64_t row = 0; row < rows; ++row) {
        added[row] = 0;
        if (added_mass) added_mass[row] = 0.0;
    }
    for (int m = 0; m < machines; ++m) {
        int64_t slack = T - load[m];
        while (slack > 0) {
            int progress = 0;
            for (int64_t x = 0; x < rows && slack > 0; ++x) {
                int64_t row = seq[x];
                if (mach[row] != m) continue;
                int e = added[row];
                if (e < kc && cand[row * kc + e] >= 0) {
                    if (added_mass) added_mass[row] = added_mass[row] + (cand_p ? cand_p[row * kc + e] : 0.0);
                    added[row] = e + 1;
                    --slack;
                    progress = 1;
                }
            }
            if (!progress) break;
        }
    }
    /* 3. augmented CSR, columns ascending */
    int64_t total = 0;
    for (int64_t row = 0; row < rows; ++row) {
        row_ptr_out[row] = (int32_t)total;
        total += (int64_t)row_ptr[row + 1] - row_ptr[row] + added[row];
    }
    row_ptr_out[rows] = (int32_t)total;
    int rc = 0;
    if (total > col_capacity || !col_idx_out) {
        rc = -4;
    } else {
        for (int64_t row = 0; row < rows; ++row) {
            int32_t *dst = col_idx_out + row_ptr_out[row];
            int64_t n = 0;
            for (int32_t e = row_ptr[row]; e < row_ptr[row + 1]; ++e) dst[n++] = col_idx[e];
            for (int e = 0; e < added[row]; ++e) dst[n++] = cand[row * kc + e];
            /* insertion sort: the row is short and almost sorted */
            for (int64_t a = 1; a < n; ++a) {
                int32_t v = dst[a];
                int64_t b = a - 1;
                while (b >= 0 && dst[b] > v) {
                    dst[b + 1] = dst[b];
                    --b;
                }
                dst[b + 1] = v;
            }
        }
    }
    free(load);
    free(mach);
    free(seq);
    return rc;
}

/* ------------------------------------------ run-time load balancing (RLB) */

/*
 * [FVAttn] §1 Key Terms (RLB) and §3: once routing has fixed every head's amount
 * of work, heads move between GPUs (P2P) so that the critical path shortens.
 * Units are (batch, head) pairs; work[r * units + i] is the selected-block count
 * of unit i of rank r (units per rank, all ranks alike).  The plan, step by step:
 * the most loaded rank (lowest index on ties) gives the least loaded rank
 * (lowest index on ties) the unit it holds with the largest work below their gap
 * (among equal works the unit with the lowest home index r * units + i), as long
 * as such a unit exists (the move then lowers both loads below the old maximum).
 * A unit may move again later.  Writes the moves in
 * order: move_unit[k] = r * units + i (the unit's home), move_src[k], move_dst[k];
 * *n_moves their number (at most max_moves).  Returns 0, -1 on bad arguments.
 */
int oracle_rlb_plan(const int64_t *work, int ranks, int units, int max_moves, int32_t *move_unit, int32_t *move_src,
                    int32_t *move_dst, int32_t *n_moves) {
    if (!work || ranks < 1 || units < 0 || max_moves < 0 || !n_moves) return -1;
    int64_t total = (int64_t)ranks * units;
    int32_t *owner = (int32_t *)malloc(sizeof(int32_t) * (total > 0 ? total : 1));
    int64_t *load = (int64_t *)calloc((size_t)ranks, sizeof(int64_t));
    if (!owner || !load) {
        free(owner);
        free(load);
        return -1;
    }
    for (int64_t u = 0; u < total; ++u) {
        owner[u] = (int32_t)(u / units);
        load[u / units] += work[u];
    }
    int k = 0;
    while (k < max_moves) {
        int src = 0, dst = 0;
        for (int r = 1; r < ranks; ++r) {
            if (load[r] > load[src]) src = r;
            if (load[r] < load[dst]) dst = r;
        }
        int64_t gap = load[src] - load[dst];
        int64_t best = -1;
        for (int64_t u = 0; u < total; ++u) {
            if (owner[u] != src || work[u] <= 0 || work[u] >= gap) continue;
            if (best < 0 || work[u] > work[best]) best = u;
        }
        if (best < 0) break;
        owner[best] = dst;
        load[src] -= work[best];
        load[dst] += work[best];
        if (move_unit) move_unit[k] = (int32_t)best;
        if (move_src) move_src[k] = src;
        if (move_dst) move_dst[k] = dst;
        ++k;
    }
    *n_moves = k;
    free(owner);
    free(load);
    return 0;
}
