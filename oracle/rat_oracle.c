/*
 * rat_oracle.c -- plain, slow CPU oracle for the RAT+ temporal-mixing operator.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and
 * its Python binding) may include, link or call this file; only the tests, the
 * smoke check and the benchmark's CPU-baseline leg use it.  It shares no code,
 * header, table or constant with the CUDA path.
 *
 * Everything is computed in IEEE double, straight from the definitions, with no
 * blocking, fusion or reordering.  OpenMP only spreads independent output rows
 * or channels over host threads; it does not change any sum's order.
 *
 * Sources (titles of the pages the operator is defined on):
 *   [RAT+]  "RAT+: Train Dense, Infer Sparse -- Recurrence Augmented Attention
 *           for Dilated Inference": Abstract; Figure 1(a) (full-sequence
 *           recurrence, L=T); Figure 1(c) (dilated attention, optional local
 *           attention); Figure 2 (prefill by a scan, decode by a step update).
 *   [MEM]   "Augmenting Attention with Exponentially Decaying Memory Improves
 *           Query-Aware KV Sparsity": section 2.1 (key and value states updated
 *           with an input-dependent gate; exponentially decaying memory).
 *   [RAT]   "RAT: Bridging RNN Efficiency and Attention Accuracy via
 *           Chunk-based Sequence Modeling": Approach (gated linear recurrence;
 *           chunk size L=T makes the layer an RNN).
 *
 * Readings taken where the pages leave a step open (each is also listed in the
 * design notes):
 *   R1 recurrence: per channel c, s_t = a_t*s_{t-1} + (1-a_t)*x_t with
 *      a_t = sigmoid(g_t); one gate tensor g drives both the key and the value
 *      recurrence; s_{-1} = init (zero unless given).
 *   R2 dilation: query t attends to { j : 0 <= j <= t, (t-j) mod D == 0 }.
 *   R3 window: W > 0 adds the dense set { j : max(0,t-W+1) <= j <= t }.
 *   R4 the two parts are two separate softmaxes merged by log-sum-exp, so a
 *      key in both sets (j = t always is) is counted once in each part.
 *   R5 score scale s = 1/sqrt(d) unless the caller gives one; the query is not
 *      recurrence-augmented; both parts read the augmented keys and values.
 *   R6 a head with recur = 0 uses a = 0, i.e. augmented keys/values equal the
 *      raw ones (D = 1, a = 0 is plain causal attention).
 *   R7 (a second reading, kept for comparison) fixed-grid dilation: query t
 *      attends to { j <= t : j mod D == D - 1 } plus t (oracle_attn_rows_grid).
 *   R8 (a variant, off by default) dedupe: a key in both parts counts once,
 *      i.e. the window part skips the keys of the dilated set
 *      (oracle_attn_rows_ex).
 *   R9 top-k block attention (oracle_attn_rows_topk): blocks of bs keys; the
 *      first and the query's own block are always kept, K more are chosen by
 *      score; the Quest-style score is the per-channel min/max upper bound
 *      sum_c max(q_c*kmin_c, q_c*kmax_c), the MoBA-style score q . mean(k);
 *      ties go to the lower block index; blocks hold the augmented keys.
 *
 * Parity pins for every function here live in tests/test_oracle_pins.py.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>

/* element (b,t,h,c) of a row-major [B,T,H,d] tensor */
static size_t idx4(int T, int H, int d, int b, long t, int h, int c)
{
    return (((size_t)b * (size_t)T + (size_t)t) * (size_t)H + (size_t)h) * (size_t)d + (size_t)c;
}

static double sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }

/*
 * R1: the gated linear recurrence, one channel at a time, t = 0 .. T-1 in order
 * ([MEM] 2.1; [RAT+] Figure 1(a) L=T; [RAT] Approach).
 *   x, g   : [B,T,H,d]           input and gate logit
 *   init   : [B,H,d] or NULL     s_{-1}; NULL means zero
 *   recur  : [H] or NULL         0 => a = 0 for that head (R6); NULL => all 1
 *   out    : [B,T,H,d]           s_t for every t
 *   final  : [B,H,d] or NULL     s_{T-1} (init when T = 0)
 */
void oracle_scan(int B, int T, int H, int d, const double *x, const double *g,
                 const double *init, const unsigned char *recur, double *out,
                 double *final)
{
    long nch = (long)B * H * d;
#pragma omp parallel for schedule(static)
    for (long ch = 0; ch < nch; ++ch) {
        int b = (int)(ch / ((long)H * d));
        int h = (int)((ch / d) % H);
        int c = (int)(ch % d);
        int rec = recur ? (recur[h] != 0) : 1;
        double s = init ? init[ch] : 0.0;
        for (long t = 0; t < T; ++t) {
            size_t e = idx4(T, H, d, b, t, h, c);
            double a = rec ? sigmoid(g[e]) : 0.0;
            s = a * s + (1.0 - a) * x[e];
            out[e] = s;
        }
        if (final) final[ch] = s;
    }
}

/*
 * Softmax of q_t against the key set `js` (n entries) of head h in batch b:
 *   z_j = scale * sum_c q[c]*k_j[c];  lse = log sum_j exp(z_j);
 *   o[c] = sum_j exp(z_j - lse) * v_j[c].
 * The maximum is subtracted before exp only to avoid overflow; it cancels.
 */
static void softmax_over(int T, int H, int d, const double *qrow, const double *k,
                         const double *v, int b, int h, const long *js, long n,
                         double scale, double *o, double *lse, double *z)
{
    double m = -INFINITY;
    for (long i = 0; i < n; ++i) {
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += qrow[c] * k[idx4(T, H, d, b, js[i], h, c)];
        z[i] = scale * acc;
        if (z[i] > m) m = z[i];
    }
    double den = 0.0;
    for (long i = 0; i < n; ++i) den += exp(z[i] - m);
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    for (long i = 0; i < n; ++i) {
        double p = exp(z[i] - m) / den;
        for (int c = 0; c < d; ++c) o[c] += p * v[idx4(T, H, d, b, js[i], h, c)];
    }
    *lse = m + log(den);
}

/* R4: merge two (output, log-sum-exp) pairs as one softmax over both sets. */
static void lse_merge(int d, const double *o1, double l1, const double *o2, double l2,
                      double *o, double *lse)
{
    double m = l1 > l2 ? l1 : l2;
    double w1 = exp(l1 - m), w2 = exp(l2 - m);
    for (int c = 0; c < d; ++c) o[c] = (w1 * o1[c] + w2 * o2[c]) / (w1 + w2);
    *lse = m + log(w1 + w2);
}

/*
 * One output row per requested (b, h, t) of the attention step over the
 * augmented keys kt and values vt ([RAT+] Abstract and Figure 1(c)).
 *   q, kt, vt : [B,T,H,d]
 *   dil, win  : [H]  dilation D_h >= 1, window W_h >= 0
 *   parts     : 1 = dilated part only (R2), 2 = window part only (R3),
 *               3 = the operator's output: dilated part, merged with the window
 *                   part when W_h > 0 (R4)
 *   rows      : nrows x 3 int64 (b, h, t)
 *   o, lse    : nrows x d, nrows
 * Returns 0, or -1 on an argument error (the outputs are then untouched).
 */
static int attn_rows_impl(int B, int T, int H, int d, const double *q, const double *kt,
                          const double *vt, const int *dil, const int *win, double scale,
                          int parts, long nrows, const int64_t *rows, double *o, double *lse,
                          int grid, int dedupe)
{
    if (parts < 1 || parts > 3) return -1;
    for (long r = 0; r < nrows; ++r) {
        int64_t b = rows[3 * r], h = rows[3 * r + 1], t = rows[3 * r + 2];
        if (b < 0 || b >= B || h < 0 || h >= H || t < 0 || t >= T) return -1;
        if (dil[h] < 1 || win[h] < 0) return -1;
        if (parts == 2 && win[h] == 0) return -1;
    }
    int err = 0;
#pragma omp parallel
    {
        long *js = (long *)malloc(sizeof(long) * (size_t)(T > 0 ? T : 1));
        double *z = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
        double *o1 = (double *)malloc(sizeof(double) * (size_t)d);
        double *o2 = (double *)malloc(sizeof(double) * (size_t)d);
        if (!js || !z || !o1 || !o2) {
#pragma omp atomic write
            err = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (long r = 0; r < nrows; ++r) {
            if (err) continue;
            int b = (int)rows[3 * r], h = (int)rows[3 * r + 1];
            long t = (long)rows[3 * r + 2];
            const double *qrow = q + idx4(T, H, d, b, t, h, 0);
            int D = dil[h], W = win[h];
            double l1 = 0.0, l2 = 0.0;
            if (parts & 1) {
                long n = 0;
                if (!grid) { /* R2: j <= t with (t - j) mod D == 0 */
                    for (long j = 0; j <= t; ++j)
                        if ((t - j) % D == 0) js[n++] = j;
                } else {    /* fixed grid: j <= t on the grid j mod D == D - 1, plus t */
                    for (long j = 0; j <= t; ++j)
                        if (j % D == D - 1 || j == t) js[n++] = j;
                }
                softmax_over(T, H, d, qrow, kt, vt, b, h, js, n, scale, o1, &l1, z);
            }
            if ((parts & 2) && W > 0) { /* R3: max(0, t-W+1) <= j <= t */
                long n = 0;
                for (long j = 0; j <= t; ++j)
                    if (j >= t - W + 1) js[n++] = j;
                if (dedupe) { /* R8: keys the dilated part holds count once */
                    long n2 = 0;
                    for (long i = 0; i < n; ++i) {
                        const long j = js[i];
                        const int in_dil = grid ? (j % D == D - 1 || j == t) : ((t - j) % D == 0);
                        if (!in_dil) js[n2++] = j;
                    }
                    n = n2;
                }
                softmax_over(T, H, d, qrow, kt, vt, b, h, js, n, scale, o2, &l2, z);
            }
            double *orow = o + (size_t)r * (size_t)d;
            if (parts == 1 || (parts == 3 && W == 0)) {
                for (int c = 0; c < d; ++c) orow[c] = o1[c];
                lse[r] = l1;
            } else if (parts == 2) {
                for (int c = 0; c < d; ++c) orow[c] = o2[c];
                lse[r] = l2;
            } else {
                lse_merge(d, o1, l1, o2, l2, orow, &lse[r]);
            }
        }
        free(js); free(z); free(o1); free(o2);
    }
    return err ? -1 : 0;
}

int oracle_attn_rows(int B, int T, int H, int d, const double *q, const double *kt,
                     const double *vt, const int *dil, const int *win, double scale,
                     int parts, long nrows, const int64_t *rows, double *o, double *lse)
{
    return attn_rows_impl(B, T, H, d, q, kt, vt, dil, win, scale, parts, nrows, rows, o, lse, 0, 0);
}

/*
 * The same rows under the fixed-grid reading of dilation, kept for comparison
 * with R4 ([RAT+] Abstract: dilation cuts the KV cache by a factor of D;
 * [RAT] Approach: attention over chunk-level keys, one per chunk of D tokens).
 * Query t's dilated part attends to the keys on a grid shared by all queries,
 * { j <= t : j mod D == D - 1 }, plus t itself; so a decode cache needs only
 * one row per D positions.  For t with t mod D == D - 1 the set equals R2's.
 * The window part and the merge are R3 and R4, unchanged.
 */
int oracle_attn_rows_grid(int B, int T, int H, int d, const double *q, const double *kt,
                          const double *vt, const int *dil, const int *win, double scale,
                          int parts, long nrows, const int64_t *rows, double *o, double *lse)
{
    return attn_rows_impl(B, T, H, d, q, kt, vt, dil, win, scale, parts, nrows, rows, o, lse, 1, 0);
}

/*
 * Both readings and both merge variants in one call: grid != 0 takes the
 * fixed-grid dilated set (R7), dedupe != 0 drops from the window part the keys
 * the dilated part already holds (R8), so that the merge is one softmax over
 * the union of the two sets rather than over their multiset.
 */
int oracle_attn_rows_ex(int B, int T, int H, int d, const double *q, const double *kt,
                        const double *vt, const int *dil, const int *win, double scale,
                        int parts, long nrows, const int64_t *rows, double *o, double *lse,
                        int grid, int dedupe)
{
    return attn_rows_impl(B, T, H, d, q, kt, vt, dil, win, scale, parts, nrows, rows, o, lse,
                          grid != 0, dedupe != 0);
}

/*
 * Top-k block attention over the augmented keys/values, the sparse-inference
 * setting the pages evaluate on RAT+ ([RAT+] Figure 3 and Tables 17-18;
 * [MEM] "Sparse inference settings").  Keys are grouped into blocks of `bs`
 * consecutive positions.  Query t (in block c = floor(t / bs)) attends, over
 * j <= t, to the keys of
 *   - block 0 and block c (the first and the local block are always kept),
 *   - the K highest-scoring of blocks 1 .. c-1 (all of them when there are at
 *     most K; equal scores go to the lower block index).
 * A block's score against q_t:
 *   mode 0 (Quest-style, per-channel min/max statistics of the block's keys):
 *          sum_c max(q_c * kmin_c, q_c * kmax_c), an upper bound of q.k over
 *          any key inside the block's per-channel ranges;
 *   mode 1 (MoBA-style, mean-pooled keys): q . mean_j(k_j).
 * Reading R9 (the pages name the methods and their statistics but print no
 * formula): the Quest score is that upper bound; K counts the blocks chosen
 * besides the first and the local one; the blocks hold the augmented keys.
 * Output and log-sum-exp are those of one softmax over the attended keys
 * (scale as in R5).
 */

/* R9 block selection for query row t of (b, h): marks keep[0 .. c] (c = t/bs)
 * and lists the picked candidates in picks[0 .. K) in the order they are
 * taken (-1 when fewer than K candidates exist).  *gap receives the score of
 * the last pick minus the best score left out (+inf when nothing is left out
 * or nothing is picked), how far the selection is from a tie. */
static void topk_pick(int T, int H, int d, const double *qrow, const double *kt, int b, int h, long t,
                      int bs, int K, int mode, double *score, unsigned char *keep, int *picks, double *gap)
{
    const long c = t / bs;
    for (long blk = 0; blk <= c; ++blk) keep[blk] = (blk == 0 || blk == c);
    /* scores of the candidate blocks 1 .. c-1 (whole blocks, all j < c*bs <= t) */
    for (long blk = 1; blk < c; ++blk) {
        double sc = 0.0;
        for (int ch = 0; ch < d; ++ch) {
            double lo = INFINITY, hi = -INFINITY, sum = 0.0;
            for (long j = blk * bs; j < (blk + 1) * bs; ++j) {
                const double x = kt[idx4(T, H, d, b, j, h, ch)];
                if (x < lo) lo = x;
                if (x > hi) hi = x;
                sum += x;
            }
            if (mode == 0) {
                const double a1 = qrow[ch] * lo, a2 = qrow[ch] * hi;
                sc += a1 > a2 ? a1 : a2;
            } else {
                sc += qrow[ch] * (sum / (double)bs);
            }
        }
        score[blk] = sc;
    }
    /* the K best candidates, ties to the lower index */
    double last = INFINITY;
    for (int pick = 0; pick < K; ++pick) {
        long best = -1;
        for (long blk = 1; blk < c; ++blk)
            if (!keep[blk] && (best < 0 || score[blk] > score[best])) best = blk;
        if (picks) picks[pick] = (int)best;
        if (best < 0) continue;
        keep[best] = 1;
        last = score[best];
    }
    if (gap) {
        double rest = -INFINITY;
        for (long blk = 1; blk < c; ++blk)
            if (!keep[blk] && score[blk] > rest) rest = score[blk];
        *gap = (rest == -INFINITY || last == INFINITY) ? INFINITY : last - rest;
    }
}

/* Rows of top-k block attention.  Returns 0, or -1 on an argument error. */
int oracle_attn_rows_topk(int B, int T, int H, int d, const double *q, const double *kt,
                          const double *vt, int bs, int K, int mode, double scale, long nrows,
                          const int64_t *rows, double *o, double *lse)
{
    if (bs < 1 || K < 0 || (mode != 0 && mode != 1)) return -1;
    for (long r = 0; r < nrows; ++r) {
        int64_t b = rows[3 * r], h = rows[3 * r + 1], t = rows[3 * r + 2];
        if (b < 0 || b >= B || h < 0 || h >= H || t < 0 || t >= T) return -1;
    }
    const long nblk = (T + bs - 1) / bs;
    int err = 0;
#pragma omp parallel
    {
        long *js = (long *)malloc(sizeof(long) * (size_t)(T > 0 ? T : 1));
        double *z = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
        double *score = (double *)malloc(sizeof(double) * (size_t)(nblk > 0 ? nblk : 1));
        unsigned char *keep = (unsigned char *)malloc((size_t)(nblk > 0 ? nblk : 1));
        if (!js || !z || !score || !keep) {
#pragma omp atomic write
            err = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (long r = 0; r < nrows; ++r) {
            if (err) continue;
            int b = (int)rows[3 * r], h = (int)rows[3 * r + 1];
            long t = (long)rows[3 * r + 2];
            const double *qrow = q + idx4(T, H, d, b, t, h, 0);
            topk_pick(T, H, d, qrow, kt, b, h, t, bs, K, mode, score, keep, NULL, NULL);
            long n = 0;
            for (long j = 0; j <= t; ++j)
                if (keep[j / bs]) js[n++] = j;
            softmax_over(T, H, d, qrow, kt, vt, b, h, js, n, scale, o + (size_t)r * (size_t)d, &lse[r], z);
        }
        free(js); free(z); free(score); free(keep);
    }
    return err ? -1 : 0;
}

/* The R9 selection itself for each row: sel (nrows x K, in pick order, -1
 * padded) and gap (nrows), as topk_pick defines them.  Returns 0 or -1. */
int oracle_topk_select(int B, int T, int H, int d, const double *q, const double *kt, int bs, int K,
                       int mode, long nrows, const int64_t *rows, int *sel, double *gap)
{
    if (bs < 1 || K < 0 || (mode != 0 && mode != 1)) return -1;
    for (long r = 0; r < nrows; ++r) {
        int64_t b = rows[3 * r], h = rows[3 * r + 1], t = rows[3 * r + 2];
        if (b < 0 || b >= B || h < 0 || h >= H || t < 0 || t >= T) return -1;
    }
    const long nblk = (T + bs - 1) / bs;
    int err = 0;
#pragma omp parallel
    {
        double *score = (double *)malloc(sizeof(double) * (size_t)(nblk > 0 ? nblk : 1));
        unsigned char *keep = (unsigned char *)malloc((size_t)(nblk > 0 ? nblk : 1));
        if (!score || !keep) {
#pragma omp atomic write
            err = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (long r = 0; r < nrows; ++r) {
            if (err) continue;
            int b = (int)rows[3 * r], h = (int)rows[3 * r + 1];
            long t = (long)rows[3 * r + 2];
            topk_pick(T, H, d, q + idx4(T, H, d, b, t, h, 0), kt, b, h, t, bs, K, mode, score, keep,
                      sel + (size_t)r * (size_t)K, &gap[r]);
        }
        free(score); free(keep);
    }
    return err ? -1 : 0;
}

/*
 * One decode step ([RAT+] Figure 2: "a simple step update" for the recurrence,
 * then attention of the new query over the cached augmented keys/values).
 * For every batch entry b the new token sits at position t = pos[b]:
 *   1. R1 one step: s <- a*s + (1-a)*x for x = k and x = v (a = 0 when
 *      recur_h = 0), with a = sigmoid(g);
 *   2. the new augmented key/value s is stored as row t of the history;
 *   3. the output is oracle_attn_rows' row (b, h, t) with parts = 3 over the
 *      history rows 0..t.
 *   q, k, v, g          : [B,H,d]   the new token
 *   state_k, state_v    : [B,H,d]   s_{t-1} in, s_t out
 *   hist_k, hist_v      : [B,cap,H,d] augmented keys/values in natural order;
 *                                      rows < pos[b] are read, row pos[b] written
 *   o, lse              : [B,H,d], [B,H]
 * Returns 0, or -1 on an argument error.
 */
int oracle_decode_step(int B, int H, int d, int cap, const int *pos, const double *q,
                       const double *k, const double *v, const double *g,
                       const int *dil, const int *win, const unsigned char *recur,
                       double scale, double *state_k, double *state_v, double *hist_k,
                       double *hist_v, double *o, double *lse)
{
    for (int b = 0; b < B; ++b)
        if (pos[b] < 0 || pos[b] >= cap) return -1;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
            for (int c = 0; c < d; ++c) {
                size_t e = ((size_t)b * H + h) * d + c;
                double a = (recur == NULL || recur[h]) ? sigmoid(g[e]) : 0.0;
                state_k[e] = a * state_k[e] + (1.0 - a) * k[e];
                state_v[e] = a * state_v[e] + (1.0 - a) * v[e];
                hist_k[idx4(cap, H, d, b, pos[b], h, c)] = state_k[e];
                hist_v[idx4(cap, H, d, b, pos[b], h, c)] = state_v[e];
            }
    /* the query of the new token laid out as row pos[b] of a [B,cap,H,d] tensor */
    double *qfull = (double *)calloc((size_t)B * cap * H * d, sizeof(double));
    int64_t *rows = (int64_t *)malloc(sizeof(int64_t) * 3 * (size_t)B * H);
    if (!qfull || !rows) { free(qfull); free(rows); return -1; }
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            for (int c = 0; c < d; ++c)
                qfull[idx4(cap, H, d, b, pos[b], h, c)] = q[((size_t)b * H + h) * d + c];
            int64_t *rw = rows + 3 * ((size_t)b * H + h);
            rw[0] = b; rw[1] = h; rw[2] = pos[b];
        }
    int rc = oracle_attn_rows(B, cap, H, d, qfull, hist_k, hist_v, dil, win, scale, 3,
                              (long)B * H, rows, o, lse);
    free(qfull);
    free(rows);
    return rc;
}
