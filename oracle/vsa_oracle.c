/*
 * vsa_oracle.c -- plain fp64 CPU oracle for spatial-temporal block-sparse attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg may load or call this library.  It shares no code, header, table or
 * helper with the CUDA path: every rule below is written out again here from its
 * definition, in the most direct form, with no blocking, fusion or reordering.
 *
 * Sources (web pages on sparse attention for video diffusion transformers):
 *   [SVG]  "Sparse Video-Gen: Accelerating Video Diffusion Transformers with
 *          Spatial-Temporal Sparsity" (summary page), section "Approach": heads are
 *          spatial (block-wise attention inside a frame) or temporal (same position
 *          across frames); a profiling pass over about 1% of the query rows picks the
 *          pattern with the lower error per head; temporal heads are re-laid out from
 *          token-major to frame-major order so that their blocks are contiguous.
 *          Table "Measured effects": sparsity values 0.13 / 0.18 / 0.35 (kept fraction),
 *          profiling fraction 1%.
 *   [USV]  "USV: Unified Sparsification for Accelerating Video Diffusion Models",
 *          Figure 2 caption: Q/K/V are split into local 3D cubes; long-range cubes are
 *          chosen by top-k on coarse (pooled) attention.
 *   [OSP]  "OSP-Next: ..." section "Method": the sparse attention stays compatible with
 *          FlashAttention kernels, i.e. it is ordinary softmax(QK^T * scale) V restricted
 *          to the kept keys.
 *
 * Readings where the pages give no formula:
 *   - attention is softmax(q.k / sqrt(d)) over the allowed keys, times V;
 *   - a head's layout maps token t = f*S + s (S = Hl*Wl) to a slot: identity for spatial
 *     heads, s*F + f for temporal heads (frame-major), and for cube heads
 *     cube*V + in-cube offset with cubes ordered row-major over (F/cf, Hl/ch, Wl/cw) and
 *     V = cf*ch*cw slots per cube (partial edge cubes keep their padded slots);
 *   - block of a token = slot / block;  block i of a spatial head covers frames
 *     [a_i, b_i], of a temporal head positions [a_i, b_i]; blocks i, j are kept when
 *     those intervals are at most w apart (the block-level cover of |f_q - f_k| <= w_s,
 *     respectively |s_q - s_k| <= w_t);
 *   - the window is the smallest w whose kept-block fraction reaches the target;
 *   - cube selection: fp64 mean of Q and K over each cube's real tokens, score
 *     qbar_c . kbar_c' (a plain fp64 dot product), keep the top k per row (score
 *     descending, ties to the smaller index) together with the cube itself;
 *   - profiling rows rho_i = floor((2i+1) N / (2r)), r = ceil(frac * N); error = mean
 *     squared difference to dense attention on those rows under the block masks that
 *     would be executed; ties go to the spatial pattern;
 *   - a row with no allowed key has output 0 and log-sum-exp -inf.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC -ffp-contract=off (no -ffast-math, no fused
 * multiply-adds: every product and sum is rounded on its own, as written).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_SPATIAL 0
#define OR_TEMPORAL 1
#define OR_CUBE 2

static int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

/* Number of cubes of a grid: ceil(F/cf) * ceil(Hl/ch) * ceil(Wl/cw). */
int64_t or_num_cubes(int64_t F, int64_t Hl, int64_t Wl, int64_t cf, int64_t ch, int64_t cw)
{
    return ceil_div(F, cf) * ceil_div(Hl, ch) * ceil_div(Wl, cw);
}

/* Rows of a head's buffer in its layout: N for spatial/temporal, cubes * cube volume for cube. */
int64_t or_layout_rows(int kind, int64_t F, int64_t Hl, int64_t Wl, int64_t cf, int64_t ch, int64_t cw)
{
    if (kind == OR_CUBE) return or_num_cubes(F, Hl, Wl, cf, ch, cw) * cf * ch * cw;
    return F * Hl * Wl;
}

/*
 * Slot of every natural token under the layout of `kind` ([SVG] Approach: token-major to
 * frame-major transformation; [USV] Figure 2: local 3D cubes).
 */
void or_layout_slots(int kind, int64_t F, int64_t Hl, int64_t Wl, int64_t cf, int64_t ch, int64_t cw,
                     int64_t *slot)
{
    int64_t S = Hl * Wl, N = F * S;
    int64_t nch = ceil_div(Hl, ch), ncw = ceil_div(Wl, cw), vol = cf * ch * cw;
    for (int64_t t = 0; t < N; ++t) {
        int64_t f = t / S, s = t % S, h = s / Wl, w = s % Wl;
        if (kind == OR_SPATIAL) {
            slot[t] = t;
        } else if (kind == OR_TEMPORAL) {
            slot[t] = s * F + f;
        } else {
            int64_t c = ((f / cf) * nch + h / ch) * ncw + w / cw;
            int64_t r = ((f % cf) * ch + h % ch) * cw + w % cw;
            slot[t] = c * vol + r;
        }
    }
}

/*
 * Pattern block mask for a spatial (group G = S tokens per frame, natural order) or
 * temporal (group G = F slots per position, frame-major order) head.  keep[i*nblk + j].
 * Block i spans slots [i*B, min(N,(i+1)*B) - 1]; its group interval is [a_i, b_i]
 * with a = first slot / G and b = last slot / G.
 */
void or_pattern_keep(int kind, int64_t F, int64_t Hl, int64_t Wl, int64_t block, int64_t w, uint8_t *keep)
{
    int64_t N = F * Hl * Wl;
    int64_t G = (kind == OR_SPATIAL) ? Hl * Wl : F;
    int64_t nb = ceil_div(N, block);
    for (int64_t i = 0; i < nb; ++i) {
        int64_t ai = (i * block) / G;
        int64_t bi = ((i + 1) * block < N ? (i + 1) * block - 1 : N - 1) / G;
        for (int64_t j = 0; j < nb; ++j) {
            int64_t aj = (j * block) / G;
            int64_t bj = ((j + 1) * block < N ? (j + 1) * block - 1 : N - 1) / G;
            int64_t gap = 0;
            if (aj - bi > gap) gap = aj - bi;
            if (ai - bj > gap) gap = ai - bj;
            keep[i * nb + j] = (uint8_t)(gap <= w);
        }
    }
}

/* Fraction of kept block pairs of the pattern mask with window w. */
double or_kept_fraction(int kind, int64_t F, int64_t Hl, int64_t Wl, int64_t block, int64_t w)
{
    int64_t N = F * Hl * Wl, nb = ceil_div(N, block);
    uint8_t *keep = (uint8_t *)malloc((size_t)(nb * nb));
    if (!keep) return -1.0;
    or_pattern_keep(kind, F, Hl, Wl, block, w, keep);
    int64_t cnt = 0;
    for (int64_t x = 0; x < nb * nb; ++x) cnt += keep[x];
    free(keep);
    return (double)cnt / (double)(nb * nb);
}

/*
 * Smallest window w >= 0 whose kept fraction reaches `target` ([SVG] table: the sparsity
 * values are kept fractions; reading: window = smallest one reaching the fraction).
 * Linear scan; returns the largest useful window when the target is above every fraction.
 */
int64_t or_window_for_target(int kind, int64_t F, int64_t Hl, int64_t Wl, int64_t block, double target)
{
    int64_t wmax = (kind == OR_SPATIAL) ? F - 1 : Hl * Wl - 1;
    for (int64_t w = 0; w <= wmax; ++w)
        if (or_kept_fraction(kind, F, Hl, Wl, block, w) >= target) return w;
    return wmax;
}

/*
 * Cube top-k mask ([USV] Figure 2: top-k cube selection from pooled attention).
 * q, k: natural [N, d] fp64 of one head.  keep[c*C + c'].  score (optional) [C*C].
 */
int or_cube_topk_keep(const double *q, const double *k, int64_t F, int64_t Hl, int64_t Wl, int64_t d,
                      int64_t cf, int64_t ch, int64_t cw, int64_t topk, uint8_t *keep, double *score_out)
{
    int64_t N = F * Hl * Wl, C = or_num_cubes(F, Hl, Wl, cf, ch, cw), vol = cf * ch * cw;
    int64_t *slot = (int64_t *)malloc(sizeof(int64_t) * (size_t)N);
    double *qbar = (double *)calloc((size_t)(C * d), sizeof(double));
    double *kbar = (double *)calloc((size_t)(C * d), sizeof(double));
    int64_t *count = (int64_t *)calloc((size_t)C, sizeof(int64_t));
    double *score = score_out ? score_out : (double *)malloc(sizeof(double) * (size_t)(C * C));
    if (!slot || !qbar || !kbar || !count || !score) return -1;
    or_layout_slots(OR_CUBE, F, Hl, Wl, cf, ch, cw, slot);
    /* pooled means over each cube's real tokens */
    for (int64_t t = 0; t < N; ++t) {
        int64_t c = slot[t] / vol;
        count[c] += 1;
        for (int64_t x = 0; x < d; ++x) {
            qbar[c * d + x] += q[t * d + x];
            kbar[c * d + x] += k[t * d + x];
        }
    }
    for (int64_t c = 0; c < C; ++c)
        for (int64_t x = 0; x < d; ++x) {
            qbar[c * d + x] /= (double)count[c];
            kbar[c * d + x] /= (double)count[c];
        }
    /* coarse scores: plain fp64 dot products */
#pragma omp parallel for schedule(static)
    for (int64_t c = 0; c < C; ++c)
        for (int64_t c2 = 0; c2 < C; ++c2) {
            double acc = 0.0;
            for (int64_t x = 0; x < d; ++x) acc += qbar[c * d + x] * kbar[c2 * d + x];
            score[c * C + c2] = acc;
        }
    /* per row: pick the best remaining column topk times (selection by repeated max) */
#pragma omp parallel for schedule(static)
    for (int64_t c = 0; c < C; ++c) {
        uint8_t *row = keep + c * C;
        memset(row, 0, (size_t)C);
        int64_t picks = topk < C ? topk : C;
        for (int64_t p = 0; p < picks; ++p) {
            int64_t best = -1;
            for (int64_t c2 = 0; c2 < C; ++c2) {
                if (row[c2]) continue;
                if (best < 0 || score[c * C + c2] > score[c * C + best]) best = c2;
            }
            row[best] = 1;
        }
        row[c] = 1;
    }
    free(slot); free(qbar); free(kbar); free(count);
    if (!score_out) free(score);
    return 0;
}

/*
 * Masked softmax attention on selected query rows ([OSP] Method: FlashAttention-compatible
 * sparse attention; [SVG] Approach: block-wise masks).  Everything in natural token order:
 * key u is allowed for query t when keep[qblock(t) * nblk + block(u)] is set, with
 * qblock(t) = qslot[t] / block under the queries' layout and block(u) = slot[u] / block
 * under the keys' layout (the same map except for the semantic permutation, which orders
 * queries and keys by their own clusters).  q, k, v: [N, d] fp64.  out: [nrows, d];
 * lse: [nrows] (natural log), or NULL.
 */
void or_attention_rows_qk(const double *q, const double *k, const double *v, int64_t N, int64_t d, double scale,
                          const int64_t *qslot, const int64_t *slot, int64_t block, const uint8_t *keep,
                          int64_t nblk, const int64_t *rows, int64_t nrows, double *out, double *lse)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t t = rows[r];
        int64_t bi = qslot[t] / block;
        const double *qt = q + t * d;
        double *o = out + r * d;
        double m = -INFINITY;
        for (int64_t u = 0; u < N; ++u) {
            if (!keep[bi * nblk + slot[u] / block]) continue;
            double s = 0.0;
            for (int64_t x = 0; x < d; ++x) s += qt[x] * k[u * d + x];
            s *= scale;
            if (s > m) m = s;
        }
        for (int64_t x = 0; x < d; ++x) o[x] = 0.0;
        if (m == -INFINITY) {
            if (lse) lse[r] = -INFINITY;
            continue;
        }
        double sum = 0.0;
        for (int64_t u = 0; u < N; ++u) {
            if (!keep[bi * nblk + slot[u] / block]) continue;
            double s = 0.0;
            for (int64_t x = 0; x < d; ++x) s += qt[x] * k[u * d + x];
            double p = exp(s * scale - m);
            sum += p;
            for (int64_t x = 0; x < d; ++x) o[x] += p * v[u * d + x];
        }
        for (int64_t x = 0; x < d; ++x) o[x] /= sum;
        if (lse) lse[r] = m + log(sum);
    }
}

/* The same with one layout for queries and keys (every head kind of [SVG] and [USV]). */
void or_attention_rows(const double *q, const double *k, const double *v, int64_t N, int64_t d, double scale,
                       const int64_t *slot, int64_t block, const uint8_t *keep, int64_t nblk,
                       const int64_t *rows, int64_t nrows, double *out, double *lse)
{
    or_attention_rows_qk(q, k, v, N, d, scale, slot, slot, block, keep, nblk, rows, nrows, out, lse);
}

/* Number of profiling rows: ceil(frac * N), clamped to [1, N]. */
int64_t or_profile_rows(int64_t N, double frac)
{
    int64_t r = (int64_t)ceil(frac * (double)N);
    if (r < 1) r = 1;
    if (r > N) r = N;
    return r;
}

/*
 * Online profiling of one head ([SVG] Approach and "Measured effects" rows on the
 * profiling fraction).  Writes mse[0] (spatial), mse[1] (temporal) and returns the
 * chosen kind (argmin, ties to spatial).  rows_out (optional, [r]) receives the rows.
 */
int or_profile_head(const double *q, const double *k, const double *v, int64_t F, int64_t Hl, int64_t Wl,
                    int64_t d, double scale, int64_t block, int64_t w_s, int64_t w_t, double frac,
                    double *mse, int64_t *rows_out)
{
    int64_t N = F * Hl * Wl, nb = ceil_div(N, block);
    int64_t r = or_profile_rows(N, frac);
    int64_t *rows = (int64_t *)malloc(sizeof(int64_t) * (size_t)r);
    int64_t *slot_id = (int64_t *)malloc(sizeof(int64_t) * (size_t)N);
    int64_t *slot_tp = (int64_t *)malloc(sizeof(int64_t) * (size_t)N);
    uint8_t *all = (uint8_t *)malloc((size_t)(nb * nb));
    uint8_t *ks = (uint8_t *)malloc((size_t)(nb * nb));
    uint8_t *kt = (uint8_t *)malloc((size_t)(nb * nb));
    double *od = (double *)malloc(sizeof(double) * (size_t)(r * d));
    double *osp = (double *)malloc(sizeof(double) * (size_t)(r * d));
    double *otp = (double *)malloc(sizeof(double) * (size_t)(r * d));
    if (!rows || !slot_id || !slot_tp || !all || !ks || !kt || !od || !osp || !otp) return -1;
    for (int64_t i = 0; i < r; ++i) rows[i] = ((2 * i + 1) * N) / (2 * r);
    if (rows_out) memcpy(rows_out, rows, sizeof(int64_t) * (size_t)r);
    or_layout_slots(OR_SPATIAL, F, Hl, Wl, 1, 1, 1, slot_id);
    or_layout_slots(OR_TEMPORAL, F, Hl, Wl, 1, 1, 1, slot_tp);
    memset(all, 1, (size_t)(nb * nb));
    or_pattern_keep(OR_SPATIAL, F, Hl, Wl, block, w_s, ks);
    or_pattern_keep(OR_TEMPORAL, F, Hl, Wl, block, w_t, kt);
    or_attention_rows(q, k, v, N, d, scale, slot_id, block, all, nb, rows, r, od, NULL);
    or_attention_rows(q, k, v, N, d, scale, slot_id, block, ks, nb, rows, r, osp, NULL);
    or_attention_rows(q, k, v, N, d, scale, slot_tp, block, kt, nb, rows, r, otp, NULL);
    double es = 0.0, et = 0.0;
    for (int64_t x = 0; x < r * d; ++x) {
        es += (osp[x] - od[x]) * (osp[x] - od[x]);
        et += (otp[x] - od[x]) * (otp[x] - od[x]);
    }
    mse[0] = es / (double)(r * d);
    mse[1] = et / (double)(r * d);
    free(rows); free(slot_id); free(slot_tp); free(all); free(ks); free(kt);
    free(od); free(osp); free(otp);
    return mse[1] < mse[0] ? OR_TEMPORAL : OR_SPATIAL;
}

/* ---------------------------------------------------------------------------------------
 * Semantic-aware permutation ([SVG2] "Sparse VideoGen2: ... Semantic-Aware Permutation",
 * abstract): tokens are clustered by k-means on their Q (respectively K) vectors,
 * reordered so that each cluster is contiguous, and a top-p budget over the clusters
 * picks the critical key clusters of each query cluster.  The page gives no formulas;
 * the readings used here:
 *   - Lloyd's k-means per head, separately on Q and on K, `iters` rounds of assignment then
 *     update; initial centroids are the rows rho_j = floor((2j+1) N / (2C));
 *   - assignment: each row goes to the centroid at the smallest squared Euclidean
 *     distance sum_x (x - c_j)^2, computed in fp64; exact ties to the smaller j;
 *   - update: a centroid is the mean of its members, computed in fp64 and stored in fp32
 *     (centroids are fp32 vectors); an empty cluster keeps its centroid;
 *   - cluster-major order: slots sorted by (cluster, token);
 *   - criticality of key cluster j for query cluster i: n_j exp(s_ij - max_j s_ij) with
 *     s_ij = scale * cq_i . ck_j (fp64); the kept clusters are the shortest prefix of the
 *     list sorted by weight (descending, ties to the smaller j) whose running sum reaches
 *     top_p times the sum of the whole list;
 *   - block pair (a, b) of the two cluster-major layouts is kept when some query slot of
 *     block a and some key slot of block b belong to a kept cluster pair.
 * ------------------------------------------------------------------------------------- */

/* Squared Euclidean distance of two fp32 vectors, in fp64. */
static double dist2(const float *a, const float *b, int64_t d)
{
    double acc = 0.0;
    for (int64_t x = 0; x < d; ++x) {
        double t = (double)a[x] - (double)b[x];
        acc += t * t;
    }
    return acc;
}

/*
 * Assignment step: label[t] = the nearest of the C centroids cent [C, d] to row t of x [N, d]
 * (fp64 squared distance, ties to the smaller index).  gap (optional, [N]) receives the
 * distance of the second-nearest centroid minus that of the nearest (0 for C = 1 or a tie).
 */
void or_kmeans_assign(const float *x, int64_t N, int64_t d, const float *cent, int64_t C, int32_t *label,
                      double *gap)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < N; ++t) {
        int64_t best = 0;
        double bd = INFINITY, second = INFINITY;
        for (int64_t j = 0; j < C; ++j) {
            double dj = dist2(x + t * d, cent + j * d, d);
            if (dj < bd) { second = bd; bd = dj; best = j; }
            else if (dj < second) second = dj;
        }
        label[t] = (int32_t)best;
        if (gap) gap[t] = C > 1 ? second - bd : 0.0;
    }
}

/*
 * Update step: cent[j] = fp32 of the fp64 mean of the rows labelled j; an empty cluster keeps
 * cent[j].  count [C] receives the member counts.  Returns 0, or -1 on allocation failure.
 */
int or_kmeans_update(const float *x, int64_t N, int64_t d, const int32_t *label, int64_t C, float *cent,
                     int32_t *count)
{
    double *sum = (double *)calloc((size_t)(C * d), sizeof(double));
    if (!sum) return -1;
    memset(count, 0, sizeof(int32_t) * (size_t)C);
    for (int64_t t = 0; t < N; ++t) {
        int64_t j = label[t];
        count[j] += 1;
        for (int64_t q = 0; q < d; ++q) sum[j * d + q] += (double)x[t * d + q];
    }
    for (int64_t j = 0; j < C; ++j)
        if (count[j] > 0)
            for (int64_t q = 0; q < d; ++q) cent[j * d + q] = (float)(sum[j * d + q] / (double)count[j]);
    free(sum);
    return 0;
}

/*
 * k-means of one head's rows x [N, d] (fp32 values) into C clusters with `iters` >= 1
 * rounds.  Outputs: cent [C, d] after the last update, label [N] from the last assignment,
 * count [C] of that assignment.  Returns 0, or -1 on a bad argument or allocation failure.
 */
int or_kmeans(const float *x, int64_t N, int64_t d, int64_t C, int64_t iters, float *cent, int32_t *label,
              int32_t *count)
{
    if (C < 1 || C > N || iters < 1) return -1;
    for (int64_t j = 0; j < C; ++j) {
        int64_t r = ((2 * j + 1) * N) / (2 * C);
        memcpy(cent + j * d, x + r * d, sizeof(float) * (size_t)d);
    }
    for (int64_t it = 0; it < iters; ++it) {
        or_kmeans_assign(x, N, d, cent, C, label, NULL);
        if (or_kmeans_update(x, N, d, label, C, cent, count) != 0) return -1;
    }
    return 0;
}

/* Cluster-major order: perm[slot] = token, slots sorted by (label, token).  offset [C + 1]. */
void or_cluster_perm(const int32_t *label, int64_t N, int64_t C, int32_t *perm, int32_t *offset)
{
    for (int64_t j = 0; j <= C; ++j) offset[j] = 0;
    for (int64_t t = 0; t < N; ++t) offset[label[t] + 1] += 1;
    for (int64_t j = 0; j < C; ++j) offset[j + 1] += offset[j];
    int32_t *next = (int32_t *)malloc(sizeof(int32_t) * (size_t)(C > 0 ? C : 1));
    if (!next) return;
    for (int64_t j = 0; j < C; ++j) next[j] = offset[j];
    for (int64_t t = 0; t < N; ++t) perm[next[label[t]]++] = (int32_t)t;
    free(next);
}

/*
 * Top-p key clusters of every query cluster.  keep[i * Ck + j]; a query cluster with no
 * member keeps nothing, an empty key cluster is never kept.  scale and p as described
 * above (0 < p <= 1).
 */
/*
 * Criticality weights of every key cluster for every query cluster: w[i * Ck + j] =
 * n_j exp(s_ij - max_j s_ij), s_ij = scale * cq_i . ck_j (fp64), over the non-empty key
 * clusters; -1 marks an empty key cluster (or every entry of an empty query cluster).
 */
void or_semantic_weights(const float *cq, const int32_t *nq, int64_t Cq, const float *ck, const int32_t *nk,
                         int64_t Ck, int64_t d, double scale, double *w)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < Cq; ++i) {
        double *row = w + i * Ck;
        double m = -INFINITY;
        for (int64_t j = 0; j < Ck; ++j) {
            row[j] = -1.0;
            if (nq[i] == 0 || nk[j] == 0) continue;
            double acc = 0.0;
            for (int64_t x = 0; x < d; ++x) acc += (double)cq[i * d + x] * (double)ck[j * d + x];
            row[j] = scale * acc;
            if (row[j] > m) m = row[j];
        }
        for (int64_t j = 0; j < Ck; ++j)
            if (nq[i] > 0 && nk[j] > 0) row[j] = (double)nk[j] * exp(row[j] - m);
    }
}

void or_semantic_keep(const float *cq, const int32_t *nq, int64_t Cq, const float *ck, const int32_t *nk,
                      int64_t Ck, int64_t d, double scale, double p, uint8_t *keep)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < Cq; ++i) {
        uint8_t *row = keep + i * Ck;
        memset(row, 0, (size_t)Ck);
        if (nq[i] == 0) continue;
        double *w = (double *)malloc(sizeof(double) * (size_t)Ck);
        uint8_t *used = (uint8_t *)calloc((size_t)Ck, 1);
        if (!w || !used) { free(w); free(used); continue; }
        double m = -INFINITY;
        for (int64_t j = 0; j < Ck; ++j) {
            if (nk[j] == 0) continue;
            double acc = 0.0;
            for (int64_t x = 0; x < d; ++x) acc += (double)cq[i * d + x] * (double)ck[j * d + x];
            w[j] = scale * acc;
            if (w[j] > m) m = w[j];
        }
        int64_t live = 0;
        for (int64_t j = 0; j < Ck; ++j)
            if (nk[j] > 0) { w[j] = (double)nk[j] * exp(w[j] - m); ++live; }
        /* the list sorted by weight, by repeated selection of the largest remaining entry */
        int64_t *order = (int64_t *)malloc(sizeof(int64_t) * (size_t)(live > 0 ? live : 1));
        if (!order) { free(w); free(used); continue; }
        for (int64_t pos = 0; pos < live; ++pos) {
            int64_t best = -1;
            for (int64_t j = 0; j < Ck; ++j) {
                if (nk[j] == 0 || used[j]) continue;
                if (best < 0 || w[j] > w[best]) best = j;
            }
            used[best] = 1;
            order[pos] = best;
        }
        double total = 0.0;
        for (int64_t pos = 0; pos < live; ++pos) total += w[order[pos]];
        double target = p * total, cum = 0.0;
        for (int64_t pos = 0; pos < live; ++pos) {
            row[order[pos]] = 1;
            cum += w[order[pos]];
            if (cum >= target) break;
        }
        free(order); free(w); free(used);
    }
}

/* ---------------------------------------------------------------------------------------
 * FP8 Q and K ("Sparse Video-Gen" summary page, "Measured effects": FP8 quantisation on top
 * of the sparse attention).  The page gives no format details; the readings used here:
 *   - e4m3 values (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; largest 448,
 *     subnormals down to 2^-9), round to nearest with ties to even;
 *   - one scale per block of `block` rows of a head's layout: the smallest power of two 2^e
 *     with max |x| <= 448 * 2^e over the block (e = 0 for an all-zero block); the stored code
 *     is e4m3(x / 2^e) and the value it stands for is e4m3(x / 2^e) * 2^e.
 * ------------------------------------------------------------------------------------- */

/* e4m3 code of y (|y| <= 448), rounded to the nearest value, ties to even. */
static uint8_t e4m3_code(double y)
{
    uint8_t sign = (y < 0.0 || (y == 0.0 && signbit(y))) ? 0x80 : 0x00;
    double a = fabs(y);
    if (a < ldexp(1.0, -6)) {                       /* subnormal range: spacing 2^-9 */
        double m = nearbyint(a / ldexp(1.0, -9));  /* 0..8; 8 is the smallest normal */
        if (m >= 8.0) return (uint8_t)(sign | (1 << 3));
        return (uint8_t)(sign | (int)m);
    }
    int E = (int)floor(log2(a));
    if (ldexp(1.0, E) > a) E -= 1;                  /* guard log2 rounding */
    if (ldexp(1.0, E + 1) <= a) E += 1;
    double m = nearbyint(a / ldexp(1.0, E - 3));    /* 8..16 */
    if (m >= 16.0) { m = 8.0; E += 1; }
    return (uint8_t)(sign | ((E + 7) << 3) | ((int)m - 8));
}

/* Value of an e4m3 code. */
double or_e4m3_value(uint8_t c)
{
    int e = (c >> 3) & 0xF, m = c & 7;
    double v = e == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return (c & 0x80) ? -v : v;
}

/*
 * Quantise one head's rows x [rows, d] in blocks of `block` rows: code [rows, d] (e4m3) and
 * scale_exp [ceil(rows / block)] (the block's power-of-two exponent e).
 */
void or_quantize_e4m3(const double *x, int64_t rows, int64_t d, int64_t block, uint8_t *code, int32_t *scale_exp)
{
    int64_t nb = ceil_div(rows, block);
    for (int64_t b = 0; b < nb; ++b) {
        int64_t r0 = b * block, r1 = (b + 1) * block < rows ? (b + 1) * block : rows;
        double amax = 0.0;
        for (int64_t i = r0 * d; i < r1 * d; ++i)
            if (fabs(x[i]) > amax) amax = fabs(x[i]);
        int e = 0;
        if (amax > 0.0) {
            e = (int)ceil(log2(amax / 448.0)) - 1;
            while (amax > 448.0 * ldexp(1.0, e)) ++e;     /* smallest e with amax <= 448 * 2^e */
            while (amax <= 448.0 * ldexp(1.0, e - 1)) --e;
        }
        scale_exp[b] = e;
        for (int64_t i = r0 * d; i < r1 * d; ++i) code[i] = e4m3_code(ldexp(x[i], -e));
    }
}
