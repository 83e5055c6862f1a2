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
 * Readings where the pages give no formula (each is listed with its reason in the
 * design notes of the repository):
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
 *   - cube selection: fp64 mean of Q and K over each cube's real tokens (summed in token
 *     order), score qbar_c . kbar_c' (summed in dimension order, one fused multiply-add
 *     per term), keep the top k per row (score descending, ties to the smaller index)
 *     together with the cube itself;
 *   - profiling rows rho_i = floor((2i+1) N / (2r)), r = ceil(frac * N); error = mean
 *     squared difference to dense attention on those rows under the block masks that
 *     would be executed; ties go to the spatial pattern;
 *   - a row with no allowed key has output 0 and log-sum-exp -inf.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC -ffp-contract=off (no -ffast-math; the only fused
 * multiply-adds are the explicit fma() calls of the coarse scores).
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
    /* coarse scores: fp64 dot products in dimension order, one fused multiply-add per term */
#pragma omp parallel for schedule(static)
    for (int64_t c = 0; c < C; ++c)
        for (int64_t c2 = 0; c2 < C; ++c2) {
            double acc = 0.0;
            for (int64_t x = 0; x < d; ++x) acc = fma(qbar[c * d + x], kbar[c2 * d + x], acc);
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
 * key u is allowed for query t when keep[block(t) * nblk + block(u)] is set, with
 * block(x) = slot[x] / block.  q, k, v: [N, d] fp64.  out: [nrows, d]; lse: [nrows]
 * (natural log), or NULL.
 */
void or_attention_rows(const double *q, const double *k, const double *v, int64_t N, int64_t d, double scale,
                       const int64_t *slot, int64_t block, const uint8_t *keep, int64_t nblk,
                       const int64_t *rows, int64_t nrows, double *out, double *lse)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t t = rows[r];
        int64_t bi = slot[t] / block;
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
