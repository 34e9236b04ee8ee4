/*
 * nabla_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, explicit-loop CPU restatement of NABLA block-sparse attention,
 * written from "NABLA: Neighborhood Adaptive Block-Level Attention" (the
 * technical summary, section "手法: NABLA").  It exists so that the CUDA path
 * can be checked against something written independently of it.  Only the test
 * suite, the smoke check and the benchmark's CPU-baseline leg may load it; the
 * product library never links, calls or falls back to it, and it shares no
 * code, header, table or helper with the CUDA sources.
 *
 * Two precisions live here, on purpose:
 *
 *  - the plain definition in float64 (oracle_pool_f64, oracle_mask_f64,
 *    oracle_attn_fwd, oracle_attn_bwd): every step as the page states it, with
 *    no blocking or reordering;
 *
 *  - the decision path in the precision the GPU kernels take the mask decision
 *    in (oracle_pool_f32, oracle_mask): block means summed in float32 in
 *    ascending token order, block scores as a float32 fused multiply-add chain
 *    in ascending feature order, weights exp() in float64 from those float32
 *    scores, and the cumulative mass in exact 2^-40 fixed point.  A floating
 *    point comparison decides an integer set here, so both sides take that
 *    decision in the same precision.  Tests pin this path to the float64
 *    definition on every row whose decision is not within rounding of the cut.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -mfma -shared -fPIC (no fast-math:
 * the float32 sums must run strictly in the order written).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* scalar helpers                                                            */
/* ------------------------------------------------------------------------ */

static float bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* ------------------------------------------------------------------------ */
/* Fractal flattening (section "トークン再順序付け (Fractal Flattening)").     */
/* Tokens of each P x P spatial patch become contiguous; frames keep their   */
/* order.  One level of patches, patch grid row-major, row-major inside the  */
/* patch.                                                                     */
/* ------------------------------------------------------------------------ */

int64_t oracle_flat_index(int t, int y, int x, int T, int H, int W, int P)
{
    (void)T;
    int64_t Hp = H / P, Wp = W / P;
    int64_t patch = ((int64_t)t * Hp + y / P) * Wp + x / P;
    return patch * (int64_t)P * P + (int64_t)(y % P) * P + (x % P);
}

/* in/out viewed as [outer, T, H, W, inner_bytes] (grid order) and
 * [outer, N, inner_bytes] (flattened order).  inverse=0: grid -> flat. */
void oracle_flatten(const uint8_t *in, uint8_t *out, int64_t outer, int T, int H,
                    int W, int P, int64_t inner_bytes, int inverse)
{
    int64_t N = (int64_t)T * H * W;
    for (int64_t o = 0; o < outer; ++o)
        for (int t = 0; t < T; ++t)
            for (int y = 0; y < H; ++y)
                for (int x = 0; x < W; ++x) {
                    int64_t n_grid = ((int64_t)t * H + y) * W + x;
                    int64_t n_flat = oracle_flat_index(t, y, x, T, H, W, P);
                    int64_t src = inverse ? n_flat : n_grid;
                    int64_t dst = inverse ? n_grid : n_flat;
                    memcpy(out + (o * N + dst) * inner_bytes,
                           in + (o * N + src) * inner_bytes, (size_t)inner_bytes);
                }
}

/* ------------------------------------------------------------------------ */
/* Block mean-pooling of Q and K (section "適応型マスク構築", bullet           */
/* "ダウンサンプリング").  Block i = flattened tokens [i*L, (i+1)*L), L = P*P. */
/* x: [BH, N, D] bf16 bits, flattened order.                                  */
/* ------------------------------------------------------------------------ */

/* float64 definition: arithmetic mean of the L rows. */
void oracle_pool_f64(const uint16_t *x, double *xbar, int64_t BH, int64_t N, int D, int L)
{
    int64_t nb = N / L;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t bh = 0; bh < BH; ++bh)
        for (int64_t i = 0; i < nb; ++i)
            for (int d = 0; d < D; ++d) {
                double acc = 0.0;
                for (int r = 0; r < L; ++r)
                    acc += (double)bf16_to_f32(x[((bh * N) + i * L + r) * D + d]);
                xbar[(bh * nb + i) * D + d] = acc / (double)L;
            }
}

/* Decision precision: float32 running sum in ascending token order, then
 * multiplied by 1/L (exact for L a power of two). */
void oracle_pool_f32(const uint16_t *x, float *xbar, int64_t BH, int64_t N, int D, int L)
{
    int64_t nb = N / L;
    float inv = 1.0f / (float)L;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t bh = 0; bh < BH; ++bh)
        for (int64_t i = 0; i < nb; ++i)
            for (int d = 0; d < D; ++d) {
                float acc = 0.0f;
                for (int r = 0; r < L; ++r)
                    acc = acc + bf16_to_f32(x[((bh * N) + i * L + r) * D + d]);
                xbar[(bh * nb + i) * D + d] = acc * inv;
            }
}

/* ------------------------------------------------------------------------ */
/* Sliding Tile Attention window (section "STA とのハイブリッド統合").        */
/* Blocks are tiles of one frame; block i <-> (t, ph, pw),                    */
/* i = (t*Hp + ph)*Wp + pw.  The window is truncated at the grid border.      */
/* ------------------------------------------------------------------------ */

#define ORACLE_NO_STA 1u
#define ORACLE_FULL_STA 2u

int oracle_sta(int64_t i, int64_t j, int Hp, int Wp, int wt, int wh, int ww, unsigned flags)
{
    if (flags & ORACLE_FULL_STA) return 1;
    if (flags & ORACLE_NO_STA) return 0;
    int64_t ti = i / ((int64_t)Hp * Wp), tj = j / ((int64_t)Hp * Wp);
    int64_t hi = (i / Wp) % Hp, hj = (j / Wp) % Hp;
    int64_t wi = i % Wp, wj = j % Wp;
    return llabs(ti - tj) <= wt / 2 && llabs(hi - hj) <= wh / 2 && llabs(wi - wj) <= ww / 2;
}

/* ------------------------------------------------------------------------ */
/* Reduced attention map + per-row CDF cut (bullets "縮小されたアテンション",   */
/* "CDF 閾値処理").  For each row the blocks are ranked by score, descending   */
/* (equal scores: lower block index first); the kept set is the shortest     */
/* prefix of that ranking whose cumulative probability reaches p.  p >= 1    */
/* keeps every block.  Keeping the blocks whose ascending cumulative mass     */
/* exceeds 1-p is the same set: the block of rank k is kept exactly when the */
/* mass strictly before it is < p.                                            */
/* ------------------------------------------------------------------------ */

typedef struct {
    double key; /* score; larger first */
    int64_t j;  /* block index; smaller first on equal key */
} rank_item;

static int rank_cmp(const void *a, const void *b)
{
    const rank_item *x = (const rank_item *)a, *y = (const rank_item *)b;
    if (x->key > y->key) return -1;
    if (x->key < y->key) return 1;
    return (x->j < y->j) ? -1 : (x->j > y->j);
}

/* Writes the full mask M = adaptive OR STA OR diagonal for every row:
 *   bits    [BH, nb, ceil(nb/32)] (bit j%32 of word j/32)
 *   row_idx [BH, nb, nb] ascending j, row_cnt [BH, nb]
 *   col_idx [BH, nb, nb] ascending i, col_cnt [BH, nb]   (may be NULL)
 *   adapt_cnt [BH, nb] size of the adaptive set alone     (may be NULL)
 * The caller owns all buffers.  "keep" is the per-row adaptive indicator
 * produced by one of the two cut routines below. */
static void emit_mask(const uint8_t *keep_all, int64_t BH, int64_t nb, int Hp, int Wp,
                      int wt, int wh, int ww, unsigned flags, uint32_t *bits,
                      uint16_t *row_idx, int32_t *row_cnt, uint16_t *col_idx,
                      int32_t *col_cnt)
{
    int64_t words = (nb + 31) / 32;
#pragma omp parallel for schedule(static)
    for (int64_t bh = 0; bh < BH; ++bh) {
        for (int64_t i = 0; i < nb; ++i) {
            const uint8_t *keep = keep_all + (bh * nb + i) * nb;
            uint32_t *brow = bits ? bits + (bh * nb + i) * words : NULL;
            if (brow) memset(brow, 0, (size_t)words * 4);
            int32_t c = 0;
            for (int64_t j = 0; j < nb; ++j) {
                int m = keep[j] || oracle_sta(i, j, Hp, Wp, wt, wh, ww, flags) || (i == j);
                if (!m) continue;
                if (brow) brow[j / 32] |= 1u << (j % 32);
                if (row_idx) row_idx[(bh * nb + i) * nb + c] = (uint16_t)j;
                ++c;
            }
            if (row_cnt) row_cnt[bh * nb + i] = c;
        }
        if (col_idx || col_cnt) {
            for (int64_t j = 0; j < nb; ++j) {
                int32_t c = 0;
                for (int64_t i = 0; i < nb; ++i) {
                    const uint8_t *keep = keep_all + (bh * nb + i) * nb;
                    int m = keep[j] || oracle_sta(i, j, Hp, Wp, wt, wh, ww, flags) || (i == j);
                    if (!m) continue;
                    if (col_idx) col_idx[(bh * nb + j) * nb + c] = (uint16_t)i;
                    ++c;
                }
                if (col_cnt) col_cnt[bh * nb + j] = c;
            }
        }
    }
}

/* float64 definition of the cut on one row of probabilities prob[0..nb).
 * Returns the number kept; keep[] gets 0/1.  cum_before / cum_at receive the
 * cumulative mass before and including the last kept block (for band tests). */
static int64_t cut_row_f64(const double *score, int64_t nb, double p, uint8_t *keep,
                           rank_item *scratch, double *cum_before, double *cum_at)
{
    memset(keep, 0, (size_t)nb);
    if (p >= 1.0) {
        memset(keep, 1, (size_t)nb);
        if (cum_before) *cum_before = 1.0;
        if (cum_at) *cum_at = 1.0;
        return nb;
    }
    double smax = -INFINITY;
    for (int64_t j = 0; j < nb; ++j) smax = fmax(smax, score[j]);
    double z = 0.0;
    for (int64_t j = 0; j < nb; ++j) z += exp(score[j] - smax);
    for (int64_t j = 0; j < nb; ++j) {
        scratch[j].key = score[j];
        scratch[j].j = j;
    }
    qsort(scratch, (size_t)nb, sizeof(rank_item), rank_cmp);
    double c = 0.0, before = 0.0;
    int64_t k = 0;
    while (k < nb && c < p) {
        before = c;
        c += exp(scratch[k].key - smax) / z;
        keep[scratch[k].j] = 1;
        ++k;
    }
    if (cum_before) *cum_before = before;
    if (cum_at) *cum_at = c;
    return k;
}

/* Plain float64 mask: pooled means in float64, scores scale * <qbar_i, kbar_j>
 * summed in float64, softmax in float64, cut on the probabilities.
 * qbar/kbar: [BH, nb, D] float64.  Also reports, per row, the cumulative mass
 * before and at the last kept block (for the band rule). */
void oracle_mask_f64(const double *qbar, const double *kbar, int64_t BH, int64_t nb, int D,
                     int Hp, int Wp, double p, double scale, int wt, int wh, int ww,
                     unsigned flags, uint32_t *bits, uint16_t *row_idx, int32_t *row_cnt,
                     uint16_t *col_idx, int32_t *col_cnt, int32_t *adapt_cnt,
                     double *cum_before, double *cum_at)
{
    uint8_t *keep_all = (uint8_t *)malloc((size_t)(BH * nb * nb));
#pragma omp parallel
    {
        double *score = (double *)malloc(sizeof(double) * (size_t)nb);
        rank_item *scratch = (rank_item *)malloc(sizeof(rank_item) * (size_t)nb);
#pragma omp for collapse(2) schedule(dynamic, 16)
        for (int64_t bh = 0; bh < BH; ++bh)
            for (int64_t i = 0; i < nb; ++i) {
                const double *qi = qbar + (bh * nb + i) * D;
                for (int64_t j = 0; j < nb; ++j) {
                    const double *kj = kbar + (bh * nb + j) * D;
                    double s = 0.0;
                    for (int d = 0; d < D; ++d) s += qi[d] * kj[d];
                    score[j] = scale * s;
                }
                double cb, ca;
                int64_t k = cut_row_f64(score, nb, p, keep_all + (bh * nb + i) * nb, scratch,
                                        &cb, &ca);
                if (adapt_cnt) adapt_cnt[bh * nb + i] = (int32_t)k;
                if (cum_before) cum_before[bh * nb + i] = cb;
                if (cum_at) cum_at[bh * nb + i] = ca;
            }
        free(score);
        free(scratch);
    }
    emit_mask(keep_all, BH, nb, Hp, Wp, wt, wh, ww, flags, bits, row_idx, row_cnt, col_idx,
              col_cnt);
    free(keep_all);
}

/* The cut in decision precision, on one row of float32 scores.
 *   w_j = exp((double)s_j - (double)s_max)               (float64)
 *   u_j = floor(w_j * 2^40)                              (exact integer mass)
 *   U = sum u_j;  thr = (double)p * (double)U            (one rounding)
 * kept = shortest prefix of the ranking (s desc, j asc) with (double)C >= thr.
 * margin receives min(|C_before - thr|, |C_at - thr|) in units of 2^-40 of
 * the row's largest weight: how far the decision is from flipping. */
static int64_t cut_row_fixed(const float *score, int64_t nb, float p, uint8_t *keep,
                             rank_item *scratch, uint64_t *u, double *margin)
{
    memset(keep, 0, (size_t)nb);
    if (p >= 1.0f) {
        memset(keep, 1, (size_t)nb);
        if (margin) *margin = INFINITY;
        return nb;
    }
    if (p <= 0.0f) { /* the empty prefix already reaches 0: nothing to decide */
        if (margin) *margin = INFINITY;
        return 0;
    }
    float smax = -INFINITY;
    for (int64_t j = 0; j < nb; ++j) smax = fmaxf(smax, score[j]);
    uint64_t U = 0;
    for (int64_t j = 0; j < nb; ++j) {
        double w = exp((double)score[j] - (double)smax);
        u[j] = (uint64_t)ldexp(w, 40);
        U += u[j];
    }
    double thr = (double)p * (double)U;
    for (int64_t j = 0; j < nb; ++j) {
        scratch[j].key = (double)score[j];
        scratch[j].j = j;
    }
    qsort(scratch, (size_t)nb, sizeof(rank_item), rank_cmp);
    uint64_t c = 0, before = 0;
    int64_t k = 0;
    while (k < nb && (double)c < thr) {
        before = c;
        c += u[scratch[k].j];
        keep[scratch[k].j] = 1;
        ++k;
    }
    if (margin) {
        double m1 = fabs((double)before - thr), m2 = fabs((double)c - thr);
        *margin = k == 0 ? fabs((double)c - thr) : fmin(m1, m2);
    }
    return k;
}

/* Block scores of one query block in decision precision (bullet
 * "縮小されたアテンション": the attention map over the pooled blocks):
 *   s_j = (fmaf chain over d = 0..D-1 of qi[d] * kbar_j[d], starting from 0)
 *         * scale,
 * every operation in float32.  kbar_bh: [nb, D] float32 of the same head. */
static void scores_row_f32(const float *qi, const float *kbar_bh, int64_t nb, int D, float scale,
                           float *score)
{
    for (int64_t j = 0; j < nb; ++j) {
        const float *kj = kbar_bh + j * D;
        float s = 0.0f;
        for (int d = 0; d < D; ++d) s = fmaf(qi[d], kj[d], s);
        score[j] = s * scale;
    }
}

/* All block scores, qbar/kbar: [BH, nb, D] float32 -> scores [BH, nb, nb]. */
void oracle_scores_f32(const float *qbar, const float *kbar, int64_t BH, int64_t nb, int D,
                       float scale, float *scores)
{
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t bh = 0; bh < BH; ++bh)
        for (int64_t i = 0; i < nb; ++i)
            scores_row_f32(qbar + (bh * nb + i) * D, kbar + bh * nb * D, nb, D, scale,
                           scores + (bh * nb + i) * nb);
}

/* Mask in decision precision from given float32 score rows [BH, nb, nb]:
 * the cut of cut_row_fixed on each row, then OR with STA and the diagonal. */
void oracle_mask_from_scores(const float *scores, int64_t BH, int64_t nb, int Hp, int Wp,
                             float p, int wt, int wh, int ww, unsigned flags, uint32_t *bits,
                             uint16_t *row_idx, int32_t *row_cnt, uint16_t *col_idx,
                             int32_t *col_cnt, int32_t *adapt_cnt, double *margin)
{
    uint8_t *keep_all = (uint8_t *)malloc((size_t)(BH * nb * nb));
#pragma omp parallel
    {
        uint64_t *u = (uint64_t *)malloc(sizeof(uint64_t) * (size_t)nb);
        rank_item *scratch = (rank_item *)malloc(sizeof(rank_item) * (size_t)nb);
#pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < BH * nb; ++r) {
            double mg;
            int64_t k = cut_row_fixed(scores + r * nb, nb, p, keep_all + r * nb, scratch, u, &mg);
            if (adapt_cnt) adapt_cnt[r] = (int32_t)k;
            if (margin) margin[r] = mg;
        }
        free(u);
        free(scratch);
    }
    emit_mask(keep_all, BH, nb, Hp, Wp, wt, wh, ww, flags, bits, row_idx, row_cnt, col_idx,
              col_cnt);
    free(keep_all);
}

/* Mask in decision precision from float32 pooled means (oracle_pool_f32):
 * scores_row_f32 then cut_row_fixed on every row, then OR with STA and the
 * diagonal. */
void oracle_mask(const float *qbar, const float *kbar, int64_t BH, int64_t nb, int D, int Hp,
                 int Wp, float p, float scale, int wt, int wh, int ww, unsigned flags,
                 uint32_t *bits, uint16_t *row_idx, int32_t *row_cnt, uint16_t *col_idx,
                 int32_t *col_cnt, int32_t *adapt_cnt, double *margin)
{
    uint8_t *keep_all = (uint8_t *)malloc((size_t)(BH * nb * nb));
#pragma omp parallel
    {
        float *score = (float *)malloc(sizeof(float) * (size_t)nb);
        uint64_t *u = (uint64_t *)malloc(sizeof(uint64_t) * (size_t)nb);
        rank_item *scratch = (rank_item *)malloc(sizeof(rank_item) * (size_t)nb);
#pragma omp for collapse(2) schedule(dynamic, 16)
        for (int64_t bh = 0; bh < BH; ++bh)
            for (int64_t i = 0; i < nb; ++i) {
                scores_row_f32(qbar + (bh * nb + i) * D, kbar + bh * nb * D, nb, D, scale,
                               score);
                double mg;
                int64_t k = cut_row_fixed(score, nb, p, keep_all + (bh * nb + i) * nb, scratch,
                                          u, &mg);
                if (adapt_cnt) adapt_cnt[bh * nb + i] = (int32_t)k;
                if (margin) margin[bh * nb + i] = mg;
            }
        free(score);
        free(u);
        free(scratch);
    }
    emit_mask(keep_all, BH, nb, Hp, Wp, wt, wh, ww, flags, bits, row_idx, row_cnt, col_idx,
              col_cnt);
    free(keep_all);
}

/* ------------------------------------------------------------------------ */
/* DynamicRad-style masks ("DynamicRad: Content-Adaptive Sparse Attention     */
/* for Long Video Diffusion", section 2.A "Dual-Mode Strategy"), emitted in   */
/* the same format: selected OR STA OR diagonal.                              */
/* ------------------------------------------------------------------------ */

typedef struct {
    int64_t d; /* squared distance to the query's patch, in patch units */
    int64_t p; /* patch index in the frame; smaller first on equal d */
} patch_item;

static int patch_cmp(const void *a, const void *b)
{
    const patch_item *x = (const patch_item *)a, *y = (const patch_item *)b;
    if (x->d != y->d) return x->d < y->d ? -1 : 1;
    return (x->p < y->p) ? -1 : (x->p > y->p);
}

/* Static-Ratio mode (no content scoring; a fixed retention ratio by temporal
 * distance).  Query block i = (t_i, ph_i, pw_i) keeps, in frame t with
 * dt = |t - t_i|, the k(dt) = ceil(min(1, max(lambda, gamma^dt)) * Hp*Wp)
 * patches nearest to (ph_i, pw_i) (squared distance, then patch index);
 * gamma^dt is the product of dt factors gamma in double precision.
 * adapt_cnt (may be NULL) gets the number of selected blocks per row. */
void oracle_dr_static(int64_t BH, int64_t nb, int T, int Hp, int Wp, double gamma, double lambda,
                      int wt, int wh, int ww, unsigned flags, uint32_t *bits, uint16_t *row_idx,
                      int32_t *row_cnt, uint16_t *col_idx, int32_t *col_cnt, int32_t *adapt_cnt)
{
    int64_t HW = (int64_t)Hp * Wp;
    uint8_t *keep_all = (uint8_t *)calloc((size_t)(BH * nb * nb), 1);
#pragma omp parallel
    {
        patch_item *order = (patch_item *)malloc(sizeof(patch_item) * (size_t)HW);
#pragma omp for collapse(2) schedule(dynamic, 16)
        for (int64_t bh = 0; bh < BH; ++bh)
            for (int64_t i = 0; i < nb; ++i) {
                int64_t ti = i / HW, qh = (i % HW) / Wp, qw = i % Wp;
                uint8_t *keep = keep_all + (bh * nb + i) * nb;
                for (int64_t p = 0; p < HW; ++p) {
                    int64_t dh = p / Wp - qh, dw = p % Wp - qw;
                    order[p].d = dh * dh + dw * dw;
                    order[p].p = p;
                }
                qsort(order, (size_t)HW, sizeof(patch_item), patch_cmp);
                int32_t c = 0;
                for (int64_t t = 0; t < T; ++t) {
                    int64_t dt = t > ti ? t - ti : ti - t;
                    double g = 1.0;
                    for (int64_t n = 0; n < dt; ++n) g = g * gamma;
                    double r = fmin(1.0, fmax(lambda, g));
                    int64_t k = (int64_t)fmin(ceil(r * (double)HW), (double)HW);
                    for (int64_t m = 0; m < k; ++m) keep[t * HW + order[m].p] = 1;
                    c += (int32_t)k;
                }
                if (adapt_cnt) adapt_cnt[bh * nb + i] = c;
            }
        free(order);
    }
    emit_mask(keep_all, BH, nb, Hp, Wp, wt, wh, ww, flags, bits, row_idx, row_cnt, col_idx,
              col_cnt);
    free(keep_all);
}

/* Dynamic-Threshold mode (pre-softmax logits as the importance proxy): with
 * the decision-precision pooled scores s_ij (scores_row_f32), keep j where the
 * float32 difference max_j s_ij - s_ij is at most tau. */
void oracle_dr_threshold(const float *qbar, const float *kbar, int64_t BH, int64_t nb, int D,
                         int Hp, int Wp, float tau, float scale, int wt, int wh, int ww,
                         unsigned flags, uint32_t *bits, uint16_t *row_idx, int32_t *row_cnt,
                         uint16_t *col_idx, int32_t *col_cnt, int32_t *adapt_cnt)
{
    uint8_t *keep_all = (uint8_t *)calloc((size_t)(BH * nb * nb), 1);
#pragma omp parallel
    {
        float *score = (float *)malloc(sizeof(float) * (size_t)nb);
#pragma omp for collapse(2) schedule(dynamic, 16)
        for (int64_t bh = 0; bh < BH; ++bh)
            for (int64_t i = 0; i < nb; ++i) {
                scores_row_f32(qbar + (bh * nb + i) * D, kbar + bh * nb * D, nb, D, scale, score);
                float smax = -INFINITY;
                for (int64_t j = 0; j < nb; ++j) smax = fmaxf(smax, score[j]);
                uint8_t *keep = keep_all + (bh * nb + i) * nb;
                int32_t c = 0;
                for (int64_t j = 0; j < nb; ++j) {
                    float gap = smax - score[j];
                    if (gap <= tau) {
                        keep[j] = 1;
                        ++c;
                    }
                }
                if (adapt_cnt) adapt_cnt[bh * nb + i] = c;
            }
        free(score);
    }
    emit_mask(keep_all, BH, nb, Hp, Wp, wt, wh, ww, flags, bits, row_idx, row_cnt, col_idx,
              col_cnt);
    free(keep_all);
}

/* Stand-alone cuts on given score rows (used by the brute-force pins). */
int64_t oracle_cut_row_f64(const double *score, int64_t nb, double p, uint8_t *keep)
{
    rank_item *scratch = (rank_item *)malloc(sizeof(rank_item) * (size_t)nb);
    int64_t k = cut_row_f64(score, nb, p, keep, scratch, NULL, NULL);
    free(scratch);
    return k;
}

int64_t oracle_cut_row_fixed(const float *score, int64_t nb, float p, uint8_t *keep)
{
    rank_item *scratch = (rank_item *)malloc(sizeof(rank_item) * (size_t)nb);
    uint64_t *u = (uint64_t *)malloc(sizeof(uint64_t) * (size_t)nb);
    int64_t k = cut_row_fixed(score, nb, p, keep, scratch, u, NULL);
    free(scratch);
    free(u);
    return k;
}

/* ------------------------------------------------------------------------ */
/* Block-sparse attention over M (bullet "拡張" and section "STA とのハイブリッド */
/* 統合": attention is computed exactly on the kept blocks).  For query token  */
/* n in block i the keys are all tokens of all blocks j in row i of M:        */
/*   O_n = sum_m softmax_m(scale * q_n . k_m) v_m,  LSE_n = log sum_m e^(..). */
/* Inputs are float64 [BH, N, D] in flattened order (callers widen bf16).     */
/* ------------------------------------------------------------------------ */

/* One query row: fills o[D] and returns LSE.  logit: scratch of >= cnt*L. */
static double fwd_row(const double *q, const double *k, const double *v, int64_t bh,
                      int64_t n, int64_t N, int D, int L, const uint16_t *list, int32_t cnt,
                      double scale, double *o, double *logit)
{
    const double *qn = q + (bh * N + n) * D;
    double mx = -INFINITY;
    int64_t c = 0;
    for (int32_t e = 0; e < cnt; ++e) {
        int64_t j = list[e];
        for (int r = 0; r < L; ++r, ++c) {
            const double *km = k + (bh * N + j * L + r) * D;
            double s = 0.0;
            for (int d = 0; d < D; ++d) s += qn[d] * km[d];
            logit[c] = scale * s;
            mx = fmax(mx, logit[c]);
        }
    }
    double l = 0.0;
    for (int64_t e = 0; e < c; ++e) l += exp(logit[e] - mx);
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    c = 0;
    for (int32_t e = 0; e < cnt; ++e) {
        int64_t j = list[e];
        for (int r = 0; r < L; ++r, ++c) {
            const double *vm = v + (bh * N + j * L + r) * D;
            double pr = exp(logit[c] - mx) / l;
            for (int d = 0; d < D; ++d) o[d] += pr * vm[d];
        }
    }
    return mx + log(l);
}

/* Forward on selected query blocks (sel_bh[s], sel_i[s]); sel == NULL means
 * every (bh, i) in order.  o: [n_sel, L, D], lse: [n_sel, L]. */
void oracle_attn_fwd(const double *q, const double *k, const double *v, int64_t BH,
                     int64_t N, int D, int L, const uint16_t *row_idx, const int32_t *row_cnt,
                     double scale, const int64_t *sel_bh, const int64_t *sel_i, int64_t n_sel,
                     double *o, double *lse)
{
    int64_t nb = N / L;
    if (!sel_bh) n_sel = BH * nb;
#pragma omp parallel
    {
        double *logit = (double *)malloc(sizeof(double) * (size_t)N);
#pragma omp for schedule(dynamic, 1)
        for (int64_t s = 0; s < n_sel; ++s) {
            int64_t bh = sel_bh ? sel_bh[s] : s / nb;
            int64_t i = sel_i ? sel_i[s] : s % nb;
            const uint16_t *list = row_idx + (bh * nb + i) * nb;
            int32_t cnt = row_cnt[bh * nb + i];
            for (int r = 0; r < L; ++r)
                lse[s * L + r] = fwd_row(q, k, v, bh, i * L + r, N, D, L, list, cnt, scale,
                                         o + (s * L + r) * D, logit);
        }
        free(logit);
    }
}

/* Backward of the same function (training through the sparse attention):
 *   Dl_n = dO_n . O_n,  P_nm = exp(scale q_n.k_m - LSE_n),
 *   dV_m = sum_n P_nm dO_n,  dP_nm = dO_n . v_m,  dS_nm = P_nm (dP_nm - Dl_n),
 *   dQ_n = scale sum_m dS_nm k_m,  dK_m = scale sum_n dS_nm q_n,
 * summed over the pairs (n, m) whose blocks are in M.  O and LSE are
 * recomputed here in float64 from the forward definition.
 * dQ for the selected query blocks (dq_bh, dq_i) -> dq [n_dq, L, D];
 * dK, dV for the selected key blocks (kv_bh, kv_j) -> dk, dv [n_kv, L, D].
 * A NULL selection means every block, in order. */
void oracle_attn_bwd(const double *q, const double *k, const double *v, const double *dout,
                     int64_t BH, int64_t N, int D, int L, const uint16_t *row_idx,
                     const int32_t *row_cnt, const uint16_t *col_idx, const int32_t *col_cnt,
                     double scale, const int64_t *dq_bh, const int64_t *dq_i, int64_t n_dq,
                     const int64_t *kv_bh, const int64_t *kv_j, int64_t n_kv, double *dq,
                     double *dk, double *dv)
{
    int64_t nb = N / L;
    if (!dq_bh) n_dq = BH * nb;
    if (!kv_bh) n_kv = BH * nb;

    /* Row statistics (LSE_n, Dl_n) for every query block any output needs. */
    uint8_t *need = (uint8_t *)calloc((size_t)(BH * nb), 1);
    for (int64_t s = 0; s < n_dq; ++s)
        need[(dq_bh ? dq_bh[s] : s / nb) * nb + (dq_i ? dq_i[s] : s % nb)] = 1;
    for (int64_t s = 0; s < n_kv; ++s) {
        int64_t bh = kv_bh ? kv_bh[s] : s / nb;
        int64_t j = kv_j ? kv_j[s] : s % nb;
        const uint16_t *clist = col_idx + (bh * nb + j) * nb;
        for (int32_t e = 0; e < col_cnt[bh * nb + j]; ++e) need[bh * nb + clist[e]] = 1;
    }
    double *lse = (double *)malloc(sizeof(double) * (size_t)(BH * N));
    double *dl = (double *)malloc(sizeof(double) * (size_t)(BH * N));
#pragma omp parallel
    {
        double *logit = (double *)malloc(sizeof(double) * (size_t)N);
        double *o = (double *)malloc(sizeof(double) * (size_t)D);
#pragma omp for schedule(dynamic, 1)
        for (int64_t bi = 0; bi < BH * nb; ++bi) {
            if (!need[bi]) continue;
            int64_t bh = bi / nb, i = bi % nb;
            const uint16_t *list = row_idx + (bh * nb + i) * nb;
            int32_t cnt = row_cnt[bh * nb + i];
            for (int r = 0; r < L; ++r) {
                int64_t n = i * L + r;
                lse[bh * N + n] = fwd_row(q, k, v, bh, n, N, D, L, list, cnt, scale, o, logit);
                const double *don = dout + (bh * N + n) * D;
                double acc = 0.0;
                for (int d = 0; d < D; ++d) acc += don[d] * o[d];
                dl[bh * N + n] = acc;
            }
        }
        free(logit);
        free(o);
    }

    /* dQ: each selected query row over its own row list. */
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t s = 0; s < n_dq; ++s) {
        int64_t bh = dq_bh ? dq_bh[s] : s / nb;
        int64_t i = dq_i ? dq_i[s] : s % nb;
        const uint16_t *list = row_idx + (bh * nb + i) * nb;
        int32_t cnt = row_cnt[bh * nb + i];
        for (int r = 0; r < L; ++r) {
            int64_t n = i * L + r;
            const double *qn = q + (bh * N + n) * D;
            const double *don = dout + (bh * N + n) * D;
            double *g = dq + (s * L + r) * D;
            for (int d = 0; d < D; ++d) g[d] = 0.0;
            for (int32_t e = 0; e < cnt; ++e) {
                int64_t j = list[e];
                for (int rr = 0; rr < L; ++rr) {
                    const double *km = k + (bh * N + j * L + rr) * D;
                    const double *vm = v + (bh * N + j * L + rr) * D;
                    double sc = 0.0, dp = 0.0;
                    for (int d = 0; d < D; ++d) {
                        sc += qn[d] * km[d];
                        dp += don[d] * vm[d];
                    }
                    double pr = exp(scale * sc - lse[bh * N + n]);
                    double ds = pr * (dp - dl[bh * N + n]);
                    for (int d = 0; d < D; ++d) g[d] += scale * ds * km[d];
                }
            }
        }
    }

    /* dK, dV: each selected key block over its column list. */
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t s = 0; s < n_kv; ++s) {
        int64_t bh = kv_bh ? kv_bh[s] : s / nb;
        int64_t j = kv_j ? kv_j[s] : s % nb;
        double *gk = dk + s * L * D, *gv = dv + s * L * D;
        for (int64_t e = 0; e < (int64_t)L * D; ++e) gk[e] = gv[e] = 0.0;
        const uint16_t *clist = col_idx + (bh * nb + j) * nb;
        int32_t ccnt = col_cnt[bh * nb + j];
        for (int32_t e = 0; e < ccnt; ++e) {
            int64_t i = clist[e];
            for (int r = 0; r < L; ++r) {
                int64_t n = i * L + r;
                const double *qn = q + (bh * N + n) * D;
                const double *don = dout + (bh * N + n) * D;
                for (int rr = 0; rr < L; ++rr) {
                    const double *km = k + (bh * N + j * L + rr) * D;
                    const double *vm = v + (bh * N + j * L + rr) * D;
                    double sc = 0.0, dp = 0.0;
                    for (int d = 0; d < D; ++d) {
                        sc += qn[d] * km[d];
                        dp += don[d] * vm[d];
                    }
                    double pr = exp(scale * sc - lse[bh * N + n]);
                    double ds = pr * (dp - dl[bh * N + n]);
                    for (int d = 0; d < D; ++d) {
                        gv[rr * D + d] += pr * don[d];
                        gk[rr * D + d] += scale * ds * qn[d];
                    }
                }
            }
        }
    }
    free(need);
    free(lse);
    free(dl);
}
