/*
 * CPU oracle for SparSTAR's per-scale block-sparse attention forward.
 *
 * TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.  Only the test suite, the
 * smoke check and the CPU-baseline leg of the benchmark load this library.
 * It shares no code, header, table or helper with the CUDA path: it is a
 * plain, slow, deliberately unblocked restatement of what the method
 * computes, so that a reader can check it against the method's description
 * by eye.
 *
 * Sources (all on the pages describing SparSTAR, arXiv 2608.10519):
 *   [R-carry]  pith.science review of SparSTAR, "What carries the argument":
 *              contiguous 128-token blocks taken in the order the attention
 *              kernel walks them, block-averaged q and k,
 *              S_ij = tau * qbar_i^T kbar_j with
 *              tau = D^-1/2, the block-average identity, the text (and, in
 *              Clip 1, the last image-pyramid reference) always kept,
 *              reference and current blocks ranked jointly under a density
 *              schedule, forward-only block mask (per-row count + index
 *              list, no reverse index).
 *   [R-core]   same review, "Extended reading notes / Core claim":
 *              block-wise Top-K recomputed at every scale and head.
 *   [R-ref]    same review, "Referee Report", minor comment 5: the block-wise
 *              Top-K of one figure and the fresh aggregated-QK selection of
 *              one table are the same mechanism.
 *   [R-settle] same review, "What would settle it": replacing the block
 *              score by the exact token-wise Top-K at the same densities is
 *              the test of whether block aggregation costs fidelity.
 *   [R-abs]    SparSTAR abstract (mlsanity.com/paper/2608.10519): block
 *              scores computed anew per scale and head from that scale's
 *              own Q and K; only the chosen blocks are attended, forward
 *              only.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *   - One block grid over the concatenated keys, one over the queries;
 *     the last block of each grid may be partial and is averaged over its
 *     real tokens.
 *   - The fp32 means are summed in a fixed order (8 stripes by token index
 *     mod 8, ascending inside a stripe, stripes combined as a fixed tree),
 *     then divided once by the real token count.  The fp32 score is a
 *     sequential fused multiply-add over d ascending, then one multiply by
 *     tau.  These orders are this implementation's specification; the
 *     pages fix none.
 *   - Budget k = ceil(density * C) over the C non-forced blocks, ties to
 *     the lower block index; output list = forced prefix, then the chosen
 *     candidates ascending.
 *   - Attention scale tau = D^-1/2 (the score's tau); no causal mask; keys
 *     with index >= Lk do not exist.
 *
 * Data layout of every tensor: [B, H, L, D] row-major, D contiguous.
 * dtype 0 = bf16 (stored as uint16 bit patterns), 1 = fp32.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fopenmp -fPIC
 *        -shared (x86-64 SSE arithmetic, FLT_EVAL_METHOD == 0).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_BLOCK 128

#if defined(__FLT_EVAL_METHOD__) && __FLT_EVAL_METHOD__ != 0
#error "the oracle needs IEEE single-precision evaluation (FLT_EVAL_METHOD 0)"
#endif

/* ---------------------------------------------------------------- inputs */

/* bf16 -> fp32 is exact: the bf16 pattern is the top half of the fp32 one. */
static float orc_bf16_to_f32(uint16_t h)
{
    uint32_t bits = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return f;
}

static float orc_load(const void *x, int dtype, int64_t idx)
{
    if (dtype == 0)
        return orc_bf16_to_f32(((const uint16_t *)x)[idx]);
    return ((const float *)x)[idx];
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

static int64_t orc_nblocks(int64_t L) { return (L + ORC_BLOCK - 1) / ORC_BLOCK; }

/* ------------------------------------------------------- block structure */

/* Forced blocks: every key block that holds at least one text token or one
 * Clip-1 image-reference token ([R-carry]: text and the Clip-1 reference
 * are never dropped, so no forced token may be).  Keys are ordered
 * [text | image_ref | ref | cur], so the forced tokens are the prefix
 * 0 .. text_len + image_ref_len - 1. */
int64_t orc_forced_blocks(int64_t text_len, int64_t image_ref_len)
{
    if (text_len < 0 || image_ref_len < 0)
        return -1;
    return orc_nblocks(text_len + image_ref_len);
}

/* Selected blocks per query block: the forced prefix plus
 * k = ceil(density * C) of the C = nKB - nF candidates ([R-carry] density
 * schedule; rounding rule as read above).  Returns -1 on bad arguments. */
int64_t orc_select_count(int64_t nKB, int64_t nF, double density)
{
    if (nKB <= 0 || nF < 0 || nF > nKB || !(density > 0.0) || !(density <= 1.0))
        return -1;
    int64_t C = nKB - nF;
    double kd = ceil(density * (double)C);
    int64_t k = (int64_t)kd;
    if (k < 0) k = 0;
    if (k > C) k = C;
    return nF + k;
}

/* ------------------------------------------------------------ step 1: pool */

/* Block mean in fp32, fixed order ([R-carry] block-averaged vectors).
 * For a block of n real tokens t = 0..n-1 and one coordinate d:
 *   stripe r (r = 0..7) = x[r] + x[r+8] + x[r+16] + ... in ascending t,
 *                         starting from +0.0f;
 *   total = ((s0+s1)+(s2+s3)) + ((s4+s5)+(s6+s7));
 *   mean  = total / (float)n   (one IEEE division).
 * xbar: [B, H, ceil(L/128), D] fp32. */
void orc_pool_f32(const void *x, int dtype, int64_t B, int64_t H, int64_t L,
                  int64_t D, float *xbar)
{
    const int64_t nblk = orc_nblocks(L);
    const int64_t nrow = B * H * nblk;
#pragma omp parallel for schedule(static)
    for (int64_t row = 0; row < nrow; ++row) {
        const int64_t bh = row / nblk;
        const int64_t blk = row % nblk;
        const int64_t t0 = blk * ORC_BLOCK;
        const int64_t n = (L - t0 < ORC_BLOCK) ? (L - t0) : ORC_BLOCK;
        for (int64_t d = 0; d < D; ++d) {
            float s[8];
            for (int r = 0; r < 8; ++r)
                s[r] = 0.0f;
            for (int64_t t = 0; t < n; ++t) {
                const int64_t idx = (bh * L + t0 + t) * D + d;
                s[t % 8] = s[t % 8] + orc_load(x, dtype, idx);
            }
            const float left = (s[0] + s[1]) + (s[2] + s[3]);
            const float right = (s[4] + s[5]) + (s[6] + s[7]);
            const float total = left + right;
            xbar[row * D + d] = total / (float)n;
        }
    }
}

/* Block mean in fp64: the plain definition (sum of the block's real tokens
 * divided by their count). */
void orc_pool_f64(const void *x, int dtype, int64_t B, int64_t H, int64_t L,
                  int64_t D, double *xbar)
{
    const int64_t nblk = orc_nblocks(L);
    const int64_t nrow = B * H * nblk;
#pragma omp parallel for schedule(static)
    for (int64_t row = 0; row < nrow; ++row) {
        const int64_t bh = row / nblk;
        const int64_t blk = row % nblk;
        const int64_t t0 = blk * ORC_BLOCK;
        const int64_t n = (L - t0 < ORC_BLOCK) ? (L - t0) : ORC_BLOCK;
        for (int64_t d = 0; d < D; ++d) {
            double acc = 0.0;
            for (int64_t t = 0; t < n; ++t)
                acc += (double)orc_load(x, dtype, (bh * L + t0 + t) * D + d);
            xbar[row * D + d] = acc / (double)n;
        }
    }
}

/* ----------------------------------------------------------- step 2: score */

/* S_ij = tau * qbar_i . kbar_j ([R-carry], the paper's Eq. 2), fp32:
 *   acc = +0.0f; for d = 0..D-1: acc = fmaf(qbar[d], kbar[d], acc);
 *   S = acc * tau   (one IEEE multiply; tau is passed in as fp32).
 * S: [B, H, nQB, nKB] fp32.  Forced blocks are scored too. */
void orc_score_f32(const float *qbar, const float *kbar, int64_t B, int64_t H,
                   int64_t nQB, int64_t nKB, int64_t D, float tau, float *S)
{
    const int64_t nrow = B * H * nQB;
#pragma omp parallel for schedule(static)
    for (int64_t row = 0; row < nrow; ++row) {
        const int64_t bh = row / nQB;
        const float *qi = qbar + row * D;
        for (int64_t j = 0; j < nKB; ++j) {
            const float *kj = kbar + (bh * nKB + j) * D;
            float acc = 0.0f;
            for (int64_t d = 0; d < D; ++d)
                acc = fmaf(qi[d], kj[d], acc);
            S[row * nKB + j] = acc * tau;
        }
    }
}

/* Same score in fp64 with tau = 1/sqrt(D) in fp64. */
void orc_score_f64(const double *qbar, const double *kbar, int64_t B, int64_t H,
                   int64_t nQB, int64_t nKB, int64_t D, double *S)
{
    const double tau = 1.0 / sqrt((double)D);
    const int64_t nrow = B * H * nQB;
#pragma omp parallel for schedule(static)
    for (int64_t row = 0; row < nrow; ++row) {
        const int64_t bh = row / nQB;
        const double *qi = qbar + row * D;
        for (int64_t j = 0; j < nKB; ++j) {
            const double *kj = kbar + (bh * nKB + j) * D;
            double acc = 0.0;
            for (int64_t d = 0; d < D; ++d)
                acc += qi[d] * kj[d];
            S[row * nKB + j] = tau * acc;
        }
    }
}

/* ---------------------------------------------------------- step 2b: select */

typedef struct {
    double score;
    int32_t j;
} orc_cand;

/* Higher score first; equal scores (IEEE equality, so -0 == +0) go to the
 * lower block index. */
static int orc_cand_cmp(const void *pa, const void *pb)
{
    const orc_cand *a = (const orc_cand *)pa, *b = (const orc_cand *)pb;
    if (a->score > b->score) return -1;
    if (a->score < b->score) return 1;
    return (a->j < b->j) ? -1 : (a->j > b->j);
}

static int orc_int_cmp(const void *pa, const void *pb)
{
    const int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

/* One row of the clip-aware block Top-K ([R-carry] policy, [R-ref]):
 * forced blocks 0..nF-1 are kept; the candidates nF..nKB-1 (blocks of the
 * earlier clip's context and of this scale, in one pool) are sorted by score and the
 * first k kept; the list is written forced-first, then the chosen
 * candidates in ascending block order. */
static void orc_select_row(const double *scores, int64_t nKB, int64_t nF,
                           int64_t k, int32_t *out, orc_cand *tmp)
{
    const int64_t C = nKB - nF;
    for (int64_t c = 0; c < C; ++c) {
        tmp[c].score = scores[nF + c];
        tmp[c].j = (int32_t)(nF + c);
    }
    qsort(tmp, (size_t)C, sizeof(orc_cand), orc_cand_cmp);
    for (int64_t f = 0; f < nF; ++f)
        out[f] = (int32_t)f;
    for (int64_t c = 0; c < k; ++c)
        out[nF + c] = tmp[c].j;
    qsort(out + nF, (size_t)k, sizeof(int32_t), orc_int_cmp);
}

static int orc_select_common(const float *S32, const double *S64, int64_t B,
                             int64_t H, int64_t nQB, int64_t nKB, int64_t nF,
                             double density, int32_t *kv_idx, int32_t *kv_cnt,
                             int64_t max_sel)
{
    const int64_t sel = orc_select_count(nKB, nF, density);
    if (sel < 0 || sel > max_sel)
        return -1;
    const int64_t k = sel - nF;
    const int64_t nrow = B * H * nQB;
    int bad = 0;
#pragma omp parallel
    {
        double *row_scores = (double *)malloc(sizeof(double) * (size_t)nKB);
        orc_cand *tmp = (orc_cand *)malloc(sizeof(orc_cand) * (size_t)nKB);
#pragma omp for schedule(static)
        for (int64_t row = 0; row < nrow; ++row) {
            for (int64_t j = 0; j < nKB; ++j) {
                /* fp32 scores are compared exactly as fp32 values: the
                 * widening to double preserves order and equality. */
                const double s = S32 ? (double)S32[row * nKB + j] : S64[row * nKB + j];
                if (!isfinite(s)) {
#pragma omp atomic write
                    bad = 1;
                }
                row_scores[j] = s;
            }
            orc_select_row(row_scores, nKB, nF, k, kv_idx + row * max_sel, tmp);
            for (int64_t c = sel; c < max_sel; ++c)
                kv_idx[row * max_sel + c] = -1;
            kv_cnt[row] = (int32_t)sel;
        }
        free(row_scores);
        free(tmp);
    }
    return bad ? -2 : 0;
}

/* Selection on fp32 scores (the bit-exact target).  kv_idx:
 * [B,H,nQB,max_sel] int32 (unused tail slots = -1), kv_cnt: [B,H,nQB].
 * Returns 0, -1 (bad sizes / density) or -2 (non-finite score). */
int orc_select_f32(const float *S, int64_t B, int64_t H, int64_t nQB, int64_t nKB,
                   int64_t nF, double density, int32_t *kv_idx, int32_t *kv_cnt,
                   int64_t max_sel)
{
    return orc_select_common(S, NULL, B, H, nQB, nKB, nF, density, kv_idx, kv_cnt,
                             max_sel);
}

/* Same selection on fp64 scores (the mathematical selection). */
int orc_select_f64(const double *S, int64_t B, int64_t H, int64_t nQB, int64_t nKB,
                   int64_t nF, double density, int32_t *kv_idx, int32_t *kv_cnt,
                   int64_t max_sel)
{
    return orc_select_common(NULL, S, B, H, nQB, nKB, nF, density, kv_idx, kv_cnt,
                             max_sel);
}

/* Near-tie gap of one row of fp64 scores: with the candidate scores sorted
 * descending s(1) >= s(2) >= ..., gap = s(k) - s(k+1) and scale =
 * max_j |S_j| over the candidates.  Writes gap (or +inf when k == 0 or
 * k == C) and scale per row. */
void orc_near_tie_gaps(const double *S, int64_t nrow, int64_t nKB, int64_t nF,
                       int64_t k, double *gap, double *scale)
{
    const int64_t C = nKB - nF;
#pragma omp parallel
    {
        orc_cand *tmp = (orc_cand *)malloc(sizeof(orc_cand) * (size_t)(C > 0 ? C : 1));
#pragma omp for schedule(static)
        for (int64_t row = 0; row < nrow; ++row) {
            double mx = 0.0;
            for (int64_t c = 0; c < C; ++c) {
                tmp[c].score = S[row * nKB + nF + c];
                tmp[c].j = (int32_t)(nF + c);
                if (fabs(tmp[c].score) > mx) mx = fabs(tmp[c].score);
            }
            qsort(tmp, (size_t)C, sizeof(orc_cand), orc_cand_cmp);
            gap[row] = (k <= 0 || k >= C) ? INFINITY : tmp[k - 1].score - tmp[k].score;
            scale[row] = mx;
        }
        free(tmp);
    }
}

/* --------------------------------------------------------- step 3: attention */

/* Forward attention over the selected blocks, fp64, for a list of query
 * rows ([R-carry] forward-only sparse path, [R-abs]).  For query row r of
 * head bh (query block i = r / 128) the visible keys are the tokens t of
 * every listed key block j with 128 j <= t < min(128 (j+1), Lk):
 *   s_t   = tau * q_r . k_t,  tau = 1/sqrt(D) in fp64
 *   out_r = sum_t exp(s_t - m) v_t / sum_t exp(s_t - m),  m = max_t s_t
 *   lse_r = m + log(sum_t exp(s_t - m))          (natural log)
 * A row with no visible key gets out = 0 and lse = -inf.
 * rows: flat indices bh * Lq + r.  out: [n_rows, D] fp64, lse: [n_rows]. */
void orc_attn_rows_f64(const void *q, const void *k, const void *v, int dtype,
                       int64_t B, int64_t H, int64_t Lq, int64_t Lk, int64_t D,
                       const int32_t *kv_idx, const int32_t *kv_cnt, int64_t max_sel,
                       int64_t n_rows, const int64_t *rows, double *out, double *lse)
{
    (void)B;
    (void)H;
    const int64_t nQB = orc_nblocks(Lq);
    const int64_t nKB = orc_nblocks(Lk);
    const double tau = 1.0 / sqrt((double)D);
#pragma omp parallel
    {
        double *qv = (double *)malloc(sizeof(double) * (size_t)D);
        double *s = (double *)malloc(sizeof(double) * (size_t)(max_sel * ORC_BLOCK + 1));
#pragma omp for schedule(dynamic, 16)
        for (int64_t n = 0; n < n_rows; ++n) {
            const int64_t flat = rows[n];
            const int64_t bh = flat / Lq;
            const int64_t r = flat % Lq;
            const int64_t i = r / ORC_BLOCK;
            const int64_t list = bh * nQB + i;
            int64_t cnt = kv_cnt[list];
            if (cnt > max_sel) cnt = max_sel;
            for (int64_t d = 0; d < D; ++d)
                qv[d] = (double)orc_load(q, dtype, (bh * Lq + r) * D + d);

            /* pass 1: scores of every visible key, in list order */
            int64_t nvis = 0;
            double m = -INFINITY;
            for (int64_t c = 0; c < cnt; ++c) {
                const int64_t j = kv_idx[list * max_sel + c];
                if (j < 0 || j >= nKB) continue;
                for (int64_t t = j * ORC_BLOCK; t < (j + 1) * ORC_BLOCK && t < Lk; ++t) {
                    double dot = 0.0;
                    for (int64_t d = 0; d < D; ++d)
                        dot += qv[d] * (double)orc_load(k, dtype, (bh * Lk + t) * D + d);
                    s[nvis] = tau * dot;
                    if (s[nvis] > m) m = s[nvis];
                    ++nvis;
                }
            }
            double *o = out + n * D;
            for (int64_t d = 0; d < D; ++d)
                o[d] = 0.0;
            if (nvis == 0) {
                lse[n] = -INFINITY;
                continue;
            }
            /* pass 2: softmax weights and the weighted sum of values */
            double l = 0.0;
            int64_t u = 0;
            for (int64_t c = 0; c < cnt; ++c) {
                const int64_t j = kv_idx[list * max_sel + c];
                if (j < 0 || j >= nKB) continue;
                for (int64_t t = j * ORC_BLOCK; t < (j + 1) * ORC_BLOCK && t < Lk; ++t) {
                    const double p = exp(s[u++] - m);
                    l += p;
                    for (int64_t d = 0; d < D; ++d)
                        o[d] += p * (double)orc_load(v, dtype, (bh * Lk + t) * D + d);
                }
            }
            for (int64_t d = 0; d < D; ++d)
                o[d] /= l;
            lse[n] = m + log(l);
        }
        free(qv);
        free(s);
    }
}

/* ------------------------------------------- diagnostic: retained mass */

static int orc_desc_double(const void *a, const void *b)
{
    const double x = *(const double *)a, y = *(const double *)b;
    return (x < y) - (x > y);
}

/* Retained attention mass of a block list and the token-wise bound at the
 * same budget, for the given flat query rows (bh * Lq + r), in fp64.
 * [R-core]: block-wise Top-K recomputed at every scale stays close to the
 * token-wise upper bound in retained attention mass; [R-settle]: the exact
 * token-wise Top-K at the same densities is the comparison.  With the dense
 * weights p_t = exp(tau q.k_t) / sum_u exp(tau q.k_u) over every key t < Lk:
 *   lse_dense   = log sum_t exp(tau q.k_t)             (natural log);
 *   mass_block  = sum of p_t over the tokens of the row's listed blocks;
 *   mass_forced = sum of p_t over the tokens of blocks 0 .. nF-1;
 *   M           = real tokens in the listed blocks j >= nF (the candidate
 *                 budget the block list spends);
 *   mass_tok    = mass_forced + the sum of the M largest p_t over the
 *                 candidate tokens t >= 128 nF.
 * Reading: the bound keeps the policy's forced blocks and spends the same
 * number of candidate tokens freely, so mass_forced <= mass_block <=
 * mass_tok <= 1.  List entries outside [0, nKB) are ignored, as in the
 * attention. */
void orc_retained_mass_f64(const void *q, const void *k, int dtype, int64_t B, int64_t H,
                           int64_t Lq, int64_t Lk, int64_t D, int64_t nF,
                           const int32_t *kv_idx, const int32_t *kv_cnt, int64_t max_sel,
                           int64_t n_rows, const int64_t *rows, double *lse_dense,
                           double *mass_block, double *mass_tok, double *mass_forced)
{
    (void)B;
    (void)H;
    const int64_t nQB = orc_nblocks(Lq);
    const int64_t nKB = orc_nblocks(Lk);
    const double tau = 1.0 / sqrt((double)D);
    int64_t f_end = nF * ORC_BLOCK; /* first candidate token */
    if (f_end > Lk) f_end = Lk;
#pragma omp parallel
    {
        double *qv = (double *)malloc(sizeof(double) * (size_t)D);
        double *s = (double *)malloc(sizeof(double) * (size_t)Lk);
        double *cand = (double *)malloc(sizeof(double) * (size_t)(Lk - f_end + 1));
        char *listed = (char *)malloc((size_t)nKB);
#pragma omp for schedule(dynamic, 1)
        for (int64_t n = 0; n < n_rows; ++n) {
            const int64_t flat = rows[n];
            const int64_t bh = flat / Lq;
            const int64_t r = flat % Lq;
            const int64_t list = bh * nQB + r / ORC_BLOCK;
            for (int64_t d = 0; d < D; ++d)
                qv[d] = (double)orc_load(q, dtype, (bh * Lq + r) * D + d);
            /* every key's score, and the softmax normaliser */
            double m = -INFINITY;
            for (int64_t t = 0; t < Lk; ++t) {
                double dot = 0.0;
                for (int64_t d = 0; d < D; ++d)
                    dot += qv[d] * (double)orc_load(k, dtype, (bh * Lk + t) * D + d);
                s[t] = tau * dot;
                if (s[t] > m) m = s[t];
            }
            double z = 0.0;
            for (int64_t t = 0; t < Lk; ++t)
                z += exp(s[t] - m);
            const double lse = m + log(z);
            /* the row's listed blocks */
            for (int64_t j = 0; j < nKB; ++j)
                listed[j] = 0;
            int64_t cnt = kv_cnt[list];
            if (cnt > max_sel) cnt = max_sel;
            for (int64_t c = 0; c < cnt; ++c) {
                const int64_t j = kv_idx[list * max_sel + c];
                if (j >= 0 && j < nKB) listed[j] = 1;
            }
            double mb = 0.0, mf = 0.0;
            int64_t budget = 0;
            for (int64_t t = 0; t < Lk; ++t) {
                const double p = exp(s[t] - lse);
                if (listed[t / ORC_BLOCK]) {
                    mb += p;
                    if (t >= f_end) ++budget;
                }
                if (t < f_end) mf += p;
            }
            /* the M largest candidate weights */
            const int64_t nc = Lk - f_end;
            for (int64_t t = 0; t < nc; ++t)
                cand[t] = exp(s[f_end + t] - lse);
            qsort(cand, (size_t)nc, sizeof(double), orc_desc_double);
            double top = 0.0;
            for (int64_t t = 0; t < budget && t < nc; ++t)
                top += cand[t];
            lse_dense[n] = lse;
            mass_block[n] = mb;
            mass_forced[n] = mf;
            mass_tok[n] = mf + top;
        }
        free(qv);
        free(s);
        free(cand);
        free(listed);
    }
}

/* --------------------------------------- diagnostic: lists reused across scales */

/* The image of one target token: its segment g's source token at offset
 * floor(p * len_s[g] / len_t[g]), or -1 when len_s[g] = 0. */
static int64_t orc_image(int64_t t, const int64_t *off_s, const int64_t *off_t,
                         const int64_t *len_s, const int64_t *len_t)
{
    for (int g = 0; g < 4; ++g) {
        if (t >= off_t[g] && t < off_t[g] + len_t[g]) {
            if (len_s[g] == 0) return -1;
            return off_s[g] + (t - off_t[g]) * len_s[g] / len_t[g];
        }
    }
    return -1;
}

/* The block lists of a source scale carried to a target scale by position:
 * the "reuse" that the method argues against ([R-core]: a selection
 * carried from one scale to another keeps less of the attention mass than
 * a fresh one, so the method selects anew at every scale; the review's Figure 1: a
 * mask carried over from an earlier scale can leave out blocks that matter
 * at the new one).  The pages give no map between two scales' token
 * positions; the reading used (listed in the design notes) resamples the
 * block mask by nearest neighbour along the token order:
 *   - keys at both scales are the segments [text | image_ref | ref | cur];
 *     segment g has len_s[g] tokens at the source and len_t[g] at the
 *     target (queries are the cur segment);
 *   - the target token at offset p of segment g has as image the source
 *     token at offset floor(p * len_s[g] / len_t[g]) of the same segment,
 *     and none when len_s[g] = 0;
 *   - the centre of a block of n real tokens starting at token a is token
 *     a + floor((n - 1) / 2);
 *   - target query block i uses the list of the source query block holding
 *     the image of i's centre query token;
 *   - target key block j is kept when j < nF_t (forced at the target) or
 *     when the source block holding the image of j's centre token is in
 *     that list.
 * Output kv_idx_t [B,H,nQB_t,max_sel_t]: the kept blocks ascending, unused
 * slots -1; kv_cnt_t [B,H,nQB_t].  Source entries outside [0, nKB_s) are
 * ignored; a source count above max_sel_s is read as max_sel_s.
 * Returns 0; -1 if a row keeps more than max_sel_t blocks (nothing past
 * the stride is written); -2 if len_s[3] = 0 < len_t[3]. */
int orc_transfer_lists(const int32_t *idx_s, const int32_t *cnt_s, int64_t max_sel_s,
                       int64_t B, int64_t H, const int64_t *len_s, const int64_t *len_t,
                       int32_t *idx_t, int32_t *cnt_t, int64_t max_sel_t)
{
    int64_t off_s[4], off_t[4], Lk_s = 0, Lk_t = 0;
    for (int g = 0; g < 4; ++g) {
        off_s[g] = Lk_s;
        off_t[g] = Lk_t;
        Lk_s += len_s[g];
        Lk_t += len_t[g];
    }
    const int64_t nKB_s = orc_nblocks(Lk_s), nKB_t = orc_nblocks(Lk_t);
    const int64_t nQB_s = orc_nblocks(len_s[3]), nQB_t = orc_nblocks(len_t[3]);
    const int64_t nF_t = orc_forced_blocks(len_t[0], len_t[1]);
    if (len_t[3] > 0 && len_s[3] == 0) return -2;
    int overflow = 0;
#pragma omp parallel for schedule(dynamic, 4) reduction(| : overflow)
    for (int64_t row = 0; row < B * H * nQB_t; ++row) {
        const int64_t bh = row / nQB_t;
        const int64_t i = row % nQB_t;
        /* the source row: the block of the image of i's centre query token */
        const int64_t qa = i * ORC_BLOCK;
        const int64_t qn = (len_t[3] - qa < ORC_BLOCK) ? len_t[3] - qa : ORC_BLOCK;
        const int64_t q_img = (qa + (qn - 1) / 2) * len_s[3] / len_t[3];
        const int64_t src_row = bh * nQB_s + q_img / ORC_BLOCK;
        int64_t n_src = cnt_s[src_row];
        if (n_src > max_sel_s) n_src = max_sel_s;
        if (n_src < 0) n_src = 0;
        const int32_t *list = idx_s + src_row * max_sel_s;
        int64_t n = 0;
        for (int64_t j = 0; j < nKB_t; ++j) {
            int keep = j < nF_t;
            if (!keep) {
                const int64_t a = j * ORC_BLOCK;
                const int64_t nj = (Lk_t - a < ORC_BLOCK) ? Lk_t - a : ORC_BLOCK;
                const int64_t img = orc_image(a + (nj - 1) / 2, off_s, off_t, len_s, len_t);
                if (img >= 0) {
                    const int64_t sb = img / ORC_BLOCK;
                    for (int64_t c = 0; c < n_src; ++c)
                        if (list[c] >= 0 && list[c] < nKB_s && list[c] == sb) {
                            keep = 1;
                            break;
                        }
                }
            }
            if (keep) {
                if (n < max_sel_t) idx_t[row * max_sel_t + n] = (int32_t)j;
                ++n;
            }
        }
        if (n > max_sel_t) overflow = 1;
        for (int64_t c = n; c < max_sel_t; ++c)
            idx_t[row * max_sel_t + c] = -1;
        cnt_t[row] = (int32_t)n;
    }
    return overflow ? -1 : 0;
}
