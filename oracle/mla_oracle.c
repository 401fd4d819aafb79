/*
 * mla_oracle.c -- fp64 CPU oracle for absorbed-form MLA decode.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the correctness reference that the
 * GPU path is checked against.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load it.  It shares no code, header, table
 * or constant with the CUDA library, and the CUDA library never calls it.
 *
 * What it computes (all arithmetic in IEEE double):
 *
 *   For every sequence b, query position i < s_q and head h:
 *     n_i    = clamp(seqlen_b - s_q + 1 + i, 0, seqlen_b)      visible tokens
 *     k_j    = kv_cache[block_table[b][j / 64]][j % 64][0:576]  token j's row
 *     s_j    = scale * sum_{d<576} q[b,i,h,d] * k_j[d]          score
 *     m      = max_j s_j,   l = sum_j exp(s_j - m)
 *     out[c] = sum_j exp(s_j - m) * k_j[c] / l                  c < 512
 *     lse    = m + ln(l)
 *   with out = 0, lse = -inf when n_i = 0.
 *
 * Sources (the pages the method is taken from):
 *   - "FlashMLA-ETAP: Efficient Transpose Attention Pipeline for Accelerating
 *     MLA Inference on NVIDIA H20 GPUs" (gist.science explainer), technical
 *     summary, "Methodology / core mechanism": the standard flow S = Q K^T,
 *     P = softmax(S), O = P V, and the transposed flow S^T = K Q^T,
 *     P^T = softmax(S^T), O = (V^T P^T)^T that the method uses instead.
 *     "Problem statement" and "Limitations": decode with 1-2 query tokens,
 *     16 heads, head dim 576, context up to 64K.
 *   - "FlashMLA: compressing the KV cache to one eighth" (jsqmd.com),
 *     "FlashMLA compute flow", step 4: online softmax over KV tiles with a
 *     running max and running sum.  The printed loop updates the running sum
 *     after overwriting the running max, so its rescale factor is always 1;
 *     the recurrence below uses exp(m_old - m_new) as the algebra requires.
 *   - The juejin.cn "FlashMLA" post, section 2: attention is Softmax(Q K^T) V.
 *
 * Readings where the pages are silent (each is listed with its reason in the
 * design notes): the 576 = 512 latent + 64 rope split and V = the first 512
 * columns of the cached row; scale applied to the fp64 scores, never folded
 * into q; natural-log lse; query i of s_q sees seqlen - s_q + 1 + i tokens;
 * an empty visible context gives out = 0 and lse = -inf; rows past the
 * visible count never enter the arithmetic, whatever bytes they hold.
 *
 * Inputs are the same bf16 bit patterns the GPU reads, widened exactly to
 * double.  Four forms are provided:
 *   mla_oracle_direct       the definition above, one (b, i, h) at a time;
 *   mla_oracle_transposed   the transposed flow, as whole matrices per
 *                           sequence: S^T = K Q^T, column softmax, O^T = V^T P^T;
 *   mla_oracle_online       the tiled online-softmax recurrence;
 *   mla_oracle_split_merge  per-range partial results merged through their lse;
 *   mla_oracle_merge_states the merge step alone, on given partial results
 *                           (the context-parallel form: each of W ranks
 *                           attends over its own range of the tokens);
 *   mla_oracle_direct_fp8   the definition over an FP8 (e4m3) cache with one
 *                           fp32 scale per cached token;
 *   mla_oracle_naive        the non-absorbed form: each token's key and value
 *                           decompressed from its latent row by per-head
 *                           up-projection matrices, then softmax(Q K^T) V
 *                           with 192-wide keys and 128-wide values (see the
 *                           comment above that function).
 * They agree to rounding; the tests pin each one to closed forms, library
 * routines and invariants.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_DQK 576   /* q / k row width: 512 latent + 64 rope           */
#define ORC_DNOPE 128 /* non-absorbed form: decompressed key / value width */
#define ORC_DROPE 64  /* rope columns (the last 64 of a cached row)        */
#define ORC_DV 512    /* v width: the first 512 columns of the same row   */
#define ORC_PAGE 64   /* tokens per paged block                          */

#define ORC_OK 0
#define ORC_BAD_ARG -1
#define ORC_BAD_BLOCK -2
#define ORC_NO_MEMORY -3

/* bf16 is the top half of an IEEE binary32; widening to double is exact. */
static double bf16_to_double(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Number of cached tokens that query i of an s_q-token query may attend to. */
static int64_t visible_tokens(int64_t seqlen, int s_q, int i)
{
    int64_t n = seqlen - s_q + 1 + i;
    if (n < 0) n = 0;
    if (n > seqlen) n = seqlen;
    return n;
}

typedef struct {
    const uint16_t *q;
    const uint16_t *kv;
    const int32_t *block_table;
    const int32_t *seqlens;
    int B, s_q, H;
    int64_t num_blocks;
    int max_blocks;
    double scale;
} problem_t;

/* Row of token j of sequence b, found through the page table; NULL if the
 * table entry does not name a block of the cache. */
static const uint16_t *token_row(const problem_t *p, int b, int64_t j)
{
    int64_t page = j / ORC_PAGE;
    if (page >= p->max_blocks) return NULL;
    int32_t blk = p->block_table[(int64_t)b * p->max_blocks + page];
    if (blk < 0 || (int64_t)blk >= p->num_blocks) return NULL;
    return p->kv + ((int64_t)blk * ORC_PAGE + j % ORC_PAGE) * ORC_DQK;
}

static const uint16_t *query_row(const problem_t *p, int b, int i, int h)
{
    return p->q + (((int64_t)b * p->s_q + i) * p->H + h) * ORC_DQK;
}

static int check_problem(const problem_t *p)
{
    if (!p->q || !p->kv || !p->block_table || !p->seqlens) return ORC_BAD_ARG;
    if (p->B < 0 || p->s_q < 1 || p->H < 1 || p->max_blocks < 1) return ORC_BAD_ARG;
    for (int b = 0; b < p->B; ++b) {
        int64_t L = p->seqlens[b];
        if (L < 0) return ORC_BAD_ARG;
        for (int64_t j = 0; j < L; j += ORC_PAGE)
            if (!token_row(p, b, j)) return ORC_BAD_BLOCK;
    }
    return ORC_OK;
}

/* Selected sequences: the listed ones, or all of them when list == NULL. */
static int list_len(const problem_t *p, const int32_t *list, int n_list)
{
    return list ? n_list : p->B;
}
static int list_at(const int32_t *list, int k) { return list ? list[k] : k; }

int mla_oracle_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* Direct form: the definition, one (b, i, h) output row at a time.          */
/* ------------------------------------------------------------------------ */
int mla_oracle_direct(const uint16_t *q, const uint16_t *kv_cache,
                      const int32_t *block_table, const int32_t *seqlens,
                      int B, int s_q, int H, int64_t num_blocks, int max_blocks,
                      double scale, const int32_t *seq_list, int n_seq_list,
                      double *out, double *lse)
{
    problem_t p = {q, kv_cache, block_table, seqlens, B, s_q, H, num_blocks,
                   max_blocks, scale};
    int rc = check_problem(&p);
    if (rc != ORC_OK) return rc;
    const int nb = list_len(&p, seq_list, n_seq_list);
    const int64_t rows = (int64_t)nb * s_q * H;
    int failed = 0;

#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < rows; ++r) {
        const int b = list_at(seq_list, (int)(r / ((int64_t)s_q * H)));
        const int i = (int)((r / H) % s_q);
        const int h = (int)(r % H);
        const int64_t n = visible_tokens(seqlens[b], s_q, i);
        double *o = out + (((int64_t)b * s_q + i) * H + h) * ORC_DV;
        double *ls = lse + ((int64_t)b * s_q + i) * H + h;
        for (int c = 0; c < ORC_DV; ++c) o[c] = 0.0;
        if (n == 0) {
            *ls = -INFINITY;
            continue;
        }
        double *s = (double *)malloc((size_t)n * sizeof(double));
        if (!s) {
            failed = 1;
            continue;
        }
        double qv[ORC_DQK];
        const uint16_t *qr = query_row(&p, b, i, h);
        for (int d = 0; d < ORC_DQK; ++d) qv[d] = bf16_to_double(qr[d]);

        /* scores and their maximum */
        double m = -INFINITY;
        for (int64_t j = 0; j < n; ++j) {
            const uint16_t *k = token_row(&p, b, j);
            double dot = 0.0;
            for (int d = 0; d < ORC_DQK; ++d) dot += qv[d] * bf16_to_double(k[d]);
            s[j] = scale * dot;
            if (s[j] > m) m = s[j];
        }
        /* softmax weights, their sum, and the weighted sum of value rows */
        double l = 0.0;
        for (int64_t j = 0; j < n; ++j) {
            const uint16_t *k = token_row(&p, b, j);
            const double w = exp(s[j] - m);
            l += w;
            for (int c = 0; c < ORC_DV; ++c) o[c] += w * bf16_to_double(k[c]);
        }
        for (int c = 0; c < ORC_DV; ++c) o[c] /= l;
        *ls = m + log(l);
        free(s);
    }
    return failed ? ORC_NO_MEMORY : ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Transposed form (the method's flow): per sequence, with N = s_q * H       */
/* query columns and n = seqlen key rows,                                     */
/*   S^T[j][c] = sum_d K[j][d] * Q^T[d][c]          (n x N)                   */
/*   P^T       = softmax of each column of S^T, masked to its visible rows    */
/*   O^T[c'][c] = sum_j V^T[c'][j] * P^T[j][c]      (512 x N)                 */
/*   O = (O^T)^T                                                             */
/* ------------------------------------------------------------------------ */
int mla_oracle_transposed(const uint16_t *q, const uint16_t *kv_cache,
                          const int32_t *block_table, const int32_t *seqlens,
                          int B, int s_q, int H, int64_t num_blocks, int max_blocks,
                          double scale, const int32_t *seq_list, int n_seq_list,
                          double *out, double *lse)
{
    problem_t p = {q, kv_cache, block_table, seqlens, B, s_q, H, num_blocks,
                   max_blocks, scale};
    int rc = check_problem(&p);
    if (rc != ORC_OK) return rc;
    const int nb = list_len(&p, seq_list, n_seq_list);
    const int N = s_q * H;
    int failed = 0;

#pragma omp parallel for schedule(dynamic, 1)
    for (int sb = 0; sb < nb; ++sb) {
        const int b = list_at(seq_list, sb);
        const int64_t n = seqlens[b];
        double *K = (double *)malloc((size_t)(n > 0 ? n : 1) * ORC_DQK * sizeof(double));
        double *QT = (double *)malloc((size_t)ORC_DQK * N * sizeof(double));
        double *ST = (double *)malloc((size_t)(n > 0 ? n : 1) * N * sizeof(double));
        double *OT = (double *)malloc((size_t)ORC_DV * N * sizeof(double));
        double *colmax = (double *)malloc((size_t)N * sizeof(double));
        double *colsum = (double *)malloc((size_t)N * sizeof(double));
        if (!K || !QT || !ST || !OT || !colmax || !colsum) {
            failed = 1;
            free(K); free(QT); free(ST); free(OT); free(colmax); free(colsum);
            continue;
        }
        /* K: the sequence's key rows, in token order, gathered through pages */
        for (int64_t j = 0; j < n; ++j) {
            const uint16_t *k = token_row(&p, b, j);
            for (int d = 0; d < ORC_DQK; ++d) K[j * ORC_DQK + d] = bf16_to_double(k[d]);
        }
        /* Q^T: column c = i * H + h holds query row (i, h) */
        for (int i = 0; i < s_q; ++i)
            for (int h = 0; h < H; ++h) {
                const uint16_t *qr = query_row(&p, b, i, h);
                for (int d = 0; d < ORC_DQK; ++d)
                    QT[(int64_t)d * N + i * H + h] = bf16_to_double(qr[d]);
            }
        /* S^T = scale * K Q^T; masked entries take -inf */
        for (int64_t j = 0; j < n; ++j)
            for (int c = 0; c < N; ++c) {
                const int i = c / H;
                if (j >= visible_tokens(n, s_q, i)) {
                    ST[j * N + c] = -INFINITY;
                    continue;
                }
                double dot = 0.0;
                for (int d = 0; d < ORC_DQK; ++d) dot += K[j * ORC_DQK + d] * QT[(int64_t)d * N + c];
                ST[j * N + c] = scale * dot;
            }
        /* column-wise softmax of S^T */
        for (int c = 0; c < N; ++c) {
            double m = -INFINITY;
            for (int64_t j = 0; j < n; ++j)
                if (ST[j * N + c] > m) m = ST[j * N + c];
            colmax[c] = m;
            double l = 0.0;
            for (int64_t j = 0; j < n; ++j) {
                const double w = (m == -INFINITY) ? 0.0 : exp(ST[j * N + c] - m);
                ST[j * N + c] = w; /* S^T now holds the unnormalised P^T */
                l += w;
            }
            colsum[c] = l;
            for (int64_t j = 0; j < n; ++j)
                if (l > 0.0) ST[j * N + c] /= l;
        }
        /* O^T = V^T P^T, with V^T[c'][j] = K[j][c'] for c' < 512 */
        for (int cv = 0; cv < ORC_DV; ++cv)
            for (int c = 0; c < N; ++c) {
                double acc = 0.0;
                for (int64_t j = 0; j < n; ++j) acc += K[j * ORC_DQK + cv] * ST[j * N + c];
                OT[(int64_t)cv * N + c] = acc;
            }
        /* O = (O^T)^T, scattered back to out[b, i, h, :] */
        for (int c = 0; c < N; ++c) {
            const int i = c / H, h = c % H;
            double *o = out + (((int64_t)b * s_q + i) * H + h) * ORC_DV;
            for (int cv = 0; cv < ORC_DV; ++cv) o[cv] = OT[(int64_t)cv * N + c];
            lse[((int64_t)b * s_q + i) * H + h] =
                colsum[c] > 0.0 ? colmax[c] + log(colsum[c]) : -INFINITY;
        }
        free(K); free(QT); free(ST); free(OT); free(colmax); free(colsum);
    }
    return failed ? ORC_NO_MEMORY : ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Online form: tokens are visited in tiles of `tile` rows; after each tile   */
/*   m_new = max(m_old, max_j s_j)                                            */
/*   l     = exp(m_old - m_new) * l + sum_j exp(s_j - m_new)                  */
/*   acc   = exp(m_old - m_new) * acc + sum_j exp(s_j - m_new) * v_j          */
/* and out = acc / l, lse = m + ln(l) at the end.                              */
/* ------------------------------------------------------------------------ */
int mla_oracle_online(const uint16_t *q, const uint16_t *kv_cache,
                      const int32_t *block_table, const int32_t *seqlens,
                      int B, int s_q, int H, int64_t num_blocks, int max_blocks,
                      double scale, int tile, const int32_t *seq_list, int n_seq_list,
                      double *out, double *lse)
{
    problem_t p = {q, kv_cache, block_table, seqlens, B, s_q, H, num_blocks,
                   max_blocks, scale};
    int rc = check_problem(&p);
    if (rc != ORC_OK) return rc;
    if (tile < 1) return ORC_BAD_ARG;
    const int nb = list_len(&p, seq_list, n_seq_list);
    const int64_t rows = (int64_t)nb * s_q * H;
    int failed = 0;

#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < rows; ++r) {
        const int b = list_at(seq_list, (int)(r / ((int64_t)s_q * H)));
        const int i = (int)((r / H) % s_q);
        const int h = (int)(r % H);
        const int64_t n = visible_tokens(seqlens[b], s_q, i);
        double *o = out + (((int64_t)b * s_q + i) * H + h) * ORC_DV;
        double *ls = lse + ((int64_t)b * s_q + i) * H + h;
        double *s = (double *)malloc((size_t)tile * sizeof(double));
        if (!s) {
            failed = 1;
            continue;
        }
        double qv[ORC_DQK], acc[ORC_DV];
        const uint16_t *qr = query_row(&p, b, i, h);
        for (int d = 0; d < ORC_DQK; ++d) qv[d] = bf16_to_double(qr[d]);
        for (int c = 0; c < ORC_DV; ++c) acc[c] = 0.0;
        double m = -INFINITY, l = 0.0;
        for (int64_t t0 = 0; t0 < n; t0 += tile) {
            const int64_t t1 = t0 + tile < n ? t0 + tile : n;
            double tmax = -INFINITY;
            for (int64_t j = t0; j < t1; ++j) {
                const uint16_t *k = token_row(&p, b, j);
                double dot = 0.0;
                for (int d = 0; d < ORC_DQK; ++d) dot += qv[d] * bf16_to_double(k[d]);
                s[j - t0] = scale * dot;
                if (s[j - t0] > tmax) tmax = s[j - t0];
            }
            const double m_new = tmax > m ? tmax : m;
            const double alpha = (m == -INFINITY) ? 0.0 : exp(m - m_new);
            l *= alpha;
            for (int c = 0; c < ORC_DV; ++c) acc[c] *= alpha;
            for (int64_t j = t0; j < t1; ++j) {
                const uint16_t *k = token_row(&p, b, j);
                const double w = exp(s[j - t0] - m_new);
                l += w;
                for (int c = 0; c < ORC_DV; ++c) acc[c] += w * bf16_to_double(k[c]);
            }
            m = m_new;
        }
        for (int c = 0; c < ORC_DV; ++c) o[c] = (l > 0.0) ? acc[c] / l : 0.0;
        *ls = (l > 0.0) ? m + log(l) : -INFINITY;
        free(s);
    }
    return failed ? ORC_NO_MEMORY : ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Split form: the tokens of sequence b are cut into n_splits contiguous      */
/* ranges [bounds[b][k], bounds[b][k+1]).  Each range gives a partial result  */
/* (O_k normalised over its own visible tokens, lse_k; O_k = 0 and            */
/* lse_k = -inf when it sees none), and the partials are merged:              */
/*   lse = M + ln(sum_k exp(lse_k - M)),  M = max_k lse_k                      */
/*   out = sum_k exp(lse_k - lse) * O_k                                        */
/* bounds is [B][n_splits + 1], non-decreasing, from 0 to seqlen_b.            */
/* ------------------------------------------------------------------------ */
int mla_oracle_split_merge(const uint16_t *q, const uint16_t *kv_cache,
                           const int32_t *block_table, const int32_t *seqlens,
                           int B, int s_q, int H, int64_t num_blocks, int max_blocks,
                           double scale, int n_splits, const int64_t *bounds,
                           double *out, double *lse)
{
    problem_t p = {q, kv_cache, block_table, seqlens, B, s_q, H, num_blocks,
                   max_blocks, scale};
    int rc = check_problem(&p);
    if (rc != ORC_OK) return rc;
    if (n_splits < 1 || !bounds) return ORC_BAD_ARG;
    for (int b = 0; b < B; ++b) {
        const int64_t *bd = bounds + (int64_t)b * (n_splits + 1);
        if (bd[0] != 0 || bd[n_splits] != seqlens[b]) return ORC_BAD_ARG;
        for (int k = 0; k < n_splits; ++k)
            if (bd[k + 1] < bd[k]) return ORC_BAD_ARG;
    }
    const int64_t rows = (int64_t)B * s_q * H;
    int failed = 0;

#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < rows; ++r) {
        const int b = (int)(r / ((int64_t)s_q * H));
        const int i = (int)((r / H) % s_q);
        const int h = (int)(r % H);
        const int64_t n = visible_tokens(seqlens[b], s_q, i);
        const int64_t *bd = bounds + (int64_t)b * (n_splits + 1);
        double *o = out + (((int64_t)b * s_q + i) * H + h) * ORC_DV;
        double *ls = lse + ((int64_t)b * s_q + i) * H + h;
        double *part_o = (double *)malloc((size_t)n_splits * ORC_DV * sizeof(double));
        double *part_lse = (double *)malloc((size_t)n_splits * sizeof(double));
        if (!part_o || !part_lse) {
            failed = 1;
            free(part_o); free(part_lse);
            continue;
        }
        double qv[ORC_DQK];
        const uint16_t *qr = query_row(&p, b, i, h);
        for (int d = 0; d < ORC_DQK; ++d) qv[d] = bf16_to_double(qr[d]);

        for (int k = 0; k < n_splits; ++k) {
            double *po = part_o + (int64_t)k * ORC_DV;
            for (int c = 0; c < ORC_DV; ++c) po[c] = 0.0;
            const int64_t j0 = bd[k];
            const int64_t j1 = bd[k + 1] < n ? bd[k + 1] : n;
            if (j1 <= j0) {
                part_lse[k] = -INFINITY;
                continue;
            }
            double m = -INFINITY;
            for (int64_t j = j0; j < j1; ++j) {
                const uint16_t *kr = token_row(&p, b, j);
                double dot = 0.0;
                for (int d = 0; d < ORC_DQK; ++d) dot += qv[d] * bf16_to_double(kr[d]);
                if (scale * dot > m) m = scale * dot;
            }
            double l = 0.0;
            for (int64_t j = j0; j < j1; ++j) {
                const uint16_t *kr = token_row(&p, b, j);
                double dot = 0.0;
                for (int d = 0; d < ORC_DQK; ++d) dot += qv[d] * bf16_to_double(kr[d]);
                const double w = exp(scale * dot - m);
                l += w;
                for (int c = 0; c < ORC_DV; ++c) po[c] += w * bf16_to_double(kr[c]);
            }
            for (int c = 0; c < ORC_DV; ++c) po[c] /= l;
            part_lse[k] = m + log(l);
        }
        /* merge through the partial log-sum-exps */
        double M = -INFINITY;
        for (int k = 0; k < n_splits; ++k)
            if (part_lse[k] > M) M = part_lse[k];
        for (int c = 0; c < ORC_DV; ++c) o[c] = 0.0;
        if (M == -INFINITY) {
            *ls = -INFINITY;
        } else {
            double sum = 0.0;
            for (int k = 0; k < n_splits; ++k) sum += exp(part_lse[k] - M);
            const double total = M + log(sum);
            for (int k = 0; k < n_splits; ++k) {
                const double w = exp(part_lse[k] - total);
                for (int c = 0; c < ORC_DV; ++c) o[c] += w * part_o[(int64_t)k * ORC_DV + c];
            }
            *ls = total;
        }
        free(part_o); free(part_lse);
    }
    return failed ? ORC_NO_MEMORY : ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Merge of W partial states of the same output rows, each computed over a   */
/* disjoint range of the tokens (the last step of mla_oracle_split_merge,     */
/* taken on its own).  The online softmax of "FlashMLA: compressing the KV    */
/* cache" (jsqmd.com), "compute flow", step 4, carries a running max and a    */
/* running sum from one block of keys to the next; merging whole partial      */
/* results through their log-sum-exps is the same recurrence:                 */
/*   M = max_w lse_w,  lse = M + ln(sum_w exp(lse_w - M)),                    */
/*   out = sum_w exp(lse_w - lse) * out_w,                                    */
/* with out = 0 and lse = -inf when every lse_w is -inf.                      */
/* out_parts is [W][rows][512], lse_parts [W][rows]; out [rows][512].         */
/* ------------------------------------------------------------------------ */
int mla_oracle_merge_states(const double *out_parts, const double *lse_parts, int W, int64_t rows,
                            double *out, double *lse)
{
    if (!out_parts || !lse_parts || !out || !lse || W < 1 || rows < 0) return ORC_BAD_ARG;
    for (int64_t r = 0; r < rows; ++r) {
        double M = -INFINITY;
        for (int w = 0; w < W; ++w) {
            const double x = lse_parts[(int64_t)w * rows + r];
            if (x > M) M = x;
        }
        double *o = out + r * ORC_DV;
        for (int c = 0; c < ORC_DV; ++c) o[c] = 0.0;
        if (M == -INFINITY) {
            lse[r] = -INFINITY;
            continue;
        }
        double sum = 0.0;
        for (int w = 0; w < W; ++w) sum += exp(lse_parts[(int64_t)w * rows + r] - M);
        const double total = M + log(sum);
        for (int w = 0; w < W; ++w) {
            const double wt = exp(lse_parts[(int64_t)w * rows + r] - total);
            const double *po = out_parts + ((int64_t)w * rows + r) * ORC_DV;
            for (int c = 0; c < ORC_DV; ++c) o[c] += wt * po[c];
        }
        lse[r] = total;
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* FP8 cache.  The juejin.cn "FlashMLA" post, section 5 (FlashMLA against     */
/* FlashAttention), says FlashMLA runs in mixed precision such as FP8 and     */
/* BF16; it fixes no format.  The reading taken here: every cached value is  */
/* an e4m3 code with one fp32 scale per cached token, so token j's row is     */
/*   k_j[d] = e4m3(code[blk][j % 64][d]) * kscale[blk][j % 64],  d < 576,     */
/* and the queries stay bf16.  e4m3 is the OCP FP8 E4M3 format as CUDA's      */
/* __nv_fp8_e4m3 and torch's float8_e4m3fn hold it: 1 sign, 4 exponent bits  */
/* (bias 7), 3 mantissa bits, exponent 0 subnormal (mantissa * 2^-9), no     */
/* infinities, S.1111.111 NaN.  Decoding, and the product with the scale,    */
/* are exact in double.                                                       */
/* ------------------------------------------------------------------------ */
double mla_oracle_e4m3_to_double(uint8_t code)
{
    const int sign = code >> 7, ex = (code >> 3) & 15, mant = code & 7;
    double mag;
    if (ex == 15 && mant == 7) return NAN;
    if (ex == 0) mag = ldexp((double)mant, -9);
    else mag = ldexp(1.0 + mant / 8.0, ex - 7);
    return sign ? -mag : mag;
}

int mla_oracle_direct_fp8(const uint16_t *q, const uint8_t *kv_codes, const float *kv_scale,
                          const int32_t *block_table, const int32_t *seqlens,
                          int B, int s_q, int H, int64_t num_blocks, int max_blocks,
                          double scale, double *out, double *lse)
{
    if (!q || !kv_codes || !kv_scale || !block_table || !seqlens || !out || !lse) return ORC_BAD_ARG;
    if (B < 0 || s_q < 1 || H < 1 || max_blocks < 1 || num_blocks < 0) return ORC_BAD_ARG;
    double table[256];
    for (int c = 0; c < 256; ++c) table[c] = mla_oracle_e4m3_to_double((uint8_t)c);
    const int64_t rows = (int64_t)B * s_q * H;
    int failed = 0;

#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < rows; ++r) {
        const int b = (int)(r / ((int64_t)s_q * H));
        const int i = (int)((r / H) % s_q);
        const int h = (int)(r % H);
        const int64_t n = visible_tokens(seqlens[b] < 0 ? 0 : seqlens[b], s_q, i);
        double *o = out + r * ORC_DV;
        for (int c = 0; c < ORC_DV; ++c) o[c] = 0.0;
        if (n == 0) {
            lse[r] = -INFINITY;
            continue;
        }
        double *row = (double *)malloc((size_t)n * ORC_DQK * sizeof(double));
        double *sc = (double *)malloc((size_t)n * sizeof(double));
        if (!row || !sc) {
            failed = 1;
            free(row); free(sc);
            continue;
        }
        /* dequantised rows of the visible tokens, found through the page table */
        int bad = 0;
        for (int64_t j = 0; j < n && !bad; ++j) {
            const int64_t pg = j / ORC_PAGE;
            const int32_t blk = pg < max_blocks ? block_table[(int64_t)b * max_blocks + pg] : -1;
            if (blk < 0 || (int64_t)blk >= num_blocks) { bad = 1; break; }
            const int64_t tok = (int64_t)blk * ORC_PAGE + j % ORC_PAGE;
            const double ks = (double)kv_scale[tok];
            for (int d = 0; d < ORC_DQK; ++d) row[j * ORC_DQK + d] = table[kv_codes[tok * ORC_DQK + d]] * ks;
        }
        if (bad) {
            failed = 2;
            free(row); free(sc);
            continue;
        }
        const uint16_t *qr = q + r * ORC_DQK;
        double top = -INFINITY;
        for (int64_t j = 0; j < n; ++j) {
            double acc = 0.0;
            for (int d = 0; d < ORC_DQK; ++d) acc += bf16_to_double(qr[d]) * row[j * ORC_DQK + d];
            sc[j] = scale * acc;
            if (sc[j] > top) top = sc[j];
        }
        double total = 0.0;
        for (int64_t j = 0; j < n; ++j) {
            const double wj = exp(sc[j] - top);
            total += wj;
            for (int c = 0; c < ORC_DV; ++c) o[c] += wj * row[j * ORC_DQK + c];
        }
        for (int c = 0; c < ORC_DV; ++c) o[c] /= total;
        lse[r] = top + log(total);
        free(row); free(sc);
    }
    return failed == 2 ? ORC_BAD_BLOCK : failed ? ORC_NO_MEMORY : ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Non-absorbed form.  "FlashMLA: compressing the KV cache to one eighth"    */
/* (jsqmd.com), "MLA compression principle" and "FlashMLA compute flow",     */
/* steps 1-5: the cache holds a compressed latent row per token, and each    */
/* KV tile is decompressed when it is used -- K_tile = C_KV_tile W_UK,       */
/* V_tile = C_KV_tile W_UV -- before S = Q K^T, the online softmax and       */
/* O += softmax(S) V.  With the latent rows of the absorbed form (512 latent */
/* columns c, then 64 rope columns) and per-head matrices:                   */
/*   k_j[e]        = sum_{c<512} C_j[c] * w_uk[h][e][c]     e < 128          */
/*   k_j[128 + r]  = C_j[512 + r]                           r < 64 (rope)    */
/*   v_j[e]        = sum_{c<512} C_j[c] * w_uv[h][e][c]     e < 128          */
/*   s_j           = scale * sum_{d<192} q[b,i,h,d] * k_j[d]                 */
/*   out[e]        = sum_j softmax(s)_j * v_j[e],  lse = ln sum_j exp(s_j)   */
/* over the same visible tokens as the absorbed form.  Readings: the rope    */
/* columns are cached already rotated and are shared by every head (the      */
/* absorbed form's layout), so no rotation happens here; the up-projection   */
/* matrices are stored as [H][128][512] (row e of head h holds the latent    */
/* coefficients of output dimension e).  Everything in fp64, decompressed    */
/* per token without any intermediate rounding.                              */
/*   q     [B, s_q, H, 192] bf16 (128 decompressed-key columns, then rope)   */
/*   w_uk, w_uv  [H, 128, 512] bf16                                          */
/*   out   [B, s_q, H, 128], lse [B, s_q, H] (fp64)                          */
/* ------------------------------------------------------------------------ */
int mla_oracle_naive(const uint16_t *q, const uint16_t *kv_cache, const uint16_t *w_uk, const uint16_t *w_uv,
                     const int32_t *block_table, const int32_t *seqlens,
                     int B, int s_q, int H, int64_t num_blocks, int max_blocks,
                     double scale, const int32_t *seq_list, int n_seq_list,
                     double *out, double *lse)
{
    /* q is not a 576-wide row here: the page-table check only needs the
     * cache, so the problem record carries the cache with a stand-in q */
    problem_t p = {kv_cache, kv_cache, block_table, seqlens, B, s_q, H, num_blocks, max_blocks, scale};
    if (!q || !w_uk || !w_uv) return ORC_BAD_ARG;
    int rc = check_problem(&p);
    if (rc != ORC_OK) return rc;
    const int nb = list_len(&p, seq_list, n_seq_list);
    const int64_t rows = (int64_t)nb * s_q * H;
    const int dq = ORC_DNOPE + ORC_DROPE;
    int failed = 0;

#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < rows; ++r) {
        const int b = list_at(seq_list, (int)(r / ((int64_t)s_q * H)));
        const int i = (int)((r / H) % s_q);
        const int h = (int)(r % H);
        const int64_t n = visible_tokens(seqlens[b], s_q, i);
        double *o = out + (((int64_t)b * s_q + i) * H + h) * ORC_DNOPE;
        double *ls = lse + ((int64_t)b * s_q + i) * H + h;
        for (int e = 0; e < ORC_DNOPE; ++e) o[e] = 0.0;
        if (n == 0) {
            *ls = -INFINITY;
            continue;
        }
        double *s = (double *)malloc((size_t)n * sizeof(double));
        double *v = (double *)malloc((size_t)n * ORC_DNOPE * sizeof(double));
        double *wk = (double *)malloc((size_t)ORC_DNOPE * ORC_DV * sizeof(double));
        double *wv = (double *)malloc((size_t)ORC_DNOPE * ORC_DV * sizeof(double));
        if (!s || !v || !wk || !wv) {
            failed = 1;
            free(s); free(v); free(wk); free(wv);
            continue;
        }
        const uint16_t *wkh = w_uk + (int64_t)h * ORC_DNOPE * ORC_DV;
        const uint16_t *wvh = w_uv + (int64_t)h * ORC_DNOPE * ORC_DV;
        for (int64_t t = 0; t < (int64_t)ORC_DNOPE * ORC_DV; ++t) {
            wk[t] = bf16_to_double(wkh[t]);
            wv[t] = bf16_to_double(wvh[t]);
        }
        double qv[ORC_DNOPE + ORC_DROPE];
        const uint16_t *qr = q + (((int64_t)b * s_q + i) * H + h) * dq;
        for (int d = 0; d < dq; ++d) qv[d] = bf16_to_double(qr[d]);

        /* per token: decompress k and v from the latent row, score */
        double m = -INFINITY;
        for (int64_t j = 0; j < n; ++j) {
            const uint16_t *row = token_row(&p, b, j);
            double c[ORC_DV];
            for (int x = 0; x < ORC_DV; ++x) c[x] = bf16_to_double(row[x]);
            double dot = 0.0;
            for (int e = 0; e < ORC_DNOPE; ++e) {
                double ke = 0.0, ve = 0.0;
                for (int x = 0; x < ORC_DV; ++x) {
                    ke += c[x] * wk[(int64_t)e * ORC_DV + x];
                    ve += c[x] * wv[(int64_t)e * ORC_DV + x];
                }
                dot += qv[e] * ke;
                v[j * ORC_DNOPE + e] = ve;
            }
            for (int x = 0; x < ORC_DROPE; ++x) dot += qv[ORC_DNOPE + x] * bf16_to_double(row[ORC_DV + x]);
            s[j] = scale * dot;
            if (s[j] > m) m = s[j];
        }
        double l = 0.0;
        for (int64_t j = 0; j < n; ++j) {
            const double w = exp(s[j] - m);
            l += w;
            for (int e = 0; e < ORC_DNOPE; ++e) o[e] += w * v[j * ORC_DNOPE + e];
        }
        for (int e = 0; e < ORC_DNOPE; ++e) o[e] /= l;
        *ls = m + log(l);
        free(s); free(v); free(wk); free(wv);
    }
    return failed ? ORC_NO_MEMORY : ORC_OK;
}
