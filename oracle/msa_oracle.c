/*
 * MSA oracle: plain, slow, float64 CPU definitions of the MiniMax Sparse Attention hot path.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product library links, loads or calls this file.
 * Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline leg may use it.
 *
 * Every function restates a definition from the source pages, in the pages' notation:
 *   - index score   S^{idx,(r)}_{i,j} = Q^{idx,(r)}_i . K^{idx}_j / sqrt(d_idx)
 *       ("MSA Indexer vs DSA Lightning Indexer", section 2.1 scoring function;
 *        "KL alignment in MSA", section 2.1 student)
 *   - block max     M_{i,b} = max_{j in B_b, j <= i} S_{i,j}
 *       ("MSA Indexer vs DSA Lightning Indexer", section 2.2)
 *   - selection     I_i = TopK_b(M_{i,b}, k), plus the query's local block always included
 *       (same page, section 2.2, last sentence; MSA blog, "how the index branch selects blocks")
 *   - attention     o = sum_{s in S} softmax_S(q.k_s / sqrt d) v_s, exact on the selected set
 *       ("2.4 training-native sparse", eq (2))
 *   - teacher       P^{(r)}_{i,j} = (1/G) sum_{l in H_r} softmax_J(S^{(l)})_j  (probabilities averaged)
 *       ("KL alignment in MSA", section 2.2)
 *   - student       P^{idx,(r)}_{i,j} = softmax_J(S^{idx,(r)})_j on the same token set J
 *       ("KL alignment in MSA", section 2.1)
 *   - loss          L_KL = 1/(N H_kv) sum_i sum_r KL(stopgrad(P_i^{(r)}) || P_i^{idx,(r)})
 *       ("KL alignment in MSA", section 3)
 *   - logit grad    dKL/dz_j = P^idx_j - P_j ("KL alignment in MSA", section 3, key gradient)
 *   - attention bwd dL/dz_j = alpha_j g.(v_j - o) on the fixed selected set, zero elsewhere
 *       ("2.4 training-native sparse", section 2.2, eq (11))
 *   - FP8 keys      selector keys kept in bf16 for training, quantised to FP8 for serving
 *       ("4.1.1 supervision and joint training", section 2; "MSA Indexer vs DSA Lightning
 *        Indexer", section 3.1: the indexer can run in FP8). Reading: e4m3 with one fp32 scale
 *        per row, scale = max|x| / 448, codes rounded to nearest (ties to even), saturated.
 *   - cutoff margin Delta_i = r_(k) - r_(k+1) ("4.1.1 supervision and joint training", eq (9))
 *
 * Readings of points the pages leave open (each is listed in the design notes):
 *   - local_mode 0 (the reading the GPU library implements): Top-k runs over the query's
 *     complete past blocks {0..b_i-1}; the local block b_i is added on top, so a row holds
 *     min(k, b_i) + 1 blocks. local_mode 1: the local block takes one of the k slots (Top-(k-1)
 *     over past blocks, plus local). local_mode 2: Top-k over all blocks 0..b_i (the local
 *     block ranked by its causal max), then the local block is added if it was not chosen.
 *   - ties in M go to the lower block id.
 *   - the loss is divided by B*N*H_kv (the pages' 1/(N H_kv) per sequence, averaged over a batch);
 *     the returned gradients are grad_scale times the gradient of that loss.
 *   - the teacher and the student have temperature 1.
 *
 * Pins (tests/test_oracle_pins.py): the pages' worked examples (recall/coverage, the eq (11)
 * two-position example), the deletion and partition-merge identities, dense causal attention when
 * k covers every block (against torch SDPA in float64), brute force of the selection, LSE_idx,
 * sparse attention and KL on tiny inputs, finite differences of the KL gradient, KL = 0 when the
 * student equals the teacher, decode = last prefill row, the e4m3 code values against the format's
 * table in torch, nearest-even rounding, and FP8 decode = bf16 decode on inputs that are already
 * e4m3 values with power-of-two row scales. Which of the three local-block readings
 * the method uses is not fixed by any page: that choice is parity unpinned (the code of each
 * reading is pinned, the choice between them is not).
 *
 * Inputs are read either as float64 or as raw bfloat16 bits (widened exactly to float64);
 * every sum, exp and log runs in float64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_F64 0
#define ORC_BF16 1

typedef struct {
    int B, N, H_q, H_kv, d, d_idx, block_k, topk, local_mode;
    double scale;     /* 0 -> 1/sqrt(d)     */
    double scale_idx; /* 0 -> 1/sqrt(d_idx) */
} orc_dims;

/* one input element as float64 */
static double ld(const void *p, int ty, size_t i) {
    if (ty == ORC_F64) return ((const double *)p)[i];
    uint32_t u = (uint32_t)((const uint16_t *)p)[i] << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double eff_scale(const orc_dims *D) { return D->scale != 0.0 ? D->scale : 1.0 / sqrt((double)D->d); }
static double eff_scale_idx(const orc_dims *D) {
    return D->scale_idx != 0.0 ? D->scale_idx : 1.0 / sqrt((double)D->d_idx);
}

/* ---------------------------------------------------------------------------------------------
 * Index score of one query index head against tokens 0..n_tok-1 of one sequence's shared key head.
 * q_off: element offset of Q^{idx,(r)}_i; k_base: element offset of K^{idx}_0 of the sequence.
 * -------------------------------------------------------------------------------------------- */
static void index_scores(const orc_dims *D, const void *q_idx, const void *k_idx, int ty, size_t q_off,
                         size_t k_base, int n_tok, double *s) {
    const double sc = eff_scale_idx(D);
    for (int j = 0; j < n_tok; ++j) {
        double acc = 0.0;
        for (int c = 0; c < D->d_idx; ++c)
            acc += ld(q_idx, ty, q_off + c) * ld(k_idx, ty, k_base + (size_t)j * D->d_idx + c);
        s[j] = acc * sc;
    }
}

/* M[b] = max over tokens j of block b with j <= i, for b = 0..i/block_k. */
static void block_max(const orc_dims *D, const double *s, int i, double *M) {
    const int bi = i / D->block_k;
    for (int b = 0; b <= bi; ++b) {
        double m = -INFINITY;
        int j1 = (b + 1) * D->block_k - 1;
        if (j1 > i) j1 = i;
        for (int j = b * D->block_k; j <= j1; ++j)
            if (s[j] > m) m = s[j];
        M[b] = m;
    }
}

/* order: higher M first, equal M -> lower block id first */
static int ranks_before(const double *M, int a, int b) { return M[a] > M[b] || (M[a] == M[b] && a < b); }

static int cmp_int(const void *x, const void *y) {
    int a = *(const int *)x, b = *(const int *)y;
    return (a > b) - (a < b);
}

/*
 * Block selection for query i given its block maxima M[0..b_i]. Writes topk+1 ids, ascending,
 * padded with -1. Returns the number of selected blocks. *margin receives the cutoff margin
 * r_(k) - r_(k+1) over the ranked candidates (+inf when every candidate is taken).
 */
static int select_blocks(const orc_dims *D, const double *M, int i, int32_t *sel, double *margin) {
    const int bi = i / D->block_k;
    int k = D->topk;
    int ncand = bi; /* candidates 0..bi-1 */
    if (D->local_mode == 1) k = D->topk - 1;
    if (D->local_mode == 2) ncand = bi + 1;
    if (k < 0) k = 0;
    int *order = (int *)malloc(sizeof(int) * (size_t)(ncand > 0 ? ncand : 1));
    for (int c = 0; c < ncand; ++c) order[c] = c;
    /* insertion sort by (M desc, id asc): plain and obviously correct */
    for (int x = 1; x < ncand; ++x) {
        int v = order[x], y = x - 1;
        while (y >= 0 && ranks_before(M, v, order[y])) {
            order[y + 1] = order[y];
            --y;
        }
        order[y + 1] = v;
    }
    int take = k < ncand ? k : ncand;
    *margin = (ncand > k && k > 0) ? M[order[k - 1]] - M[order[k]] : INFINITY;
    int n = 0, has_local = 0;
    for (int x = 0; x < take; ++x) {
        sel[n++] = order[x];
        if (order[x] == bi) has_local = 1;
    }
    if (!has_local) sel[n++] = bi;
    qsort(sel, (size_t)n, sizeof(int32_t), cmp_int);
    for (int x = n; x < D->topk + 1; ++x) sel[x] = -1;
    free(order);
    return n;
}

/* Causal token set J of query i for the selected blocks (ascending). Returns |J|. */
static int token_set(const orc_dims *D, const int32_t *sel, int nslots, int i, int32_t *J) {
    int n = 0;
    for (int x = 0; x < nslots; ++x) {
        int b = sel[x];
        if (b < 0) continue;
        int j1 = (b + 1) * D->block_k - 1;
        if (j1 > i) j1 = i;
        for (int j = b * D->block_k; j <= j1; ++j) J[n++] = j;
    }
    return n;
}

/*
 * Exact softmax attention of one query vector over an explicit token list ("2.4" eq (2)).
 * q_off: offset of the query vector; kv_base: offset of token 0's vector for this KV head;
 * kv_stride: elements between consecutive tokens. Writes o[d] and the log-sum-exp of the logits.
 */
static void attend_tokens(int d, double scale, const void *q, const void *k, const void *v, int ty, size_t q_off,
                          size_t kv_base, size_t kv_stride, const int32_t *J, int nJ, double *z, double *o,
                          double *lse) {
    double m = -INFINITY;
    for (int t = 0; t < nJ; ++t) {
        double acc = 0.0;
        size_t ko = kv_base + (size_t)J[t] * kv_stride;
        for (int c = 0; c < d; ++c) acc += ld(q, ty, q_off + c) * ld(k, ty, ko + c);
        z[t] = acc * scale;
        if (z[t] > m) m = z[t];
    }
    double l = 0.0;
    for (int t = 0; t < nJ; ++t) l += exp(z[t] - m);
    double L = m + log(l);
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    for (int t = 0; t < nJ; ++t) {
        double p = exp(z[t] - L);
        size_t vo = kv_base + (size_t)J[t] * kv_stride;
        for (int c = 0; c < d; ++c) o[c] += p * ld(v, ty, vo + c);
    }
    *lse = L;
}

/* ============================== exported entry points ======================================= */

/* Index scores of row (b, i), group r: s[0..i]. */
void orc_index_scores_row(const orc_dims *D, const void *q_idx, const void *k_idx, int ty, int b, int i, int r,
                          double *s) {
    size_t q_off = (((size_t)b * D->N + i) * D->H_kv + r) * D->d_idx;
    size_t k_base = (size_t)b * D->N * D->d_idx;
    index_scores(D, q_idx, k_idx, ty, q_off, k_base, i + 1, s);
}

/* Block maxima of row i from its scores s[0..i]. */
void orc_block_max_row(const orc_dims *D, const double *s, int i, double *M) { block_max(D, s, i, M); }

/* Selection from given block maxima (exposed for the pins). */
int orc_select_from_max(const orc_dims *D, const double *M, int i, int32_t *sel, double *margin) {
    return select_blocks(D, M, i, sel, margin);
}

/*
 * Index Top-k for a list of rows (flattened b*N+i; rows == NULL means all B*N rows).
 * blocks: [nrows, H_kv, topk+1]; margin: [nrows, H_kv]; lse_idx: [nrows, H_kv] or NULL, the
 * log-sum-exp of the index scores over the selected causal token set J.
 */
int orc_index_topk(const orc_dims *D, const void *q_idx, const void *k_idx, int ty, const int64_t *rows,
                   int64_t nrows, int32_t *blocks, double *margin, double *lse_idx) {
    if (!rows) nrows = (int64_t)D->B * D->N;
    const int K1 = D->topk + 1;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)D->N);
        double *M = (double *)malloc(sizeof(double) * (size_t)(D->N / D->block_k + 2));
        int32_t *J = (int32_t *)malloc(sizeof(int32_t) * (size_t)D->N);
#pragma omp for schedule(dynamic, 4)
        for (int64_t x = 0; x < nrows; ++x) {
            int64_t row = rows ? rows[x] : x;
            int b = (int)(row / D->N), i = (int)(row % D->N);
            for (int r = 0; r < D->H_kv; ++r) {
                orc_index_scores_row(D, q_idx, k_idx, ty, b, i, r, s);
                block_max(D, s, i, M);
                int32_t *sel = blocks + ((size_t)x * D->H_kv + r) * K1;
                select_blocks(D, M, i, sel, &margin[(size_t)x * D->H_kv + r]);
                if (lse_idx) {
                    int nJ = token_set(D, sel, K1, i, J);
                    double m = -INFINITY, l = 0.0;
                    for (int t = 0; t < nJ; ++t)
                        if (s[J[t]] > m) m = s[J[t]];
                    for (int t = 0; t < nJ; ++t) l += exp(s[J[t]] - m);
                    lse_idx[(size_t)x * D->H_kv + r] = m + log(l);
                }
            }
        }
        free(s);
        free(M);
        free(J);
    }
    return 0;
}

/*
 * Sparse attention for a list of rows, given the full selection tensor blocks [B, N, H_kv, topk+1].
 * out: [nrows, H_q, d]; lse: [nrows, H_q].
 */
int orc_sparse_attn(const orc_dims *D, const void *q, const void *k, const void *v, int ty, const int32_t *blocks,
                    const int64_t *rows, int64_t nrows, double *out, double *lse) {
    if (!rows) nrows = (int64_t)D->B * D->N;
    const int K1 = D->topk + 1, G = D->H_q / D->H_kv;
    const double sc = eff_scale(D);
#pragma omp parallel
    {
        int32_t *J = (int32_t *)malloc(sizeof(int32_t) * (size_t)D->N);
        double *z = (double *)malloc(sizeof(double) * (size_t)D->N);
#pragma omp for schedule(dynamic, 4)
        for (int64_t x = 0; x < nrows; ++x) {
            int64_t row = rows ? rows[x] : x;
            int b = (int)(row / D->N), i = (int)(row % D->N);
            for (int h = 0; h < D->H_q; ++h) {
                int r = h / G;
                const int32_t *sel = blocks + (((size_t)b * D->N + i) * D->H_kv + r) * K1;
                int nJ = token_set(D, sel, K1, i, J);
                size_t q_off = (((size_t)b * D->N + i) * D->H_q + h) * D->d;
                size_t kv_base = ((size_t)b * D->N * D->H_kv + r) * D->d;
                attend_tokens(D->d, sc, q, k, v, ty, q_off, kv_base, (size_t)D->H_kv * D->d, J, nJ, z,
                              out + ((size_t)x * D->H_q + h) * D->d, lse + (size_t)x * D->H_q + h);
            }
        }
        free(J);
        free(z);
    }
    return 0;
}

/*
 * Backward of the sparse attention with the selection held fixed ("2.4" page, section 2.2, eq (11):
 * with the set fixed, selected attention is ordinary attention on it, and positions outside the set
 * get no gradient). For each (b, i, h) with token set J, alpha = softmax_J(z), z_j = scale q.k_j,
 * o = sum_j alpha_j v_j and upstream gradient g = dout[b,i,h]:
 *   dL/dz_j = alpha_j g.(v_j - o)
 *   dq     = scale sum_j dL/dz_j k_j
 *   dk_j  += scale dL/dz_j q          (over every (i, h) of the group whose set holds j)
 *   dv_j  += alpha_j g
 * dq [B,N,H_q,d]; dk, dv [B,N,H_kv,d]; all float64, overwritten. Parallel over (b, group): each
 * owns its KV head's dk/dv rows and its heads' dq rows.
 */
int orc_sparse_attn_bwd(const orc_dims *D, const void *q, const void *k, const void *v, const void *dout, int ty,
                        const int32_t *blocks, double *dq, double *dk, double *dv) {
    const int K1 = D->topk + 1, G = D->H_q / D->H_kv;
    const double sc = eff_scale(D);
    memset(dq, 0, sizeof(double) * (size_t)D->B * D->N * D->H_q * D->d);
    memset(dk, 0, sizeof(double) * (size_t)D->B * D->N * D->H_kv * D->d);
    memset(dv, 0, sizeof(double) * (size_t)D->B * D->N * D->H_kv * D->d);
#pragma omp parallel
    {
        int32_t *J = (int32_t *)malloc(sizeof(int32_t) * (size_t)D->N);
        double *z = (double *)malloc(sizeof(double) * (size_t)D->N);
        double *o = (double *)malloc(sizeof(double) * (size_t)D->d);
#pragma omp for schedule(dynamic, 1)
        for (int x = 0; x < D->B * D->H_kv; ++x) {
            const int b = x / D->H_kv, r = x % D->H_kv;
            const size_t kv_base = ((size_t)b * D->N * D->H_kv + r) * D->d, kv_stride = (size_t)D->H_kv * D->d;
            for (int i = 0; i < D->N; ++i) {
                const int32_t *sel = blocks + (((size_t)b * D->N + i) * D->H_kv + r) * K1;
                const int nJ = token_set(D, sel, K1, i, J);
                for (int h = r * G; h < (r + 1) * G; ++h) {
                    const size_t q_off = (((size_t)b * D->N + i) * D->H_q + h) * D->d;
                    double lse;
                    attend_tokens(D->d, sc, q, k, v, ty, q_off, kv_base, kv_stride, J, nJ, z, o, &lse);
                    double go = 0.0;
                    for (int c = 0; c < D->d; ++c) go += ld(dout, ty, q_off + c) * o[c];
                    for (int t = 0; t < nJ; ++t) {
                        const size_t kvo = kv_base + (size_t)J[t] * kv_stride;
                        const double alpha = exp(z[t] - lse);
                        double gv = 0.0;
                        for (int c = 0; c < D->d; ++c) gv += ld(dout, ty, q_off + c) * ld(v, ty, kvo + c);
                        const double dz = alpha * (gv - go);
                        for (int c = 0; c < D->d; ++c) {
                            dq[q_off + c] += sc * dz * ld(k, ty, kvo + c);
                            dk[kvo + c] += sc * dz * ld(q, ty, q_off + c);
                            dv[kvo + c] += alpha * ld(dout, ty, q_off + c);
                        }
                    }
                }
            }
        }
        free(J);
        free(z);
        free(o);
    }
    return 0;
}

/* dq rows only (same definition as orc_sparse_attn_bwd): dq of row (b, i) depends on that row's set
 * alone, so sampled rows of a large problem can be checked. rows: flat b*N + i; dq [nrows, H_q, d]. */
int orc_sparse_attn_bwd_dq_rows(const orc_dims *D, const void *q, const void *k, const void *v, const void *dout,
                                int ty, const int32_t *blocks, const int64_t *rows, int64_t nrows, double *dq) {
    const int K1 = D->topk + 1, G = D->H_q / D->H_kv;
    const double sc = eff_scale(D);
#pragma omp parallel
    {
        int32_t *J = (int32_t *)malloc(sizeof(int32_t) * (size_t)D->N);
        double *z = (double *)malloc(sizeof(double) * (size_t)D->N);
        double *o = (double *)malloc(sizeof(double) * (size_t)D->d);
#pragma omp for schedule(dynamic, 1)
        for (int64_t x = 0; x < nrows; ++x) {
            const int b = (int)(rows[x] / D->N), i = (int)(rows[x] % D->N);
            for (int h = 0; h < D->H_q; ++h) {
                const int r = h / G;
                const int32_t *sel = blocks + (((size_t)b * D->N + i) * D->H_kv + r) * K1;
                const int nJ = token_set(D, sel, K1, i, J);
                const size_t q_off = (((size_t)b * D->N + i) * D->H_q + h) * D->d;
                const size_t kv_base = ((size_t)b * D->N * D->H_kv + r) * D->d, kv_stride = (size_t)D->H_kv * D->d;
                double lse;
                attend_tokens(D->d, sc, q, k, v, ty, q_off, kv_base, kv_stride, J, nJ, z, o, &lse);
                double go = 0.0;
                for (int c = 0; c < D->d; ++c) go += ld(dout, ty, q_off + c) * o[c];
                double *dqr = dq + ((size_t)x * D->H_q + h) * D->d;
                for (int c = 0; c < D->d; ++c) dqr[c] = 0.0;
                for (int t = 0; t < nJ; ++t) {
                    const size_t kvo = kv_base + (size_t)J[t] * kv_stride;
                    const double alpha = exp(z[t] - lse);
                    double gv = 0.0;
                    for (int c = 0; c < D->d; ++c) gv += ld(dout, ty, q_off + c) * ld(v, ty, kvo + c);
                    const double dz = alpha * (gv - go);
                    for (int c = 0; c < D->d; ++c) dqr[c] += sc * dz * ld(k, ty, kvo + c);
                }
            }
        }
        free(J);
        free(z);
        free(o);
    }
    return 0;
}

/* Attention of one query vector over an explicit token list (exposed for the pins). */
void orc_attend_tokens(int d, double scale, const double *q, const double *k, const double *v, const int32_t *J,
                       int nJ, double *o, double *lse) {
    double *z = (double *)malloc(sizeof(double) * (size_t)(nJ > 0 ? nJ : 1));
    attend_tokens(d, scale, q, k, v, ORC_F64, 0, 0, (size_t)d, J, nJ, z, o, lse);
    free(z);
}

/*
 * KL alignment and its index gradients for a list of rows, given the selection blocks
 * [B, N, H_kv, topk+1]. The teacher's per-head log-sum-exp is computed here from its definition.
 *   kl_rows: [nrows, H_kv]  KL(P || P_idx) per (row, group), not yet normalised
 *   dq_idx:  [nrows, H_kv, d_idx]
 *   dk_idx:  [B, N, d_idx], accumulated (+=) over the given rows
 *   loss:    sum over the given rows of KL / (B N H_kv)
 * Gradients are grad_scale * d(loss)/d(q_idx, k_idx) with the selection held fixed.
 */
int orc_kl(const orc_dims *D, const void *q, const void *k, const void *q_idx, const void *k_idx, int ty,
           const int32_t *blocks, double grad_scale, const int64_t *rows, int64_t nrows, double *kl_rows,
           double *dq_idx, double *dk_idx, double *loss) {
    if (!rows) nrows = (int64_t)D->B * D->N;
    const int K1 = D->topk + 1, G = D->H_q / D->H_kv;
    const double sc = eff_scale(D), sci = eff_scale_idx(D);
    const double norm = 1.0 / ((double)D->B * D->N * D->H_kv);
    const size_t dk_len = (size_t)D->B * D->N * D->d_idx;
    double total = 0.0;
#pragma omp parallel reduction(+ : total)
    {
        int32_t *J = (int32_t *)malloc(sizeof(int32_t) * (size_t)D->N);
        double *z = (double *)malloc(sizeof(double) * (size_t)D->N);
        double *P = (double *)malloc(sizeof(double) * (size_t)D->N);
        double *s = (double *)malloc(sizeof(double) * (size_t)D->N);
        double *dk_priv = (double *)calloc(dk_len, sizeof(double));
#pragma omp for schedule(dynamic, 4)
        for (int64_t x = 0; x < nrows; ++x) {
            int64_t row = rows ? rows[x] : x;
            int b = (int)(row / D->N), i = (int)(row % D->N);
            for (int r = 0; r < D->H_kv; ++r) {
                const int32_t *sel = blocks + (((size_t)b * D->N + i) * D->H_kv + r) * K1;
                int nJ = token_set(D, sel, K1, i, J);
                size_t kv_base = ((size_t)b * D->N * D->H_kv + r) * D->d;
                /* teacher: per-head softmax over J, averaged in probability space */
                for (int t = 0; t < nJ; ++t) P[t] = 0.0;
                for (int h = r * G; h < (r + 1) * G; ++h) {
                    size_t q_off = (((size_t)b * D->N + i) * D->H_q + h) * D->d;
                    double m = -INFINITY;
                    for (int t = 0; t < nJ; ++t) {
                        double acc = 0.0;
                        size_t ko = kv_base + (size_t)J[t] * D->H_kv * D->d;
                        for (int c = 0; c < D->d; ++c) acc += ld(q, ty, q_off + c) * ld(k, ty, ko + c);
                        z[t] = acc * sc;
                        if (z[t] > m) m = z[t];
                    }
                    double l = 0.0;
                    for (int t = 0; t < nJ; ++t) l += exp(z[t] - m);
                    double L = m + log(l);
                    for (int t = 0; t < nJ; ++t) P[t] += exp(z[t] - L) / G;
                }
                /* student: index softmax over the same J */
                size_t qi_off = (((size_t)b * D->N + i) * D->H_kv + r) * D->d_idx;
                size_t ki_base = (size_t)b * D->N * D->d_idx;
                double m = -INFINITY;
                for (int t = 0; t < nJ; ++t) {
                    double acc = 0.0;
                    for (int c = 0; c < D->d_idx; ++c)
                        acc += ld(q_idx, ty, qi_off + c) * ld(k_idx, ty, ki_base + (size_t)J[t] * D->d_idx + c);
                    s[t] = acc * sci;
                    if (s[t] > m) m = s[t];
                }
                double l = 0.0;
                for (int t = 0; t < nJ; ++t) l += exp(s[t] - m);
                double Lidx = m + log(l);
                /* KL(P || P_idx) = sum_j P_j (log P_j - log P_idx_j) */
                double kl = 0.0;
                for (int t = 0; t < nJ; ++t)
                    if (P[t] > 0.0) kl += P[t] * (log(P[t]) - (s[t] - Lidx));
                kl_rows[(size_t)x * D->H_kv + r] = kl;
                total += kl * norm;
                /* logit gradient (P_idx - P), chained through s_j = sci * q_idx . k_idx_j */
                double *dq = dq_idx + ((size_t)x * D->H_kv + r) * D->d_idx;
                for (int c = 0; c < D->d_idx; ++c) dq[c] = 0.0;
                for (int t = 0; t < nJ; ++t) {
                    double g = grad_scale * norm * (exp(s[t] - Lidx) - P[t]);
                    size_t ko = ki_base + (size_t)J[t] * D->d_idx;
                    for (int c = 0; c < D->d_idx; ++c) {
                        dq[c] += g * sci * ld(k_idx, ty, ko + c);
                        dk_priv[ko + c] += g * sci * ld(q_idx, ty, qi_off + c);
                    }
                }
            }
        }
#pragma omp critical
        {
            for (size_t e = 0; e < dk_len; ++e) dk_idx[e] += dk_priv[e];
        }
        free(J);
        free(z);
        free(P);
        free(s);
        free(dk_priv);
    }
    *loss = total;
    return 0;
}

/*
 * One decode step: for each sequence b, the new token sits at position L-1 with L = cache_len[b]
 * (its K, V and K_idx are already in the caches). The step is the prefill definition applied to
 * that one row over the cache. D->N is the cache capacity.
 *   q: [B, H_q, d]; q_idx: [B, H_kv, d_idx]; k_cache, v_cache: [B, N, H_kv, d]; k_idx_cache: [B, N, d_idx]
 *   blocks: [B, H_kv, topk+1]; margin: [B, H_kv]; out: [B, H_q, d]; lse: [B, H_q]
 */
int orc_decode(const orc_dims *D, const int32_t *cache_len, const void *q, const void *q_idx, const void *k_cache,
               const void *v_cache, const void *k_idx_cache, int ty, int32_t *blocks, double *margin, double *out,
               double *lse) {
    const int K1 = D->topk + 1, G = D->H_q / D->H_kv;
    const double sc = eff_scale(D);
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)D->N);
        double *M = (double *)malloc(sizeof(double) * (size_t)(D->N / D->block_k + 2));
        int32_t *J = (int32_t *)malloc(sizeof(int32_t) * (size_t)D->N);
        double *z = (double *)malloc(sizeof(double) * (size_t)D->N);
#pragma omp for schedule(dynamic, 1)
        for (int x = 0; x < D->B * D->H_kv; ++x) {
            int b = x / D->H_kv, r = x % D->H_kv;
            int i = cache_len[b] - 1;
            if (i < 0) continue;
            size_t q_off = ((size_t)b * D->H_kv + r) * D->d_idx;
            size_t k_base = (size_t)b * D->N * D->d_idx;
            index_scores(D, q_idx, k_idx_cache, ty, q_off, k_base, i + 1, s);
            block_max(D, s, i, M);
            int32_t *sel = blocks + (size_t)x * K1;
            select_blocks(D, M, i, sel, &margin[x]);
            int nJ = token_set(D, sel, K1, i, J);
            size_t kv_base = ((size_t)b * D->N * D->H_kv + r) * D->d;
            for (int h = r * G; h < (r + 1) * G; ++h)
                attend_tokens(D->d, sc, q, k_cache, v_cache, ty, ((size_t)b * D->H_q + h) * D->d, kv_base,
                              (size_t)D->H_kv * D->d, J, nJ, z, out + ((size_t)b * D->H_q + h) * D->d,
                              lse + (size_t)b * D->H_q + h);
        }
        free(s);
        free(M);
        free(J);
        free(z);
    }
    return 0;
}

/* ---------------------------------------------------------------------------------------------
 * e4m3: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits. Exponent field 0 holds the
 * subnormals m * 2^-9; field e > 0 holds (1 + m/8) * 2^(e-7); code 0x7f (and 0xff) is NaN, so the
 * largest finite value is 0x7e = 1.75 * 2^8 = 448. There are no infinities.
 * -------------------------------------------------------------------------------------------- */
double orc_e4m3_value(int code) {
    const int e = (code >> 3) & 15, m = code & 7;
    const double sign = (code & 0x80) ? -1.0 : 1.0;
    if ((code & 0x7f) == 0x7f) return NAN;
    if (e == 0) return sign * ldexp((double)m, -9);
    return sign * ldexp(1.0 + m / 8.0, e - 7);
}

/* tab[c] = value of the non-negative finite code c, c = 0..126 */
static void e4m3_table(double *tab) {
    for (int c = 0; c < 0x7f; ++c) tab[c] = orc_e4m3_value(c);
}

/* The code of the e4m3 value nearest to y, ties to the even code (even mantissa), values beyond
 * 448 in magnitude saturated to +-448. Brute force over the 127 finite magnitudes. */
static int e4m3_round_tab(float y, const double *tab) {
    const double a = fabs((double)y);
    const int sign = signbit(y) ? 0x80 : 0;
    if (a >= 448.0) return sign | 0x7e;
    int best = 0;
    double best_err = a;
    for (int c = 1; c < 0x7f; ++c) {
        const double err = fabs(a - tab[c]);
        if (err < best_err || (err == best_err && (c & 1) == 0)) {
            best = c;
            best_err = err;
        }
    }
    return sign | best;
}

int orc_e4m3_round(float y) {
    double tab[0x7f];
    e4m3_table(tab);
    return e4m3_round_tab(y, tab);
}

void orc_e4m3_values(const uint8_t *codes, int64_t n, double *out) {
    for (int64_t x = 0; x < n; ++x) out[x] = orc_e4m3_value(codes[x]);
}

void orc_e4m3_round_many(const float *y, int64_t n, uint8_t *out) {
    double tab[0x7f];
    e4m3_table(tab);
#pragma omp parallel for schedule(static)
    for (int64_t x = 0; x < n; ++x) out[x] = (uint8_t)e4m3_round_tab(y[x], tab);
}

/* Row quantisation: scale[r] = max_c |x[r,c]| / 448 and codes[r,c] = e4m3(x[r,c] / scale[r]),
 * both quotients in float32 (the precision the serving path rounds in); scale 1 for a zero row.
 * x is bf16 bits [rows, n]. */
void orc_quantize_e4m3_rows(const uint16_t *x, int64_t rows, int n, uint8_t *codes, float *scale) {
    double tab[0x7f];
    e4m3_table(tab);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        float amax = 0.0f;
        for (int c = 0; c < n; ++c) {
            const float v = (float)ld(x, ORC_BF16, (size_t)r * n + c);
            if (fabsf(v) > amax) amax = fabsf(v);
        }
        const float sc = amax > 0.0f ? amax / 448.0f : 1.0f;
        scale[r] = sc;
        for (int c = 0; c < n; ++c) {
            const float v = (float)ld(x, ORC_BF16, (size_t)r * n + c);
            const float y = v / sc;
            codes[(size_t)r * n + c] = (uint8_t)e4m3_round_tab(y, tab);
        }
    }
}

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
