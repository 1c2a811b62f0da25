/*
 * oracle.c -- TEST INFRASTRUCTURE. Not part of the library.
 *
 * A plain, slow, obviously correct fp64 CPU statement of sparse-mask scaled
 * dot-product attention and of the mask patterns it is run on. Only the test
 * suite, the smoke check and the benchmark's CPU-baseline leg load this code;
 * the library never does, and this file shares no code, header or constant with
 * the CUDA path.
 *
 * What it computes, and where each step comes from:
 *
 *   "[Proposal] Unified Interface/Implementation for Sparse Attention"
 *   (gluon-nlp issue 1407), opening post:
 *     - the user supplies an n x n CSR/COO mask; token i attends to token j
 *       exactly when mask[i, j] = 1;
 *     - attention scores are dot products q_i . k_j taken only at the mask's
 *       nonzeros (an SDDMM) and keep the mask's sparsity pattern;
 *     - the weights are a softmax over each row's nonzeros;
 *     - the context is the sparse weight matrix times V (an SpMM).
 *
 *   "support attentions in AlphaFold2" (flash-attention PR 57), first post and
 *   the mask / bias shape rules: an additive attention mask and an additive
 *   attention bias are added to the scores before the softmax. The softmax
 *   scale multiplies the dot product only (the reading that the snippet with
 *   `softmax_scale` leaves open is settled this way).
 *
 *   "Implementing and Optimizing the Scaled Dot-Product Attention on Streaming
 *   Dataflow" (review), proposed method: the row-wise max and sum are replaced by
 *   a running max and a running sum, rescaled by a delta term
 *   exp(m_old - m_new) whenever the max grows, and the division by the sum is
 *   moved after the weighted sum of V (distributive law). That second variant is
 *   kept here next to the plain two-pass definition so that the two can be
 *   checked against each other.
 *
 * Degenerate rows (no nonzeros, or every score -inf): out = 0 and lse = -inf.
 * The pages leave this open; the softmax is undefined there.
 *
 * Inputs are read at their exact values: bf16 (given as uint16 bit patterns)
 * and fp32 widen to fp64 without rounding.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* element types of the input arrays */
enum { ORC_F64 = 0, ORC_F32 = 1, ORC_BF16 = 2 };

static double read_elem(const void* base, int type, int64_t idx) {
    switch (type) {
    case ORC_F64: return ((const double*)base)[idx];
    case ORC_F32: return (double)((const float*)base)[idx];
    default: {
        uint32_t u = ((uint32_t)((const uint16_t*)base)[idx]) << 16;
        float f;
        memcpy(&f, &u, sizeof f);
        return (double)f;
    }
    }
}

/* An additive term over (b, h, i, j): the attention mask or the attention bias.
 * Strides are in elements; a stride of 0 broadcasts that dimension. */
typedef struct {
    const void* data; /* NULL: absent (adds 0) */
    int type;
    int64_t stride[4];
} orc_addend;

typedef struct {
    int64_t B, H, n, d;
    const void *q, *k, *v; /* [B, H, n, d], contiguous */
    int qkv_type;
    int64_t num_masks; /* 1 (shared by all b) or B (one per b) */
    const int64_t* row_ptr; /* [num_masks * n + 1] */
    const int32_t* col_idx;
    double scale;
    orc_addend mask, bias;
} orc_problem;

static double addend_at(const orc_addend* a, int64_t b, int64_t h, int64_t i, int64_t j) {
    if (!a->data) return 0.0;
    return read_elem(a->data, a->type,
                     b * a->stride[0] + h * a->stride[1] + i * a->stride[2] + j * a->stride[3]);
}

/* Score of nonzero (i, j) for batch b, head h: scale * <q_i, k_j> + mask + bias. */
static double score(const orc_problem* P, int64_t b, int64_t h, int64_t i, int64_t j) {
    const int64_t base = (b * P->H + h) * P->n;
    double dot = 0.0;
    for (int64_t e = 0; e < P->d; ++e)
        dot += read_elem(P->q, P->qkv_type, (base + i) * P->d + e) *
               read_elem(P->k, P->qkv_type, (base + j) * P->d + e);
    return P->scale * dot + addend_at(&P->mask, b, h, i, j) + addend_at(&P->bias, b, h, i, j);
}

static double v_at(const orc_problem* P, int64_t b, int64_t h, int64_t j, int64_t e) {
    return read_elem(P->v, P->qkv_type, ((b * P->H + h) * P->n + j) * P->d + e);
}

static void mask_row_range(const orc_problem* P, int64_t b, int64_t i, int64_t* p0, int64_t* p1) {
    const int64_t r = (P->num_masks == 1 ? 0 : b) * P->n + i;
    *p0 = P->row_ptr[r];
    *p1 = P->row_ptr[r + 1];
}

/* The plain definition: scores on the row's nonzeros, then a two-pass softmax
 * (max, then exp and sum), then the weighted sum of V rows with the normalised
 * weights. `s` is scratch of the row's length; `w` (optional) receives the
 * softmax weights in row order. */
static void row_two_pass(const orc_problem* P, int64_t b, int64_t h, int64_t i, double* s,
                         double* out, double* lse, double* w) {
    int64_t p0, p1;
    mask_row_range(P, b, i, &p0, &p1);
    const int64_t len = p1 - p0;
    double m = -INFINITY;
    for (int64_t t = 0; t < len; ++t) {
        s[t] = score(P, b, h, i, P->col_idx[p0 + t]);
        if (s[t] > m) m = s[t];
    }
    for (int64_t e = 0; e < P->d; ++e) out[e] = 0.0;
    if (len == 0 || m == -INFINITY) {
        *lse = -INFINITY;
        if (w)
            for (int64_t t = 0; t < len; ++t) w[t] = 0.0;
        return;
    }
    double l = 0.0;
    for (int64_t t = 0; t < len; ++t) {
        s[t] = exp(s[t] - m);
        l += s[t];
    }
    for (int64_t t = 0; t < len; ++t) {
        const double pw = s[t] / l;
        if (w) w[t] = pw;
        const int64_t j = P->col_idx[p0 + t];
        for (int64_t e = 0; e < P->d; ++e) out[e] += pw * v_at(P, b, h, j, e);
    }
    *lse = m + log(l);
}

/* The streaming form: one pass over the row keeping a running max m, a running
 * sum l and an unnormalised accumulator acc; when the max grows, l and acc are
 * rescaled by the delta term exp(m_old - m_new); the division by l happens once,
 * at the end. */
static void row_online(const orc_problem* P, int64_t b, int64_t h, int64_t i, double* acc,
                       double* out, double* lse) {
    int64_t p0, p1;
    mask_row_range(P, b, i, &p0, &p1);
    double m = -INFINITY, l = 0.0;
    for (int64_t e = 0; e < P->d; ++e) acc[e] = 0.0;
    for (int64_t p = p0; p < p1; ++p) {
        const int64_t j = P->col_idx[p];
        const double s = score(P, b, h, i, j);
        const double m_new = s > m ? s : m;
        if (m_new == -INFINITY) continue; /* nothing but -inf so far */
        const double delta = exp(m - m_new);
        const double ws = exp(s - m_new);
        l = l * delta + ws;
        for (int64_t e = 0; e < P->d; ++e) acc[e] = acc[e] * delta + ws * v_at(P, b, h, j, e);
        m = m_new;
    }
    if (l == 0.0) {
        for (int64_t e = 0; e < P->d; ++e) out[e] = 0.0;
        *lse = -INFINITY;
        return;
    }
    for (int64_t e = 0; e < P->d; ++e) out[e] = acc[e] / l;
    *lse = m + log(l);
}

static int64_t max_row_len(const orc_problem* P) {
    int64_t mx = 0;
    for (int64_t r = 0; r < P->num_masks * P->n; ++r) {
        const int64_t len = P->row_ptr[r + 1] - P->row_ptr[r];
        if (len > mx) mx = len;
    }
    return mx;
}

static void fill_addend(orc_addend* a, const void* data, int type, const int64_t* stride) {
    a->data = data;
    a->type = type;
    for (int t = 0; t < 4; ++t) a->stride[t] = data ? stride[t] : 0;
}

/*
 * Masked scaled dot-product attention.
 *   variant 0: plain two-pass definition; variant 1: running max / sum.
 *   rows: optional list of flat row ids (b * H + h) * n + i to compute; NULL = all,
 *         in which case n_rows must be B * H * n.
 *   out: [n_rows, d] fp64; lse: [n_rows] fp64 (natural log of the sum of
 *        exp(score) over the row, -inf for degenerate rows).
 *   threads: OpenMP threads (0 = runtime default).
 * Returns 0, or -1 when an argument is out of range.
 */
int oracle_sdpa(int variant, int64_t B, int64_t H, int64_t n, int64_t d, const void* q,
                const void* k, const void* v, int qkv_type, int64_t num_masks,
                const int64_t* row_ptr, const int32_t* col_idx, double scale, const void* mask,
                int mask_type, const int64_t* mask_stride, const void* bias, int bias_type,
                const int64_t* bias_stride, const int64_t* rows, int64_t n_rows, double* out,
                double* lse, int threads) {
    if (B < 0 || H < 0 || n < 0 || d <= 0 || (num_masks != 1 && num_masks != B)) return -1;
    if (!rows && n_rows != B * H * n) return -1;
    orc_problem P;
    P.B = B; P.H = H; P.n = n; P.d = d;
    P.q = q; P.k = k; P.v = v; P.qkv_type = qkv_type;
    P.num_masks = num_masks; P.row_ptr = row_ptr; P.col_idx = col_idx; P.scale = scale;
    fill_addend(&P.mask, mask, mask_type, mask_stride);
    fill_addend(&P.bias, bias, bias_type, bias_stride);
    for (int64_t p = 0; p < row_ptr[num_masks * n]; ++p)
        if (col_idx[p] < 0 || col_idx[p] >= n) return -1;
    const int64_t scratch = (variant == 0 ? max_row_len(&P) : d) + 1;
#ifdef _OPENMP
    if (threads > 0) omp_set_num_threads(threads);
#else
    (void)threads;
#endif
#pragma omp parallel
    {
        double* buf = (double*)malloc(sizeof(double) * (size_t)scratch);
#pragma omp for schedule(dynamic, 16)
        for (int64_t t = 0; t < n_rows; ++t) {
            const int64_t flat = rows ? rows[t] : t;
            const int64_t i = flat % n, bh = flat / n;
            const int64_t h = bh % H, b = bh / H;
            if (variant == 0)
                row_two_pass(&P, b, h, i, buf, out + t * d, lse + t, NULL);
            else
                row_online(&P, b, h, i, buf, out + t * d, lse + t);
        }
        free(buf);
    }
    return 0;
}

/* Softmax weights of one row (two-pass definition), in the row's CSR order. */
int oracle_row_weights(int64_t B, int64_t H, int64_t n, int64_t d, const void* q, const void* k,
                       const void* v, int qkv_type, int64_t num_masks, const int64_t* row_ptr,
                       const int32_t* col_idx, double scale, const void* mask, int mask_type,
                       const int64_t* mask_stride, const void* bias, int bias_type,
                       const int64_t* bias_stride, int64_t flat_row, double* weights) {
    orc_problem P;
    P.B = B; P.H = H; P.n = n; P.d = d;
    P.q = q; P.k = k; P.v = v; P.qkv_type = qkv_type;
    P.num_masks = num_masks; P.row_ptr = row_ptr; P.col_idx = col_idx; P.scale = scale;
    fill_addend(&P.mask, mask, mask_type, mask_stride);
    fill_addend(&P.bias, bias, bias_type, bias_stride);
    const int64_t i = flat_row % n, bh = flat_row / n;
    const int64_t h = bh % H, b = bh / H;
    double* s = (double*)malloc(sizeof(double) * (size_t)(max_row_len(&P) + 1));
    double* out = (double*)malloc(sizeof(double) * (size_t)d);
    double lse;
    row_two_pass(&P, b, h, i, s, out, &lse, weights);
    free(s);
    free(out);
    return 0;
}

/*
 * Gradients of masked attention: the chain rule applied to the plain definition
 * above (row_two_pass), for an upstream gradient dout = dL/dout. For each
 * (b, h, i) with weights w_ij = softmax over the row's nonzeros of s_ij and
 * out_i = sum_j w_ij v_j:
 *   dv_j  += w_ij dout_i
 *   dw_ij  = <dout_i, v_j>
 *   ds_ij  = w_ij (dw_ij - sum_k w_ik dw_ik)         (Jacobian of the softmax)
 *   dq_i  += scale ds_ij k_j ;  dk_j += scale ds_ij q_i
 *   dbias[b, h, i, j] += ds_ij, summed over the bias's broadcast dimensions
 *                        (dbias_stride: element strides of dbias, 0 = broadcast)
 * A degenerate row (weights all 0) contributes nothing. dq, dk, dv: [B, H, n, d]
 * fp64, overwritten; dbias (optional) is overwritten. Sequential (the column sums
 * and the broadcast sums would race). Returns 0, or -1 for a bad argument.
 */
int oracle_sdpa_bwd(int64_t B, int64_t H, int64_t n, int64_t d, const void* q, const void* k,
                    const void* v, int qkv_type, int64_t num_masks, const int64_t* row_ptr,
                    const int32_t* col_idx, double scale, const void* mask, int mask_type,
                    const int64_t* mask_stride, const void* bias, int bias_type,
                    const int64_t* bias_stride, const void* dout, int dout_type, double* dq,
                    double* dk, double* dv, double* dbias, const int64_t* dbias_stride,
                    int64_t dbias_elems) {
    if (B < 0 || H < 0 || n < 0 || d <= 0 || (num_masks != 1 && num_masks != B)) return -1;
    orc_problem P;
    P.B = B; P.H = H; P.n = n; P.d = d;
    P.q = q; P.k = k; P.v = v; P.qkv_type = qkv_type;
    P.num_masks = num_masks; P.row_ptr = row_ptr; P.col_idx = col_idx; P.scale = scale;
    fill_addend(&P.mask, mask, mask_type, mask_stride);
    fill_addend(&P.bias, bias, bias_type, bias_stride);
    for (int64_t p = 0; p < row_ptr[num_masks * n]; ++p)
        if (col_idx[p] < 0 || col_idx[p] >= n) return -1;
    const int64_t total = B * H * n * d;
    for (int64_t x = 0; x < total; ++x) dq[x] = dk[x] = dv[x] = 0.0;
    if (dbias)
        for (int64_t x = 0; x < dbias_elems; ++x) dbias[x] = 0.0;
    const int64_t mx = max_row_len(&P) + 1;
    double* s = (double*)malloc(sizeof(double) * (size_t)mx);
    double* w = (double*)malloc(sizeof(double) * (size_t)mx);
    double* dw = (double*)malloc(sizeof(double) * (size_t)mx);
    double* out = (double*)malloc(sizeof(double) * (size_t)d);
    for (int64_t b = 0; b < B; ++b)
        for (int64_t h = 0; h < H; ++h)
            for (int64_t i = 0; i < n; ++i) {
                const int64_t base = (b * H + h) * n;
                double lse;
                row_two_pass(&P, b, h, i, s, out, &lse, w);
                int64_t p0, p1;
                mask_row_range(&P, b, i, &p0, &p1);
                double sum_wdw = 0.0;
                for (int64_t t = 0; t < p1 - p0; ++t) {
                    const int64_t j = col_idx[p0 + t];
                    double acc = 0.0;
                    for (int64_t e = 0; e < d; ++e)
                        acc += read_elem(dout, dout_type, (base + i) * d + e) * v_at(&P, b, h, j, e);
                    dw[t] = acc;
                    sum_wdw += w[t] * acc;
                }
                for (int64_t t = 0; t < p1 - p0; ++t) {
                    const int64_t j = col_idx[p0 + t];
                    const double ds = w[t] * (dw[t] - sum_wdw);
                    for (int64_t e = 0; e < d; ++e) {
                        dv[(base + j) * d + e] += w[t] * read_elem(dout, dout_type, (base + i) * d + e);
                        dq[(base + i) * d + e] += scale * ds * read_elem(k, qkv_type, (base + j) * d + e);
                        dk[(base + j) * d + e] += scale * ds * read_elem(q, qkv_type, (base + i) * d + e);
                    }
                    if (dbias)
                        dbias[b * dbias_stride[0] + h * dbias_stride[1] + i * dbias_stride[2] +
                              j * dbias_stride[3]] += ds;
                }
            }
    free(s);
    free(w);
    free(dw);
    free(out);
    return 0;
}

/*
 * Mask patterns, by brute force over every (i, j) of the n x n grid.
 *
 * Patterns ("Sparse Attention" notes page, list of common patterns; the variable
 * window from the gluon-nlp proposal's discussion):
 *   1 sliding window:  |i - j| <= window
 *   2 variable window: i - w_i <= j <= i + w_i, w_i = half_widths[m * n + i]
 *   3 block + strided + global:
 *        (block > 0 and floor(i / block) == floor(j / block))
 *     or (stride > 0 and (j - i) is a multiple of stride)
 *     or i < n_global or j < n_global
 *   4 COO candidates: the listed columns of row r (cand_row_ptr / cand_cols),
 *     duplicates merged, plus (i, i) when add_diagonal
 *   5 dense: every (i, j)
 * Mask m (0 <= m < num_masks) covers rows m * n .. m * n + n - 1 of the output.
 * Columns come out ascending and unique. With col_idx == NULL only row_ptr is
 * filled. Returns the total number of nonzeros, or -1 for a bad argument
 * (unknown kind, candidate column out of [0, n)).
 */
int64_t oracle_mask_csr(int kind, int64_t n, int64_t num_masks, int64_t window, int64_t block,
                        int64_t stride, int64_t n_global, const int32_t* half_widths,
                        const int64_t* cand_row_ptr, const int32_t* cand_cols, int add_diagonal,
                        int64_t* row_ptr, int32_t* col_idx) {
    if (kind < 1 || kind > 5 || n < 0 || num_masks < 1) return -1;
    unsigned char* flag = (unsigned char*)malloc((size_t)(n > 0 ? n : 1));
    int64_t nnz = 0;
    row_ptr[0] = 0;
    for (int64_t m = 0; m < num_masks; ++m) {
        for (int64_t i = 0; i < n; ++i) {
            const int64_t r = m * n + i;
            memset(flag, 0, (size_t)n);
            if (kind == 4) {
                for (int64_t p = cand_row_ptr[r]; p < cand_row_ptr[r + 1]; ++p) {
                    const int64_t c = cand_cols[p];
                    if (c < 0 || c >= n) {
                        free(flag);
                        return -1;
                    }
                    flag[c] = 1;
                }
                if (add_diagonal) flag[i] = 1;
            } else {
                for (int64_t j = 0; j < n; ++j) {
                    int on = 0;
                    if (kind == 1) {
                        on = llabs(i - j) <= window;
                    } else if (kind == 2) {
                        const int64_t w = half_widths[r];
                        on = (j >= i - w) && (j <= i + w);
                    } else if (kind == 3) {
                        on = (block > 0 && i / block == j / block) ||
                             (stride > 0 && (j - i) % stride == 0) || i < n_global ||
                             j < n_global;
                    } else {
                        on = 1;
                    }
                    flag[j] = (unsigned char)on;
                }
            }
            for (int64_t j = 0; j < n; ++j) {
                if (!flag[j]) continue;
                if (col_idx) col_idx[nnz] = (int32_t)j;
                ++nnz;
            }
            row_ptr[r + 1] = nnz;
        }
    }
    free(flag);
    return nnz;
}
