/*
 * fa_oracle.c -- plain, slow, float64 CPU oracle for the attention forward path.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product library calls, links or loads
 * this file; it is built into its own shared object and only the test suite, the
 * smoke check and the benchmark's CPU-baseline leg use it. It shares no code,
 * header, table or constant with the CUDA path.
 *
 * What it computes is the plain definition of attention, written out without any
 * blocking, fusion or reordering:
 *
 *   standard attention, page "昇腾CANN跑大模型，FlashAttention这个算子你得认识一下",
 *   section "传统实现到底慢在哪": scores = Q K^T / sqrt(d_k), attn = softmax(scores),
 *   output = attn V.  The score row of each query is materialised in full.
 *
 *   causal masking, same page, section "昇腾NPU上做了什么特殊优化" and the
 *   scaled_dot_product_attention(..., is_causal=True) call of section "怎么用起来":
 *   a token sees itself and the tokens before it; a key after the query gets the
 *   score -infinity, so its softmax weight exp(-inf) is exactly 0.
 *
 *   the packed path, page "IAW 模型 FA2 vs FA3 实测", section 1: unpad takes rows of the
 *   padded (B*total_len, H, D) tensor by index (a gather); varlen attention is dense
 *   attention inside each sequence of the packed tensor; pad scatters the packed rows
 *   back by index and leaves every other row zero.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - scale <= 0 means 1/sqrt(D) (the sqrt(d_k) of the definition);
 *   - lse[i] = M_i + ln(sum_j exp(s_ij - M_i)), natural log, in units of the scaled score;
 *   - the causal mask is aligned at the first token of each sequence (queries and keys
 *     share one length per sequence, so top-left and bottom-right alignment coincide);
 *   - pad fills the rows no index names with zero bytes.
 *
 * Inputs are float64 copies of the fp16/bf16 values (widening is exact).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG (-1)
#define ORACLE_ERR_RANGE (-2)
#define ORACLE_ERR_NOMEM (-3)

int fa_oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Softmax weights of one query row over the key window [lo, hi) of a token-major
 * (N, H, D) tensor.  s_j = scale * sum_d q_d k_jd, masked keys get -inf; then
 * M = max_j s_j, w_j = exp(s_j - M) and L = sum_j w_j.  Returns M through *m_out,
 * L through *l_out and the unnormalised weights in w[0 .. hi-lo).
 * `pos` is the query's position inside its sequence (used by the causal mask only).
 */
static void score_row(const double *q, const double *k, int64_t H, int64_t D, int64_t tok,
                      int64_t head, int64_t lo, int64_t hi, int64_t pos, int causal,
                      double scale, double *w, double *m_out, double *l_out) {
    const double *qi = q + (tok * H + head) * D;
    int64_t n = hi - lo;
    for (int64_t j = 0; j < n; ++j) {
        if (causal && j > pos) {
            w[j] = -INFINITY;
            continue;
        }
        const double *kj = k + ((lo + j) * H + head) * D;
        double dot = 0.0;
        for (int64_t d = 0; d < D; ++d) dot += qi[d] * kj[d];
        w[j] = scale * dot;
    }
    double m = -INFINITY;
    for (int64_t j = 0; j < n; ++j)
        if (w[j] > m) m = w[j];
    double l = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        w[j] = exp(w[j] - m); /* exp(-inf) == 0 for masked keys */
        l += w[j];
    }
    *m_out = m;
    *l_out = l;
}

/*
 * Attention output and log-sum-exp for a list of query rows.
 *
 *   q, k, v   float64, token-major (N, H, D) (a dense (B,S,H,D) tensor is N = B*S)
 *   tok[r]    flat token of the query row r
 *   head[r]   head of row r
 *   lo[r],hi[r]  the key window [lo, hi): the query's own sequence
 *   causal    nonzero: keys after the query (position tok-lo) are masked
 *   out       (nrows, D) float64;  lse (nrows) float64;  probs optional (nrows, max_win)
 *             receiving the normalised weights w_j / L (row r uses hi-lo entries)
 *   nthreads  <= 0: the OpenMP default
 */
int fa_oracle_attention_rows(const double *q, const double *k, const double *v, int64_t N,
                             int64_t H, int64_t D, const int64_t *tok, const int64_t *head,
                             const int64_t *lo, const int64_t *hi, int64_t nrows, double scale,
                             int causal, double *out, double *lse, double *probs,
                             int64_t max_win, int nthreads) {
    if (!q || !k || !v || !tok || !head || !lo || !hi || !out || !lse) return ORACLE_ERR_ARG;
    if (H <= 0 || D <= 0 || nrows < 0 || N < 0) return ORACLE_ERR_ARG;
    if (scale <= 0.0) scale = 1.0 / sqrt((double)D);
    int64_t win = 0;
    for (int64_t r = 0; r < nrows; ++r) {
        if (lo[r] < 0 || hi[r] > N || lo[r] >= hi[r] || tok[r] < lo[r] || tok[r] >= hi[r] ||
            head[r] < 0 || head[r] >= H)
            return ORACLE_ERR_RANGE;
        if (hi[r] - lo[r] > win) win = hi[r] - lo[r];
    }
    if (probs && max_win < win) return ORACLE_ERR_ARG;
    int err = ORACLE_OK;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads)
#endif
    {
        double *w = (double *)malloc(sizeof(double) * (size_t)(win > 0 ? win : 1));
        if (!w) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            err = ORACLE_ERR_NOMEM;
        } else {
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 4)
#endif
            for (int64_t r = 0; r < nrows; ++r) {
                double m, l;
                int64_t n = hi[r] - lo[r];
                score_row(q, k, H, D, tok[r], head[r], lo[r], hi[r], tok[r] - lo[r], causal, scale,
                          w, &m, &l);
                double *o = out + r * D;
                for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
                for (int64_t j = 0; j < n; ++j) {
                    if (w[j] == 0.0) continue;
                    const double *vj = v + ((lo[r] + j) * H + head[r]) * D;
                    for (int64_t d = 0; d < D; ++d) o[d] += w[j] * vj[d];
                }
                for (int64_t d = 0; d < D; ++d) o[d] /= l;
                lse[r] = m + log(l);
                if (probs)
                    for (int64_t j = 0; j < n; ++j) probs[r * max_win + j] = w[j] / l;
            }
            free(w);
        }
    }
    return err;
}

/*
 * Unpad: out[r] = x[indices[r]] for r < nnz, rows of `row_bytes` bytes.
 * Indices must lie in [0, total_rows).
 */
int fa_oracle_unpad(const uint8_t *x, const int64_t *indices, int64_t nnz, int64_t total_rows,
                    int64_t row_bytes, uint8_t *out) {
    if ((!x && total_rows > 0) || (!indices && nnz > 0) || (!out && nnz > 0) || nnz < 0 ||
        row_bytes <= 0)
        return ORACLE_ERR_ARG;
    for (int64_t r = 0; r < nnz; ++r)
        if (indices[r] < 0 || indices[r] >= total_rows) return ORACLE_ERR_RANGE;
    for (int64_t r = 0; r < nnz; ++r)
        for (int64_t b = 0; b < row_bytes; ++b) out[r * row_bytes + b] = x[indices[r] * row_bytes + b];
    return ORACLE_OK;
}

/*
 * Pad: every row of out (total_rows x row_bytes) is zero except out[indices[r]] = x[r].
 */
int fa_oracle_pad(const uint8_t *x, const int64_t *indices, int64_t nnz, int64_t total_rows,
                  int64_t row_bytes, uint8_t *out) {
    if ((!x && nnz > 0) || (!indices && nnz > 0) || (!out && total_rows > 0) || nnz < 0 ||
        total_rows < 0 || row_bytes <= 0)
        return ORACLE_ERR_ARG;
    for (int64_t r = 0; r < nnz; ++r)
        if (indices[r] < 0 || indices[r] >= total_rows) return ORACLE_ERR_RANGE;
    for (int64_t i = 0; i < total_rows * row_bytes; ++i) out[i] = 0;
    for (int64_t r = 0; r < nnz; ++r)
        for (int64_t b = 0; b < row_bytes; ++b) out[indices[r] * row_bytes + b] = x[r * row_bytes + b];
    return ORACLE_OK;
}
