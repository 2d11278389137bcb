/*
 * attn_oracle.c -- plain fp64 CPU oracle for exact scaled-dot-product attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file; only the tests, the smoke check and the bench's CPU-baseline leg
 * do.  It shares no code, header, table or constant with the CUDA library.
 *
 * What it computes (each function names the passage it follows):
 *   "YOLO11 ... FlashAttention-2" page, section 1.2: the standard three-step
 *   attention S = Q K^T, P = softmax(S), O = P V, with S and P materialised;
 *   section 3.2's sketch and the LLM explainer page, section 1, add the
 *   1/sqrt(d) factor on the scores (here the caller's `scale`).
 *   The LLM explainer page, section 4.3, and the YOLO11 page, section 2.2:
 *   the online-softmax recurrence with a running max m and running sum l.
 *   The LLM explainer page, section 6.2 (recompute strategy): backward by
 *   recomputing S and P; the gradients are the textbook chain rule through
 *   softmax, which that passage presupposes but does not print.
 *   The LLM explainer page, section 7.1: the causal mask of GPT-style models,
 *   which hides every future position from a query: with `causal` set, row i
 *   attends to keys j <= i only (P_ij = 0 for j > i).  Every public function
 *   takes `causal` as its last argument (0: all keys).
 *
 * Layout: q, k, v, o, dO, dq, dk, dv are [B, N, H, d] row-major fp64;
 * lse is [B, H, N] fp64, natural log.  All loops are plain and sequential
 * inside one row; OpenMP only splits independent rows or heads.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static inline size_t at(int b, int n, int h, int x, int N, int H, int d)
{
    return (((size_t)b * N + n) * H + h) * (size_t)d + x;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads for later calls (n >= 1); used to time the oracle on one core.
 * Changes no arithmetic: every row is computed by one thread either way. */
void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n >= 1)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/*
 * Row i of the probability matrix, by the definition (YOLO11 page, 1.2):
 *   S_ij = scale * sum_x q_ix k_jx,  m_i = max_j S_ij,
 *   l_i = sum_j exp(S_ij - m_i),     P_ij = exp(S_ij - m_i) / l_i,
 * over the keys the row sees: j < N, or j <= i with the causal mask (LLM
 * explainer page, 7.1); P_ij = 0 for the hidden keys.
 * Writes P_i. into p[0..N) and returns m_i, l_i.
 */
static void row_probs(const double *q, const double *k, int b, int h, int i,
                      int N, int H, int d, double scale, int causal, double *p,
                      double *m_out, double *l_out)
{
    const int nk = causal ? i + 1 : N;  /* keys visible to row i */
    const double *qi = q + at(b, i, h, 0, N, H, d);
    for (int j = 0; j < nk; ++j) {
        const double *kj = k + at(b, j, h, 0, N, H, d);
        double dot = 0.0;
        for (int x = 0; x < d; ++x) dot += qi[x] * kj[x];
        p[j] = scale * dot;
    }
    double m = p[0];
    for (int j = 1; j < nk; ++j) if (p[j] > m) m = p[j];
    double l = 0.0;
    for (int j = 0; j < nk; ++j) l += exp(p[j] - m);
    for (int j = 0; j < nk; ++j) p[j] = exp(p[j] - m) / l;
    for (int j = nk; j < N; ++j) p[j] = 0.0;
    *m_out = m;
    *l_out = l;
}

/* P for every (b, h): probs is [B, H, N, N].  Small N only (tests). */
void oracle_attn_probs(const double *q, const double *k, double *probs,
                       int B, int H, int N, int d, double scale, int causal)
{
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
            for (int i = 0; i < N; ++i) {
                double m, l;
                row_probs(q, k, b, h, i, N, H, d, scale, causal,
                          probs + (((size_t)b * H + h) * N + i) * (size_t)N, &m, &l);
            }
}

/* One output row: O_i = sum_j P_ij V_j, LSE_i = m_i + ln l_i. */
static void fwd_row(const double *q, const double *k, const double *v,
                    int b, int h, int i, int N, int H, int d, double scale,
                    int causal, double *p, double *o_row, double *lse_out)
{
    double m, l;
    row_probs(q, k, b, h, i, N, H, d, scale, causal, p, &m, &l);
    for (int x = 0; x < d; ++x) o_row[x] = 0.0;
    for (int j = 0; j < N; ++j) {
        const double *vj = v + at(b, j, h, 0, N, H, d);
        for (int x = 0; x < d; ++x) o_row[x] += p[j] * vj[x];
    }
    *lse_out = m + log(l);
}

/* Forward pass by the definition, every row. */
void oracle_attn_fwd(const double *q, const double *k, const double *v,
                     double *o, double *lse, int B, int H, int N, int d,
                     double scale, int causal)
{
    long long rows = (long long)B * H * N;
#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * (size_t)N);
#pragma omp for schedule(dynamic, 16)
        for (long long r = 0; r < rows; ++r) {
            int i = (int)(r % N);
            int h = (int)((r / N) % H);
            int b = (int)(r / ((long long)N * H));
            fwd_row(q, k, v, b, h, i, N, H, d, scale, causal, p,
                    o + at(b, i, h, 0, N, H, d),
                    lse + ((size_t)b * H + h) * N + i);
        }
        free(p);
    }
}

/*
 * Forward pass for selected rows only (full-size sampling).  rows holds
 * nrows triples (b, h, i); o_rows is [nrows, d], lse_rows is [nrows].
 */
void oracle_attn_fwd_rows(const double *q, const double *k, const double *v,
                          const int *rows, int nrows, double *o_rows,
                          double *lse_rows, int B, int H, int N, int d,
                          double scale, int causal)
{
    (void)B;
#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * (size_t)N);
#pragma omp for schedule(dynamic, 1)
        for (int r = 0; r < nrows; ++r)
            fwd_row(q, k, v, rows[3 * r], rows[3 * r + 1], rows[3 * r + 2], N,
                    H, d, scale, causal, p, o_rows + (size_t)r * d, lse_rows + r);
        free(p);
    }
}

/*
 * Two-pass softmax attention: pass 1 finds m_i and l_i = sum_j exp(S_ij-m_i)
 * (sequential in j), pass 2 accumulates sum_j exp(S_ij-m_i) V_j (sequential in
 * j) and divides by l_i once.  Reference point for the online recurrence.
 */
void oracle_attn_fwd_two_pass(const double *q, const double *k, const double *v,
                              double *o, double *lse, int B, int H, int N,
                              int d, double scale)
{
    double *s = (double *)malloc(sizeof(double) * (size_t)N);
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
            for (int i = 0; i < N; ++i) {
                const double *qi = q + at(b, i, h, 0, N, H, d);
                for (int j = 0; j < N; ++j) {
                    const double *kj = k + at(b, j, h, 0, N, H, d);
                    double dot = 0.0;
                    for (int x = 0; x < d; ++x) dot += qi[x] * kj[x];
                    s[j] = scale * dot;
                }
                double m = s[0];
                for (int j = 1; j < N; ++j) if (s[j] > m) m = s[j];
                double l = 0.0;
                for (int j = 0; j < N; ++j) l += exp(s[j] - m);
                double *oi = o + at(b, i, h, 0, N, H, d);
                for (int x = 0; x < d; ++x) oi[x] = 0.0;
                for (int j = 0; j < N; ++j) {
                    double e = exp(s[j] - m);
                    const double *vj = v + at(b, j, h, 0, N, H, d);
                    for (int x = 0; x < d; ++x) oi[x] += e * vj[x];
                }
                for (int x = 0; x < d; ++x) oi[x] = oi[x] / l;
                lse[((size_t)b * H + h) * N + i] = m + log(l);
            }
    free(s);
}

/*
 * The FlashAttention-2 recurrence in fp64 (LLM explainer page, sections 4.2,
 * 4.3 and 5.2; YOLO11 page, section 2.2): the outer loop walks Q blocks of
 * block_q rows, the inner loop walks K/V blocks of block_kv rows.  Per row it
 * keeps a running max m, a running exponent sum l and an unnormalised output
 * acc.  On each K/V block: m_new = max(m, block max), alpha = exp(m - m_new),
 * l and acc are multiplied by alpha, then every key of the block adds
 * exp(S_ij - m_new) to l and exp(S_ij - m_new) V_j to acc.  After the last
 * block O_i = acc / l and LSE_i = m + ln l.
 */
void oracle_attn_fwd_online(const double *q, const double *k, const double *v,
                            double *o, double *lse, int B, int H, int N, int d,
                            double scale, int block_q, int block_kv)
{
    double *m = (double *)malloc(sizeof(double) * (size_t)block_q);
    double *l = (double *)malloc(sizeof(double) * (size_t)block_q);
    double *acc = (double *)malloc(sizeof(double) * (size_t)block_q * d);
    double *s = (double *)malloc(sizeof(double) * (size_t)block_kv);
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
            for (int q0 = 0; q0 < N; q0 += block_q) {
                int nq = (N - q0 < block_q) ? N - q0 : block_q;
                for (int r = 0; r < nq; ++r) {
                    m[r] = -INFINITY;
                    l[r] = 0.0;
                    for (int x = 0; x < d; ++x) acc[(size_t)r * d + x] = 0.0;
                }
                for (int k0 = 0; k0 < N; k0 += block_kv) {
                    int nk = (N - k0 < block_kv) ? N - k0 : block_kv;
                    for (int r = 0; r < nq; ++r) {
                        const double *qi = q + at(b, q0 + r, h, 0, N, H, d);
                        for (int c = 0; c < nk; ++c) {
                            const double *kj = k + at(b, k0 + c, h, 0, N, H, d);
                            double dot = 0.0;
                            for (int x = 0; x < d; ++x) dot += qi[x] * kj[x];
                            s[c] = scale * dot;
                        }
                        double bm = s[0];
                        for (int c = 1; c < nk; ++c) if (s[c] > bm) bm = s[c];
                        double m_new = (bm > m[r]) ? bm : m[r];
                        double alpha = exp(m[r] - m_new);
                        l[r] = l[r] * alpha;
                        double *ar = acc + (size_t)r * d;
                        for (int x = 0; x < d; ++x) ar[x] = ar[x] * alpha;
                        for (int c = 0; c < nk; ++c) {
                            double e = exp(s[c] - m_new);
                            l[r] += e;
                            const double *vj = v + at(b, k0 + c, h, 0, N, H, d);
                            for (int x = 0; x < d; ++x) ar[x] += e * vj[x];
                        }
                        m[r] = m_new;
                    }
                }
                for (int r = 0; r < nq; ++r) {
                    double *oi = o + at(b, q0 + r, h, 0, N, H, d);
                    for (int x = 0; x < d; ++x) oi[x] = acc[(size_t)r * d + x] / l[r];
                    lse[((size_t)b * H + h) * N + q0 + r] = m[r] + log(l[r]);
                }
            }
    free(m);
    free(l);
    free(acc);
    free(s);
}

/*
 * Backward pass by recompute (LLM explainer page, section 6.2, strategy 1):
 * P is rebuilt row by row from Q and K by the definition, then with upstream
 * gradient dO:
 *   dV_j += P_ij dO_i            dP_ij = dO_i . V_j
 *   D_i = sum_j P_ij dP_ij       dS_ij = P_ij (dP_ij - D_i)
 *   dQ_i = scale sum_j dS_ij K_j dK_j += scale dS_ij Q_i
 * Only query rows i in [row_begin, row_end) contribute: dq rows in that range
 * are exact, dk and dv hold the sum over those rows (all rows when the range
 * is [0, N)).  dq rows in the range, and all of dk and dv, are overwritten.
 * OpenMP splits independent (b, h) heads.
 */
void oracle_attn_bwd_rows(const double *q, const double *k, const double *v,
                          const double *dout, double *dq, double *dk, double *dv,
                          int B, int H, int N, int d, double scale,
                          int row_begin, int row_end, int causal)
{
    int heads = B * H;
#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * (size_t)N);
        double *dp = (double *)malloc(sizeof(double) * (size_t)N);
#pragma omp for schedule(dynamic, 1)
        for (int bh = 0; bh < heads; ++bh) {
            int b = bh / H, h = bh % H;
            for (int j = 0; j < N; ++j)
                for (int x = 0; x < d; ++x) {
                    dk[at(b, j, h, x, N, H, d)] = 0.0;
                    dv[at(b, j, h, x, N, H, d)] = 0.0;
                }
            for (int i = row_begin; i < row_end; ++i) {
                double m, l;
                row_probs(q, k, b, h, i, N, H, d, scale, causal, p, &m, &l);
                const double *doi = dout + at(b, i, h, 0, N, H, d);
                const double *qi = q + at(b, i, h, 0, N, H, d);
                double Di = 0.0;
                for (int j = 0; j < N; ++j) {
                    const double *vj = v + at(b, j, h, 0, N, H, d);
                    double acc = 0.0;
                    for (int x = 0; x < d; ++x) acc += doi[x] * vj[x];
                    dp[j] = acc;
                    Di += p[j] * dp[j];
                }
                double *dqi = dq + at(b, i, h, 0, N, H, d);
                for (int x = 0; x < d; ++x) dqi[x] = 0.0;
                for (int j = 0; j < N; ++j) {
                    double ds = p[j] * (dp[j] - Di);
                    const double *kj = k + at(b, j, h, 0, N, H, d);
                    double *dvj = dv + at(b, j, h, 0, N, H, d);
                    double *dkj = dk + at(b, j, h, 0, N, H, d);
                    for (int x = 0; x < d; ++x) {
                        dvj[x] += p[j] * doi[x];
                        dqi[x] += scale * ds * kj[x];
                        dkj[x] += scale * ds * qi[x];
                    }
                }
            }
        }
        free(p);
        free(dp);
    }
}

/* Backward pass over every query row (see oracle_attn_bwd_rows). */
void oracle_attn_bwd(const double *q, const double *k, const double *v,
                     const double *dout, double *dq, double *dk, double *dv,
                     int B, int H, int N, int d, double scale, int causal)
{
    oracle_attn_bwd_rows(q, k, v, dout, dq, dk, dv, B, H, N, d, scale, 0, N, causal);
}

/* dS for every (b, h): ds is [B, H, N, N] (tests of the row-sum identity). */
void oracle_attn_dscores(const double *q, const double *k, const double *v,
                         const double *dout, double *ds, int B, int H, int N,
                         int d, double scale, int causal)
{
    double *p = (double *)malloc(sizeof(double) * (size_t)N);
    double *dp = (double *)malloc(sizeof(double) * (size_t)N);
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
            for (int i = 0; i < N; ++i) {
                double m, l;
                row_probs(q, k, b, h, i, N, H, d, scale, causal, p, &m, &l);
                const double *doi = dout + at(b, i, h, 0, N, H, d);
                double Di = 0.0;
                for (int j = 0; j < N; ++j) {
                    const double *vj = v + at(b, j, h, 0, N, H, d);
                    double acc = 0.0;
                    for (int x = 0; x < d; ++x) acc += doi[x] * vj[x];
                    dp[j] = acc;
                    Di += p[j] * dp[j];
                }
                double *row = ds + (((size_t)b * H + h) * N + i) * (size_t)N;
                for (int j = 0; j < N; ++j) row[j] = p[j] * (dp[j] - Di);
            }
    free(p);
    free(dp);
}
