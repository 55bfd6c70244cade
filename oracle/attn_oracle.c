/*
 * Exact-attention oracle: a plain, slow, fp64 CPU reference.
 *
 * TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline /
 * reference arm may load this library. It shares no code, header or constant with the CUDA
 * library in exact_attention_138_b200/csrc, and the CUDA library never calls it.
 *
 * What it computes (every step in fp64; inputs are fp32 arrays, which hold fp32 values or
 * bf16-rounded values exactly, and are widened to double on read):
 *
 *   "Attention Mechanism: Revolusi Representasi Sequence", §3 "Scaled Dot-Product Attention:
 *   Formula Inti", Steps 1-4:  score[i][j] = Q[i]·K[j]; scaled by 1/sqrt(d_k) (here an explicit
 *   `scale` argument); row-wise softmax (each row sums to 1); output[i] = sum_j w[i][j]·V[j].
 *   Same page, §4.4 "Causal / Masked Attention": M[i][j] = 0 for j <= i and -inf for j > i.
 *   "Flash Attention Nedir?", section "Online Softmax": the row log-sum-exp, returned as
 *   lse[i] = m_i + ln(sum_j exp(S_ij - m_i)) (natural log).
 *
 * Layout: Q, K, V, dO, O, dQ, dK, dV are (B, H, n, d) row-major; lse and D are (B, H, n).
 *
 * Modes:
 *   oracle_fwd          the definition, with the full n x n score matrix of each (b,h)
 *                       materialised (step 1 for all rows, then mask, then max, then softmax,
 *                       then P·V).
 *   oracle_fwd_rowtiled the same steps applied to one block of query rows at a time, as in the
 *                       row-tiling script of "Efficient Attention" (section "Mengapa Memori
 *                       Attention Tumbuh Kuadratik", part 3 of efficient_attention.py). Each row
 *                       goes through the same operations in the same order, so the result equals
 *                       oracle_fwd bit for bit.
 *   oracle_fwd_online   the online-softmax recurrence of "Attention Mechanism ...", §13
 *                       "FlashAttention — How It Works" (running max m, running sum l, rescaled
 *                       O), over KV column blocks. The page prints the O update without the
 *                       factor exp(m_old - m_new) on the old term; with literal_page_form = 0 the
 *                       factor is applied (the reading that follows from the definition), with
 *                       literal_page_form = 1 the printed form is used as is (tests show that
 *                       form is wrong whenever the running max moves).
 *   oracle_fwd_rows     the definition for a list of sampled query rows only.
 *   oracle_bwd          the exact derivative of the definition (the pages only say that the
 *                       backward pass recomputes the softmax blocks: "Apa itu FlashAttention",
 *                       "Cara kerja teknik Tiling dan Recomputation", item 2). With P the softmax,
 *                       dP = dO·V^T, D_i = sum_j P_ij dP_ij, dS = P∘(dP - D), the gradients are
 *                       dV = P^T·dO, dQ = scale·dS·K, dK = scale·dS^T·Q.
 *   oracle_bwd_query_rows / oracle_bwd_key_rows   the same derivative for sampled rows.
 *   oracle_fwd_ex / oracle_bwd_ex   the definition and its derivative with a generalized mask
 *                       (sliding window of §4.5 "Sparse Attention", causal, none) and different
 *                       query / key lengths (cross-attention, §4.2); see the block before them.
 *   oracle_score_matrix_bytes   the score-matrix size B·H·n²·e of "Calculateur de mémoire
 *                       d'attention", section "La formule".
 *
 * No blocking, fusion or reordering beyond what these definitions state. OpenMP splits
 * independent rows across threads; the arithmetic of each row is the same whatever the thread.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_ERR_ARG 1
#define ORC_ERR_MEM 2

static int oracle_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

int oracle_num_threads(void) { return oracle_threads(); }

void oracle_set_num_threads(int t) {
#ifdef _OPENMP
    if (t > 0) omp_set_num_threads(t);
#else
    (void)t;
#endif
}

/* "Calculateur de mémoire d'attention", "La formule": A = B·H·s²·e bytes. */
double oracle_score_matrix_bytes(double B, double H, double n, double e) { return B * H * n * n * e; }

/* K of one head transposed to (d, n) in fp64, so that a score row can be accumulated over the
 * feature index c in its natural order 0..d-1 for every key at once. */
static double* transpose_keys(const float* K, int n, int d) {
    double* KT = (double*)malloc((size_t)n * d * sizeof(double));
    if (!KT) return NULL;
    for (int j = 0; j < n; ++j)
        for (int c = 0; c < d; ++c) KT[(size_t)c * n + j] = (double)K[(size_t)j * d + c];
    return KT;
}

/* Step 1 + 2 for one query row i: S_i[j] = scale · sum_c q_i[c]·k_j[c], then the causal mask. */
static void score_row(const float* qi, const double* KT, int n, int d, double scale, int causal,
                      int i, double* s) {
    for (int j = 0; j < n; ++j) s[j] = 0.0;
    for (int c = 0; c < d; ++c) {
        const double qc = (double)qi[c];
        const double* kc = KT + (size_t)c * n;
        for (int j = 0; j < n; ++j) s[j] += qc * kc[j];
    }
    for (int j = 0; j < n; ++j) s[j] *= scale;
    if (causal)
        for (int j = i + 1; j < n; ++j) s[j] = -INFINITY;
}

/* Step 3 + 4 for one row, in place: s -> P (row sums to 1). Returns max and sum of exp. */
static void softmax_row(double* s, int n, double* m_out, double* l_out) {
    double m = -INFINITY;
    for (int j = 0; j < n; ++j)
        if (s[j] > m) m = s[j];
    double l = 0.0;
    for (int j = 0; j < n; ++j) {
        s[j] = (s[j] == -INFINITY) ? 0.0 : exp(s[j] - m);
        l += s[j];
    }
    for (int j = 0; j < n; ++j) s[j] /= l;
    *m_out = m;
    *l_out = l;
}

/* Step 5 for one row: o = sum_j p_j · v_j, accumulated in key order. */
static void pv_row(const double* p, const float* V, int n, int d, double* o) {
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    for (int j = 0; j < n; ++j) {
        const double pj = p[j];
        const float* vj = V + (size_t)j * d;
        for (int c = 0; c < d; ++c) o[c] += pj * (double)vj[c];
    }
}

static int check_dims(int B, int H, int n, int d) {
    return (B >= 1 && H >= 1 && n >= 1 && d >= 1) ? ORC_OK : ORC_ERR_ARG;
}

/* One (b,h): the definition over query rows [r0, r1), with the score block S (rows x n)
 * materialised in full before the softmax. */
static int fwd_block(const float* Q, const double* KT, const float* V, int n, int d, double scale,
                     int causal, int r0, int r1, double* O, double* lse) {
    const int rows = r1 - r0;
    double* S = (double*)malloc((size_t)rows * n * sizeof(double));
    if (!S) return ORC_ERR_MEM;
    /* step 1 + 2: all scores of the block */
#pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; ++r)
        score_row(Q + (size_t)(r0 + r) * d, KT, n, d, scale, causal, r0 + r, S + (size_t)r * n);
    /* steps 3-6 */
#pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; ++r) {
        double m, l;
        softmax_row(S + (size_t)r * n, n, &m, &l);
        pv_row(S + (size_t)r * n, V, n, d, O + (size_t)(r0 + r) * d);
        if (lse) lse[r0 + r] = m + log(l);
    }
    free(S);
    return ORC_OK;
}

static int fwd_blocked(const float* Q, const float* K, const float* V, int B, int H, int n, int d,
                       double scale, int causal, int block_rows, double* O, double* lse) {
    if (check_dims(B, H, n, d) || block_rows < 1) return ORC_ERR_ARG;
    for (long bh = 0; bh < (long)B * H; ++bh) {
        const size_t off = (size_t)bh * n * d;
        double* KT = transpose_keys(K + off, n, d);
        if (!KT) return ORC_ERR_MEM;
        for (int r0 = 0; r0 < n; r0 += block_rows) {
            int r1 = r0 + block_rows < n ? r0 + block_rows : n;
            int rc = fwd_block(Q + off, KT, V + off, n, d, scale, causal, r0, r1, O + off,
                               lse ? lse + (size_t)bh * n : NULL);
            if (rc) { free(KT); return rc; }
        }
        free(KT);
    }
    return ORC_OK;
}

int oracle_fwd(const float* Q, const float* K, const float* V, int B, int H, int n, int d,
               double scale, int causal, double* O, double* lse) {
    return fwd_blocked(Q, K, V, B, H, n, d, scale, causal, n, O, lse);
}

int oracle_fwd_rowtiled(const float* Q, const float* K, const float* V, int B, int H, int n, int d,
                        double scale, int causal, int block_rows, double* O, double* lse) {
    return fwd_blocked(Q, K, V, B, H, n, d, scale, causal, block_rows, O, lse);
}

/* The online-softmax recurrence ("Attention Mechanism ...", §13), one query row at a time over
 * KV column blocks of block_cols keys:
 *   S = scaled scores of the block (masked);  m_new = max(m_old, rowmax(S));  P = exp(S - m_new);
 *   l_new = exp(m_old - m_new)·l_old + rowsum(P);
 *   O = (l_old/l_new)·exp(m_old - m_new)·O + (P·V_block)/l_new          (literal_page_form = 0)
 *   O = (l_old/l_new)·O + (P·V_block)/l_new                              (literal_page_form = 1)
 * exp(m_old - m_new) is taken as 0 while m_old = -inf (nothing accumulated yet). */
int oracle_fwd_online(const float* Q, const float* K, const float* V, int B, int H, int n, int d,
                      double scale, int causal, int block_cols, int literal_page_form, double* O,
                      double* lse) {
    if (check_dims(B, H, n, d) || block_cols < 1) return ORC_ERR_ARG;
    int fail = 0;
    for (long bh = 0; bh < (long)B * H; ++bh) {
        const size_t off = (size_t)bh * n * d;
        const float* Qh = Q + off;
        const float* Kh = K + off;
        const float* Vh = V + off;
#pragma omp parallel
        {
            double* s = (double*)malloc((size_t)block_cols * sizeof(double));
            double* pv = (double*)malloc((size_t)d * sizeof(double));
            if (!s || !pv) {
#pragma omp atomic write
                fail = 1;
            } else {
#pragma omp for schedule(static)
                for (int i = 0; i < n; ++i) {
                    const float* qi = Qh + (size_t)i * d;
                    double* o = O + off + (size_t)i * d;
                    double m_old = -INFINITY, l_old = 0.0;
                    for (int c = 0; c < d; ++c) o[c] = 0.0;
                    for (int j0 = 0; j0 < n; j0 += block_cols) {
                        const int j1 = j0 + block_cols < n ? j0 + block_cols : n;
                        double bmax = -INFINITY;
                        for (int j = j0; j < j1; ++j) {
                            double acc = 0.0;
                            const float* kj = Kh + (size_t)j * d;
                            for (int c = 0; c < d; ++c) acc += (double)qi[c] * (double)kj[c];
                            acc *= scale;
                            if (causal && j > i) acc = -INFINITY;
                            s[j - j0] = acc;
                            if (acc > bmax) bmax = acc;
                        }
                        const double m_new = bmax > m_old ? bmax : m_old;
                        if (m_new == -INFINITY) continue; /* block fully masked, nothing seen yet */
                        double rowsum = 0.0;
                        for (int c = 0; c < d; ++c) pv[c] = 0.0;
                        for (int j = j0; j < j1; ++j) {
                            const double p = (s[j - j0] == -INFINITY) ? 0.0 : exp(s[j - j0] - m_new);
                            rowsum += p;
                            const float* vj = Vh + (size_t)j * d;
                            for (int c = 0; c < d; ++c) pv[c] += p * (double)vj[c];
                        }
                        const double alpha = (m_old == -INFINITY) ? 0.0 : exp(m_old - m_new);
                        const double l_new = alpha * l_old + rowsum;
                        const double keep = literal_page_form ? (l_old / l_new)
                                                              : (l_old / l_new) * alpha;
                        for (int c = 0; c < d; ++c) o[c] = keep * o[c] + pv[c] / l_new;
                        m_old = m_new;
                        l_old = l_new;
                    }
                    if (lse) lse[(size_t)bh * n + i] = m_old + log(l_old);
                }
            }
            free(s);
            free(pv);
        }
        if (fail) return ORC_ERR_MEM;
    }
    return ORC_OK;
}

/* The definition for sampled query rows: rows[t] = bh*n + i. Outputs o_rows (nrows, d) and
 * lse_rows (nrows). Each row is computed exactly as oracle_fwd computes it. */
int oracle_fwd_rows(const float* Q, const float* K, const float* V, int B, int H, int n, int d,
                    double scale, int causal, const int64_t* rows, int nrows, double* o_rows,
                    double* lse_rows) {
    if (check_dims(B, H, n, d) || nrows < 0) return ORC_ERR_ARG;
    for (int t = 0; t < nrows; ++t)
        if (rows[t] < 0 || rows[t] >= (int64_t)B * H * n) return ORC_ERR_ARG;
    int fail = 0;
#pragma omp parallel
    {
        double* s = (double*)malloc((size_t)n * sizeof(double));
        double* kt = (double*)malloc((size_t)n * d * sizeof(double));
        long cached_bh = -1;
        if (!s || !kt) {
#pragma omp atomic write
            fail = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int t = 0; t < nrows; ++t) {
                const long bh = (long)(rows[t] / n);
                const int i = (int)(rows[t] % n);
                const size_t off = (size_t)bh * n * d;
                if (bh != cached_bh) {
                    for (int j = 0; j < n; ++j)
                        for (int c = 0; c < d; ++c)
                            kt[(size_t)c * n + j] = (double)K[off + (size_t)j * d + c];
                    cached_bh = bh;
                }
                double m, l;
                score_row(Q + off + (size_t)i * d, kt, n, d, scale, causal, i, s);
                softmax_row(s, n, &m, &l);
                pv_row(s, V + off, n, d, o_rows + (size_t)t * d);
                lse_rows[t] = m + log(l);
            }
        }
        free(s);
        free(kt);
    }
    return fail ? ORC_ERR_MEM : ORC_OK;
}

/* Backward, per query row i of one head: P_i (softmax row), dP_i[j] = dO_i·v_j,
 * D_i = sum_j P_ij dP_ij, dS_i[j] = P_ij (dP_ij - D_i). Writes P_i into p and dS_i into ds. */
static void bwd_row(const float* qi, const float* doi, const double* KT, const float* V, int n,
                    int d, double scale, int causal, int i, double* p, double* ds, double* D_out) {
    double m, l;
    score_row(qi, KT, n, d, scale, causal, i, p);
    softmax_row(p, n, &m, &l);
    double D = 0.0;
    for (int j = 0; j < n; ++j) {
        double dp = 0.0;
        const float* vj = V + (size_t)j * d;
        for (int c = 0; c < d; ++c) dp += (double)doi[c] * (double)vj[c];
        ds[j] = dp;
        D += p[j] * dp;
    }
    for (int j = 0; j < n; ++j) ds[j] = p[j] * (ds[j] - D);
    if (D_out) *D_out = D;
}

/* Full backward with P and dS of each (b,h) materialised (n x n each). */
int oracle_bwd(const float* Q, const float* K, const float* V, const float* dO, int B, int H, int n,
               int d, double scale, int causal, double* dQ, double* dK, double* dV, double* Dvec) {
    if (check_dims(B, H, n, d)) return ORC_ERR_ARG;
    for (long bh = 0; bh < (long)B * H; ++bh) {
        const size_t off = (size_t)bh * n * d;
        double* KT = transpose_keys(K + off, n, d);
        double* P = (double*)malloc((size_t)n * n * sizeof(double));
        double* dS = (double*)malloc((size_t)n * n * sizeof(double));
        if (!KT || !P || !dS) { free(KT); free(P); free(dS); return ORC_ERR_MEM; }
#pragma omp parallel for schedule(static)
        for (int i = 0; i < n; ++i)
            bwd_row(Q + off + (size_t)i * d, dO + off + (size_t)i * d, KT, V + off, n, d, scale,
                    causal, i, P + (size_t)i * n, dS + (size_t)i * n,
                    Dvec ? Dvec + (size_t)bh * n + i : NULL);
        /* dQ_i = scale · sum_j dS_ij k_j */
#pragma omp parallel for schedule(static)
        for (int i = 0; i < n; ++i) {
            double* g = dQ + off + (size_t)i * d;
            for (int c = 0; c < d; ++c) g[c] = 0.0;
            for (int j = 0; j < n; ++j) {
                const double w = dS[(size_t)i * n + j];
                const float* kj = K + off + (size_t)j * d;
                for (int c = 0; c < d; ++c) g[c] += w * (double)kj[c];
            }
            for (int c = 0; c < d; ++c) g[c] *= scale;
        }
        /* dK_j = scale · sum_i dS_ij q_i ;  dV_j = sum_i P_ij dO_i */
#pragma omp parallel for schedule(static)
        for (int j = 0; j < n; ++j) {
            double* gk = dK + off + (size_t)j * d;
            double* gv = dV + off + (size_t)j * d;
            for (int c = 0; c < d; ++c) { gk[c] = 0.0; gv[c] = 0.0; }
            for (int i = 0; i < n; ++i) {
                const double ws = dS[(size_t)i * n + j];
                const double wp = P[(size_t)i * n + j];
                const float* qi = Q + off + (size_t)i * d;
                const float* doi = dO + off + (size_t)i * d;
                for (int c = 0; c < d; ++c) {
                    gk[c] += ws * (double)qi[c];
                    gv[c] += wp * (double)doi[c];
                }
            }
            for (int c = 0; c < d; ++c) gk[c] *= scale;
        }
        free(KT); free(P); free(dS);
    }
    return ORC_OK;
}

/* dQ for sampled query rows (rows[t] = bh*n + i); also returns D_i. */
int oracle_bwd_query_rows(const float* Q, const float* K, const float* V, const float* dO, int B,
                          int H, int n, int d, double scale, int causal, const int64_t* rows,
                          int nrows, double* dq_rows, double* D_rows) {
    if (check_dims(B, H, n, d) || nrows < 0) return ORC_ERR_ARG;
    for (int t = 0; t < nrows; ++t)
        if (rows[t] < 0 || rows[t] >= (int64_t)B * H * n) return ORC_ERR_ARG;
    int fail = 0;
#pragma omp parallel
    {
        double* p = (double*)malloc((size_t)n * sizeof(double));
        double* ds = (double*)malloc((size_t)n * sizeof(double));
        double* kt = (double*)malloc((size_t)n * d * sizeof(double));
        long cached_bh = -1;
        if (!p || !ds || !kt) {
#pragma omp atomic write
            fail = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int t = 0; t < nrows; ++t) {
                const long bh = (long)(rows[t] / n);
                const int i = (int)(rows[t] % n);
                const size_t off = (size_t)bh * n * d;
                if (bh != cached_bh) {
                    for (int j = 0; j < n; ++j)
                        for (int c = 0; c < d; ++c)
                            kt[(size_t)c * n + j] = (double)K[off + (size_t)j * d + c];
                    cached_bh = bh;
                }
                double D;
                bwd_row(Q + off + (size_t)i * d, dO + off + (size_t)i * d, kt, V + off, n, d, scale,
                        causal, i, p, ds, &D);
                double* g = dq_rows + (size_t)t * d;
                for (int c = 0; c < d; ++c) g[c] = 0.0;
                for (int j = 0; j < n; ++j) {
                    const float* kj = K + off + (size_t)j * d;
                    for (int c = 0; c < d; ++c) g[c] += ds[j] * (double)kj[c];
                }
                for (int c = 0; c < d; ++c) g[c] *= scale;
                if (D_rows) D_rows[t] = D;
            }
        }
        free(p); free(ds); free(kt);
    }
    return fail ? ORC_ERR_MEM : ORC_OK;
}

/* dK and dV for sampled key rows of ONE head bh: keys[t] in [0, n). Every query row that can
 * see one of the keys (all rows; with the causal mask, rows i >= min key) is recomputed in full
 * (P_i, D_i, dS_i); the key rows' sums are then taken over i in increasing order. */
int oracle_bwd_key_rows(const float* Q, const float* K, const float* V, const float* dO, int B,
                        int H, int n, int d, double scale, int causal, long bh,
                        const int32_t* keys, int nkeys, double* dk_rows, double* dv_rows) {
    if (check_dims(B, H, n, d) || nkeys < 1 || bh < 0 || bh >= (long)B * H) return ORC_ERR_ARG;
    int kmin = n;
    for (int t = 0; t < nkeys; ++t) {
        if (keys[t] < 0 || keys[t] >= n) return ORC_ERR_ARG;
        if (keys[t] < kmin) kmin = keys[t];
    }
    const int i0 = causal ? kmin : 0;
    const int nq = n - i0;
    const size_t off = (size_t)bh * n * d;
    double* KT = transpose_keys(K + off, n, d);
    /* per query row, the P and dS entries at the sampled keys */
    double* Psel = (double*)malloc((size_t)nq * nkeys * sizeof(double));
    double* dSsel = (double*)malloc((size_t)nq * nkeys * sizeof(double));
    if (!KT || !Psel || !dSsel) { free(KT); free(Psel); free(dSsel); return ORC_ERR_MEM; }
    int fail = 0;
#pragma omp parallel
    {
        double* p = (double*)malloc((size_t)n * sizeof(double));
        double* ds = (double*)malloc((size_t)n * sizeof(double));
        if (!p || !ds) {
#pragma omp atomic write
            fail = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (int r = 0; r < nq; ++r) {
                const int i = i0 + r;
                bwd_row(Q + off + (size_t)i * d, dO + off + (size_t)i * d, KT, V + off, n, d,
                        scale, causal, i, p, ds, NULL);
                for (int t = 0; t < nkeys; ++t) {
                    Psel[(size_t)r * nkeys + t] = p[keys[t]];
                    dSsel[(size_t)r * nkeys + t] = ds[keys[t]];
                }
            }
        }
        free(p); free(ds);
    }
    if (!fail) {
#pragma omp parallel for schedule(static)
        for (int t = 0; t < nkeys; ++t) {
            double* gk = dk_rows + (size_t)t * d;
            double* gv = dv_rows + (size_t)t * d;
            for (int c = 0; c < d; ++c) { gk[c] = 0.0; gv[c] = 0.0; }
            for (int r = 0; r < nq; ++r) {
                const int i = i0 + r;
                const double ws = dSsel[(size_t)r * nkeys + t];
                const double wp = Psel[(size_t)r * nkeys + t];
                const float* qi = Q + off + (size_t)i * d;
                const float* doi = dO + off + (size_t)i * d;
                for (int c = 0; c < d; ++c) {
                    gk[c] += ws * (double)qi[c];
                    gv[c] += wp * (double)doi[c];
                }
            }
            for (int c = 0; c < d; ++c) gk[c] *= scale;
        }
    }
    free(KT); free(Psel); free(dSsel);
    return fail ? ORC_ERR_MEM : ORC_OK;
}

/* ------------------------------------------------------------------------------------------
 * Mask and shape variants: sliding-window attention ("Attention Mechanism ...", §4.5 Sparse
 * Attention, "Sliding Window: only neighbours ±w") and cross-attention with different query and
 * key lengths (§4.2: Q from the decoder, K and V from the encoder).
 * Query i (of nq) is aligned with key i + (nk - nq) (the last query with the last key); key j is
 * visible iff  (i + off) - wl <= j <= (i + off) + wr, where a negative wl or wr means unbounded.
 * (wl, wr) = (-1, 0) is the causal mask of §4.4 when nq = nk; (-1, -1) is no mask; (w, w) is the
 * page's ±w window. A row that sees no key gets O = 0 and LSE = -inf.
 * Q is (B,H,nq,d); K and V are (B,H,nk,d).
 * ------------------------------------------------------------------------------------------ */
static int visible(long i, long j, long off, long wl, long wr) {
    const long c = i + off;
    if (wl >= 0 && j < c - wl) return 0;
    if (wr >= 0 && j > c + wr) return 0;
    return 1;
}

/* Definition for one query row over nk keys with the generalized mask. */
static void attend_row_ex(const float* qi, const double* KT, const float* V, int nk, int d,
                          double scale, long i, long off, long wl, long wr, double* s, double* o,
                          double* lse) {
    for (int j = 0; j < nk; ++j) s[j] = 0.0;
    for (int c = 0; c < d; ++c) {
        const double qc = (double)qi[c];
        const double* kc = KT + (size_t)c * nk;
        for (int j = 0; j < nk; ++j) s[j] += qc * kc[j];
    }
    int any = 0;
    for (int j = 0; j < nk; ++j) {
        if (visible(i, j, off, wl, wr)) { s[j] *= scale; any = 1; }
        else s[j] = -INFINITY;
    }
    if (!any) {
        for (int c = 0; c < d; ++c) o[c] = 0.0;
        *lse = -INFINITY;
        return;
    }
    double m, l;
    softmax_row(s, nk, &m, &l);
    pv_row(s, V, nk, d, o);
    *lse = m + log(l);
}

int oracle_fwd_ex(const float* Q, const float* K, const float* V, int B, int H, int nq, int nk,
                  int d, double scale, int wl, int wr, double* O, double* lse) {
    if (B < 1 || H < 1 || nq < 1 || nk < 1 || d < 1) return ORC_ERR_ARG;
    const long off = (long)nk - (long)nq;
    int fail = 0;
    for (long bh = 0; bh < (long)B * H; ++bh) {
        double* KT = transpose_keys(K + (size_t)bh * nk * d, nk, d);
        if (!KT) return ORC_ERR_MEM;
#pragma omp parallel
        {
            double* s = (double*)malloc((size_t)nk * sizeof(double));
            if (!s) {
#pragma omp atomic write
                fail = 1;
            } else {
#pragma omp for schedule(static)
                for (int i = 0; i < nq; ++i)
                    attend_row_ex(Q + ((size_t)bh * nq + i) * d, KT, V + (size_t)bh * nk * d, nk, d,
                                  scale, i, off, wl, wr, s, O + ((size_t)bh * nq + i) * d,
                                  lse + (size_t)bh * nq + i);
            }
            free(s);
        }
        free(KT);
        if (fail) return ORC_ERR_MEM;
    }
    return ORC_OK;
}

/* Exact derivative with the generalized mask; P and dS of each (b,h) materialised (nq x nk). */
int oracle_bwd_ex(const float* Q, const float* K, const float* V, const float* dO, int B, int H,
                  int nq, int nk, int d, double scale, int wl, int wr, double* dQ, double* dK,
                  double* dV) {
    if (B < 1 || H < 1 || nq < 1 || nk < 1 || d < 1) return ORC_ERR_ARG;
    const long off = (long)nk - (long)nq;
    for (long bh = 0; bh < (long)B * H; ++bh) {
        const float* Qh = Q + (size_t)bh * nq * d;
        const float* dOh = dO + (size_t)bh * nq * d;
        const float* Kh = K + (size_t)bh * nk * d;
        const float* Vh = V + (size_t)bh * nk * d;
        double* KT = transpose_keys(Kh, nk, d);
        double* P = (double*)malloc((size_t)nq * nk * sizeof(double));
        double* dS = (double*)malloc((size_t)nq * nk * sizeof(double));
        if (!KT || !P || !dS) { free(KT); free(P); free(dS); return ORC_ERR_MEM; }
#pragma omp parallel for schedule(static)
        for (int i = 0; i < nq; ++i) {
            double* p = P + (size_t)i * nk;
            double* ds = dS + (size_t)i * nk;
            /* P row: the softmax of the masked scores (all zero for a row with no key) */
            for (int j = 0; j < nk; ++j) p[j] = 0.0;
            for (int c = 0; c < d; ++c) {
                const double qc = (double)Qh[(size_t)i * d + c];
                const double* kc = KT + (size_t)c * nk;
                for (int j = 0; j < nk; ++j) p[j] += qc * kc[j];
            }
            int any = 0;
            for (int j = 0; j < nk; ++j) {
                if (visible(i, j, off, wl, wr)) { p[j] *= scale; any = 1; }
                else p[j] = -INFINITY;
            }
            if (any) {
                double m, l;
                softmax_row(p, nk, &m, &l);
            } else {
                for (int j = 0; j < nk; ++j) p[j] = 0.0;
            }
            double D = 0.0;
            for (int j = 0; j < nk; ++j) {
                double dp = 0.0;
                for (int c = 0; c < d; ++c) dp += (double)dOh[(size_t)i * d + c] * (double)Vh[(size_t)j * d + c];
                ds[j] = dp;
                D += p[j] * dp;
            }
            for (int j = 0; j < nk; ++j) ds[j] = p[j] * (ds[j] - D);
        }
#pragma omp parallel for schedule(static)
        for (int i = 0; i < nq; ++i) {
            double* g = dQ + ((size_t)bh * nq + i) * d;
            for (int c = 0; c < d; ++c) g[c] = 0.0;
            for (int j = 0; j < nk; ++j) {
                const double w = dS[(size_t)i * nk + j];
                for (int c = 0; c < d; ++c) g[c] += w * (double)Kh[(size_t)j * d + c];
            }
            for (int c = 0; c < d; ++c) g[c] *= scale;
        }
#pragma omp parallel for schedule(static)
        for (int j = 0; j < nk; ++j) {
            double* gk = dK + ((size_t)bh * nk + j) * d;
            double* gv = dV + ((size_t)bh * nk + j) * d;
            for (int c = 0; c < d; ++c) { gk[c] = 0.0; gv[c] = 0.0; }
            for (int i = 0; i < nq; ++i) {
                const double ws = dS[(size_t)i * nk + j], wp = P[(size_t)i * nk + j];
                for (int c = 0; c < d; ++c) {
                    gk[c] += ws * (double)Qh[(size_t)i * d + c];
                    gv[c] += wp * (double)dOh[(size_t)i * d + c];
                }
            }
            for (int c = 0; c < d; ++c) gk[c] *= scale;
        }
        free(KT); free(P); free(dS);
    }
    return ORC_OK;
}
