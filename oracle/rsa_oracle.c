/*
 * rsa_oracle.c -- plain, slow, fp64 CPU oracle for Ring Self-Attention (RSA).
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or load this file:
 * only the test suite, the package's smoke check and the benchmark's CPU-baseline leg use it.
 * It shares no code, header, table or helper with the CUDA library.
 *
 * What RSA computes. "Sequence Parallelism: Making 4D Parallelism Possible" (Li, Xue et al.,
 * 2021; review page, Abstract and "Proposed method") splits the input sequence into chunks,
 * one per device, and passes attention embeddings around a ring while computing
 * self-attention (Ring Self-Attention). The pages give no equation and mention no
 * approximation, so the reading taken here is exact softmax attention per (batch, head):
 *
 *   S_ij = (sum_k Q_ik K_jk) / sqrt(d)          (causal: S_ij = -inf for j > i)
 *   m_i  = max_j S_ij,  l_i = sum_j exp(S_ij - m_i)
 *   P_ij = exp(S_ij - m_i) / l_i,  lse_i = m_i + ln l_i
 *   O_i  = sum_j P_ij V_j
 *
 * Backward (softmax Jacobian, derived by hand; the pages state only that the backward pass
 * runs on the same ring):
 *
 *   dV_j  = sum_i P_ij dO_i
 *   dP_ij = dO_i . V_j
 *   D_i   = sum_j P_ij dP_ij
 *   dS_ij = P_ij (dP_ij - D_i)
 *   dQ_i  = (1/sqrt d) sum_j dS_ij K_j
 *   dK_j  = (1/sqrt d) sum_i dS_ij Q_i
 *
 * Two families of entry points:
 *   - *_plain: the definitions above, row by row, for every (batch, head).
 *   - *_ring : the ring schedule taken literally. The sequence of length L is cut into N
 *     chunks of c = L/N rows; chunk n builds its c x L score slab by visiting key chunk
 *     m = (n + s) mod N at ring step s = 0..N-1 (causal: steps with m > n are skipped and
 *     block m = n is masked inside), takes the row softmax over the whole slab, then
 *     accumulates O_n = sum_s P_n[:, block m] V_m over a second ring pass. The backward
 *     pass recomputes the slab, forms dP and dS on the same schedule, accumulates dQ_n along
 *     the ring and adds each step's share into dK_m and dV_m.
 *   - *_rows / *_keys: the plain definitions for a chosen subset of query rows or key rows of
 *     one head (large problems are checked on samples).
 *
 * Layout: every tensor is [BH][L][d] (row-major, d fastest), fp64. lse is [BH][L].
 * Return value: 0 on success, -1 on a bad argument, -2 when memory could not be allocated.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define IDX(bh, i, k) (((size_t)(bh) * (size_t)L + (size_t)(i)) * (size_t)d + (size_t)(k))

/* ------------------------------------------------------------------ threads */

void rsa_oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int rsa_oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------ one query row */

/* Scores of query row i of one head against keys 0..jmax-1 (the rest are masked). */
static void score_row(const double *q, const double *K, long L, long d, long jmax,
                      double scale, double *s) {
    for (long j = 0; j < L; ++j) {
        if (j < jmax) {
            double acc = 0.0;
            for (long k = 0; k < d; ++k) acc += q[k] * K[j * d + k];
            s[j] = acc * scale;
        } else {
            s[j] = -INFINITY;
        }
    }
}

/* Row softmax of s[0..L) in place; returns lse = m + ln l. */
static double softmax_row(double *s, long L) {
    double m = -INFINITY;
    for (long j = 0; j < L; ++j)
        if (s[j] > m) m = s[j];
    double l = 0.0;
    for (long j = 0; j < L; ++j) {
        double e = (s[j] == -INFINITY) ? 0.0 : exp(s[j] - m);
        s[j] = e;
        l += e;
    }
    for (long j = 0; j < L; ++j) s[j] /= l;
    return m + log(l);
}

/* ------------------------------------------------------------------ plain forward */

int rsa_oracle_forward_plain(const double *Q, const double *K, const double *V, long BH,
                             long L, long d, int causal, double *O, double *lse) {
    if (!Q || !K || !V || !O || BH < 0 || L < 0 || d <= 0) return -1;
    const double scale = 1.0 / sqrt((double)d);
    int err = 0;
#pragma omp parallel for schedule(dynamic) collapse(2)
    for (long bh = 0; bh < BH; ++bh) {
        for (long i = 0; i < L; ++i) {
            double *p = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
            if (!p) {
#pragma omp atomic write
                err = -2;
                continue;
            }
            const double *Kh = K + IDX(bh, 0, 0);
            const double *Vh = V + IDX(bh, 0, 0);
            long jmax = causal ? i + 1 : L;
            score_row(Q + IDX(bh, i, 0), Kh, L, d, jmax, scale, p);
            double r = softmax_row(p, L);
            if (lse) lse[bh * L + i] = r;
            for (long k = 0; k < d; ++k) {
                double acc = 0.0;
                for (long j = 0; j < L; ++j) acc += p[j] * Vh[j * d + k];
                O[IDX(bh, i, k)] = acc;
            }
            free(p);
        }
    }
    return err;
}

/* Softmax probabilities P [BH][L][L] (small problems only; for the softmax pins). */
int rsa_oracle_probs_plain(const double *Q, const double *K, long BH, long L, long d,
                           int causal, double *P) {
    if (!Q || !K || !P || BH < 0 || L < 0 || d <= 0) return -1;
    const double scale = 1.0 / sqrt((double)d);
    for (long bh = 0; bh < BH; ++bh)
        for (long i = 0; i < L; ++i) {
            double *p = P + ((size_t)bh * L + i) * L;
            score_row(Q + IDX(bh, i, 0), K + IDX(bh, 0, 0), L, d, causal ? i + 1 : L, scale, p);
            softmax_row(p, L);
        }
    return 0;
}

/* ------------------------------------------------------------------ plain backward */

/* One head's backward. Row i of P is rebuilt from the scores, then dP, D_i and dS follow
 * from the definitions; dK and dV are summed over i in ascending order. */
static int backward_head(const double *Qh, const double *Kh, const double *Vh,
                         const double *dOh, long L, long d, int causal, double *dQh,
                         double *dKh, double *dVh) {
    const double scale = 1.0 / sqrt((double)d);
    double *p = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    double *dp = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    if (!p || !dp) {
        free(p);
        free(dp);
        return -2;
    }
    memset(dKh, 0, sizeof(double) * (size_t)L * (size_t)d);
    memset(dVh, 0, sizeof(double) * (size_t)L * (size_t)d);
    for (long i = 0; i < L; ++i) {
        const double *qi = Qh + i * d;
        const double *doi = dOh + i * d;
        score_row(qi, Kh, L, d, causal ? i + 1 : L, scale, p);
        softmax_row(p, L);
        double D = 0.0;
        for (long j = 0; j < L; ++j) {
            double acc = 0.0;
            for (long k = 0; k < d; ++k) acc += doi[k] * Vh[j * d + k];
            dp[j] = acc;
            D += p[j] * acc;
        }
        for (long k = 0; k < d; ++k) dQh[i * d + k] = 0.0;
        for (long j = 0; j < L; ++j) {
            double ds = p[j] * (dp[j] - D);
            for (long k = 0; k < d; ++k) {
                dQh[i * d + k] += scale * ds * Kh[j * d + k];
                dKh[j * d + k] += scale * ds * qi[k];
                dVh[j * d + k] += p[j] * doi[k];
            }
        }
    }
    free(p);
    free(dp);
    return 0;
}

int rsa_oracle_backward_plain(const double *Q, const double *K, const double *V,
                              const double *dO, long BH, long L, long d, int causal,
                              double *dQ, double *dK, double *dV) {
    if (!Q || !K || !V || !dO || !dQ || !dK || !dV || BH < 0 || L < 0 || d <= 0) return -1;
    int err = 0;
#pragma omp parallel for schedule(dynamic)
    for (long bh = 0; bh < BH; ++bh) {
        int e = backward_head(Q + IDX(bh, 0, 0), K + IDX(bh, 0, 0), V + IDX(bh, 0, 0),
                              dO + IDX(bh, 0, 0), L, d, causal, dQ + IDX(bh, 0, 0),
                              dK + IDX(bh, 0, 0), dV + IDX(bh, 0, 0));
        if (e) {
#pragma omp atomic write
            err = e;
        }
    }
    return err;
}

/* ------------------------------------------------------------------ ring schedule */

/* Score slab of chunk n of one head: S_n [c][L], built block by block in ring order. */
static void ring_slab(const double *Qh, const double *Kh, long L, long d, long N, long n,
                      int causal, double scale, double *S) {
    const long c = L / N;
    for (long s = 0; s < N; ++s) {
        const long m = (n + s) % N;
        for (long ii = 0; ii < c; ++ii) {
            const long i = n * c + ii;
            for (long jj = 0; jj < c; ++jj) {
                const long j = m * c + jj;
                double v;
                if (causal && (m > n || j > i)) {
                    v = -INFINITY;
                } else {
                    double acc = 0.0;
                    for (long k = 0; k < d; ++k) acc += Qh[i * d + k] * Kh[j * d + k];
                    v = acc * scale;
                }
                S[ii * L + j] = v;
            }
        }
    }
}

int rsa_oracle_forward_ring(const double *Q, const double *K, const double *V, long BH,
                            long L, long d, long N, int causal, double *O, double *lse) {
    if (!Q || !K || !V || !O || BH < 0 || L < 0 || d <= 0 || N <= 0 || L % N) return -1;
    const double scale = 1.0 / sqrt((double)d);
    const long c = L / N;
    int err = 0;
#pragma omp parallel for schedule(dynamic) collapse(2)
    for (long bh = 0; bh < BH; ++bh) {
        for (long n = 0; n < N; ++n) {
            double *S = (double *)malloc(sizeof(double) * (size_t)(c * L > 0 ? c * L : 1));
            if (!S) {
#pragma omp atomic write
                err = -2;
                continue;
            }
            const double *Qh = Q + IDX(bh, 0, 0), *Kh = K + IDX(bh, 0, 0);
            const double *Vh = V + IDX(bh, 0, 0);
            /* ring pass 1: the slab */
            ring_slab(Qh, Kh, L, d, N, n, causal, scale, S);
            /* softmax over the full key length */
            for (long ii = 0; ii < c; ++ii) {
                double r = softmax_row(S + ii * L, L);
                if (lse) lse[bh * L + n * c + ii] = r;
            }
            /* ring pass 2: O_n = sum_s P_n[:, block m] V_m */
            for (long ii = 0; ii < c; ++ii)
                for (long k = 0; k < d; ++k) O[IDX(bh, n * c + ii, k)] = 0.0;
            for (long s = 0; s < N; ++s) {
                const long m = (n + s) % N;
                if (causal && m > n) continue;
                for (long ii = 0; ii < c; ++ii)
                    for (long k = 0; k < d; ++k) {
                        double acc = 0.0;
                        for (long jj = 0; jj < c; ++jj)
                            acc += S[ii * L + m * c + jj] * Vh[(m * c + jj) * d + k];
                        O[IDX(bh, n * c + ii, k)] += acc;
                    }
            }
            free(S);
        }
    }
    return err;
}

int rsa_oracle_backward_ring(const double *Q, const double *K, const double *V,
                             const double *dO, long BH, long L, long d, long N, int causal,
                             double *dQ, double *dK, double *dV) {
    if (!Q || !K || !V || !dO || !dQ || !dK || !dV || BH < 0 || L < 0 || d <= 0 || N <= 0 ||
        L % N)
        return -1;
    const double scale = 1.0 / sqrt((double)d);
    const long c = L / N;
    int err = 0;
#pragma omp parallel for schedule(dynamic)
    for (long bh = 0; bh < BH; ++bh) {
        const double *Qh = Q + IDX(bh, 0, 0), *Kh = K + IDX(bh, 0, 0);
        const double *Vh = V + IDX(bh, 0, 0), *dOh = dO + IDX(bh, 0, 0);
        double *dQh = dQ + IDX(bh, 0, 0), *dKh = dK + IDX(bh, 0, 0), *dVh = dV + IDX(bh, 0, 0);
        size_t slab = (size_t)(c * L > 0 ? c * L : 1);
        double *P = (double *)malloc(sizeof(double) * slab);
        double *dP = (double *)malloc(sizeof(double) * slab);
        double *Dv = (double *)malloc(sizeof(double) * (size_t)(c > 0 ? c : 1));
        if (!P || !dP || !Dv) {
            free(P);
            free(dP);
            free(Dv);
#pragma omp atomic write
            err = -2;
            continue;
        }
        memset(dKh, 0, sizeof(double) * (size_t)L * (size_t)d);
        memset(dVh, 0, sizeof(double) * (size_t)L * (size_t)d);
        for (long n = 0; n < N; ++n) {
            /* recompute the slab and its softmax */
            ring_slab(Qh, Kh, L, d, N, n, causal, scale, P);
            for (long ii = 0; ii < c; ++ii) softmax_row(P + ii * L, L);
            /* dP_n[:, block m] = dO_n V_m^T, ring order */
            for (long s = 0; s < N; ++s) {
                const long m = (n + s) % N;
                for (long ii = 0; ii < c; ++ii)
                    for (long jj = 0; jj < c; ++jj) {
                        double acc = 0.0;
                        if (!(causal && m > n))
                            for (long k = 0; k < d; ++k)
                                acc += dOh[(n * c + ii) * d + k] * Vh[(m * c + jj) * d + k];
                        dP[ii * L + m * c + jj] = acc;
                    }
            }
            /* D_i = sum_j P_ij dP_ij, then dS = P (dP - D) in place of dP */
            for (long ii = 0; ii < c; ++ii) {
                double D = 0.0;
                for (long j = 0; j < L; ++j) D += P[ii * L + j] * dP[ii * L + j];
                Dv[ii] = D;
            }
            for (long ii = 0; ii < c; ++ii)
                for (long j = 0; j < L; ++j) dP[ii * L + j] = P[ii * L + j] * (dP[ii * L + j] - Dv[ii]);
            /* dQ_n = scale * sum_s dS_n[:, block m] K_m; dK_m, dV_m gather step s's share */
            for (long ii = 0; ii < c; ++ii)
                for (long k = 0; k < d; ++k) dQh[(n * c + ii) * d + k] = 0.0;
            for (long s = 0; s < N; ++s) {
                const long m = (n + s) % N;
                if (causal && m > n) continue;
                for (long ii = 0; ii < c; ++ii) {
                    const long i = n * c + ii;
                    for (long jj = 0; jj < c; ++jj) {
                        const long j = m * c + jj;
                        const double ds = dP[ii * L + j], p = P[ii * L + j];
                        for (long k = 0; k < d; ++k) {
                            dQh[i * d + k] += scale * ds * Kh[j * d + k];
                            dKh[j * d + k] += scale * ds * Qh[i * d + k];
                            dVh[j * d + k] += p * dOh[i * d + k];
                        }
                    }
                }
            }
        }
        free(P);
        free(dP);
        free(Dv);
    }
    return err;
}

/* ------------------------------------------------------------------ sampled rows of one head */

/* O_i and lse_i for the listed query rows of one head (pointers at the head's base). */
int rsa_oracle_forward_rows(const double *Qh, const double *Kh, const double *Vh, long L,
                            long d, int causal, const long *rows, long nrows, double *O_rows,
                            double *lse_rows) {
    if (!Qh || !Kh || !Vh || !rows || !O_rows || L <= 0 || d <= 0) return -1;
    const double scale = 1.0 / sqrt((double)d);
    int err = 0;
#pragma omp parallel for schedule(dynamic)
    for (long r = 0; r < nrows; ++r) {
        const long i = rows[r];
        if (i < 0 || i >= L) {
#pragma omp atomic write
            err = -1;
            continue;
        }
        double *p = (double *)malloc(sizeof(double) * (size_t)L);
        if (!p) {
#pragma omp atomic write
            err = -2;
            continue;
        }
        score_row(Qh + i * d, Kh, L, d, causal ? i + 1 : L, scale, p);
        double lr = softmax_row(p, L);
        if (lse_rows) lse_rows[r] = lr;
        for (long k = 0; k < d; ++k) {
            double acc = 0.0;
            for (long j = 0; j < L; ++j) acc += p[j] * Vh[j * d + k];
            O_rows[r * d + k] = acc;
        }
        free(p);
    }
    return err;
}

/* dQ_i for the listed query rows of one head. */
int rsa_oracle_backward_rows(const double *Qh, const double *Kh, const double *Vh,
                             const double *dOh, long L, long d, int causal, const long *rows,
                             long nrows, double *dQ_rows) {
    if (!Qh || !Kh || !Vh || !dOh || !rows || !dQ_rows || L <= 0 || d <= 0) return -1;
    const double scale = 1.0 / sqrt((double)d);
    int err = 0;
#pragma omp parallel for schedule(dynamic)
    for (long r = 0; r < nrows; ++r) {
        const long i = rows[r];
        if (i < 0 || i >= L) {
#pragma omp atomic write
            err = -1;
            continue;
        }
        double *p = (double *)malloc(sizeof(double) * (size_t)L);
        double *dp = (double *)malloc(sizeof(double) * (size_t)L);
        if (!p || !dp) {
            free(p);
            free(dp);
#pragma omp atomic write
            err = -2;
            continue;
        }
        score_row(Qh + i * d, Kh, L, d, causal ? i + 1 : L, scale, p);
        softmax_row(p, L);
        double D = 0.0;
        for (long j = 0; j < L; ++j) {
            double acc = 0.0;
            for (long k = 0; k < d; ++k) acc += dOh[i * d + k] * Vh[j * d + k];
            dp[j] = acc;
            D += p[j] * acc;
        }
        for (long k = 0; k < d; ++k) dQ_rows[r * d + k] = 0.0;
        for (long j = 0; j < L; ++j) {
            const double ds = p[j] * (dp[j] - D);
            for (long k = 0; k < d; ++k) dQ_rows[r * d + k] += scale * ds * Kh[j * d + k];
        }
        free(p);
        free(dp);
    }
    return err;
}

/* dK_j and dV_j for the listed key rows of one head. Every query row contributes, so the
 * row statistics lse_i and D_i are computed for all i first (O(L^2 d)). */
int rsa_oracle_backward_keys(const double *Qh, const double *Kh, const double *Vh,
                             const double *dOh, long L, long d, int causal, const long *keys,
                             long nkeys, double *dK_rows, double *dV_rows) {
    if (!Qh || !Kh || !Vh || !dOh || !keys || !dK_rows || !dV_rows || L <= 0 || d <= 0)
        return -1;
    const double scale = 1.0 / sqrt((double)d);
    double *lse = (double *)malloc(sizeof(double) * (size_t)L);
    double *Dv = (double *)malloc(sizeof(double) * (size_t)L);
    if (!lse || !Dv) {
        free(lse);
        free(Dv);
        return -2;
    }
    int err = 0;
#pragma omp parallel for schedule(dynamic)
    for (long i = 0; i < L; ++i) {
        double *p = (double *)malloc(sizeof(double) * (size_t)L);
        if (!p) {
#pragma omp atomic write
            err = -2;
            continue;
        }
        score_row(Qh + i * d, Kh, L, d, causal ? i + 1 : L, scale, p);
        lse[i] = softmax_row(p, L);
        double D = 0.0;
        for (long j = 0; j < L; ++j) {
            if (p[j] == 0.0) continue;
            double acc = 0.0;
            for (long k = 0; k < d; ++k) acc += dOh[i * d + k] * Vh[j * d + k];
            D += p[j] * acc;
        }
        Dv[i] = D;
        free(p);
    }
    if (err) {
        free(lse);
        free(Dv);
        return err;
    }
#pragma omp parallel for schedule(dynamic)
    for (long r = 0; r < nkeys; ++r) {
        const long j = keys[r];
        if (j < 0 || j >= L) {
#pragma omp atomic write
            err = -1;
            continue;
        }
        for (long k = 0; k < d; ++k) {
            dK_rows[r * d + k] = 0.0;
            dV_rows[r * d + k] = 0.0;
        }
        for (long i = causal ? j : 0; i < L; ++i) {
            double sc = 0.0, dp = 0.0;
            for (long k = 0; k < d; ++k) {
                sc += Qh[i * d + k] * Kh[j * d + k];
                dp += dOh[i * d + k] * Vh[j * d + k];
            }
            const double p = exp(sc * scale - lse[i]);
            const double ds = p * (dp - Dv[i]);
            for (long k = 0; k < d; ++k) {
                dK_rows[r * d + k] += scale * ds * Qh[i * d + k];
                dV_rows[r * d + k] += p * dOh[i * d + k];
            }
        }
    }
    free(lse);
    free(Dv);
    return err;
}

/* ------------------------------------------------------------------ linear layers of the block
 *
 * Sequence parallelism splits the whole Transformer block, not only its attention, by the
 * sequence (review page, Abstract: every device holds a chunk of the sequence; the layers
 * other than self-attention work on their own chunk's rows with no exchange). The block's
 * linear layers (the query/key/value projection, the output projection and the two layers of
 * the MLP) are, on a chunk of M rows,
 *
 *   Y[m][n] = act( sum_k X[m][k] W[n][k] + b[n] ) + R[m][n]
 *
 * with W [N][K] (out x in), an optional bias b [N] (NULL: none), an optional residual R [M][N]
 * (NULL: none) and act the identity or, when gelu != 0, the exact GELU
 *   GELU(x) = x Phi(x) = x (1 + erf(x / sqrt 2)) / 2
 * (Phi the standard normal distribution function). Row-major fp64 throughout.
 */
int rsa_oracle_linear(const double *X, const double *W, const double *b, const double *R, long M,
                      long N, long K, int gelu, double *Y) {
    if (!X || !W || !Y || M <= 0 || N <= 0 || K <= 0) return -1;
#pragma omp parallel for schedule(static)
    for (long m = 0; m < M; ++m) {
        for (long n = 0; n < N; ++n) {
            double acc = 0.0;
            for (long k = 0; k < K; ++k) acc += X[m * K + k] * W[n * K + k];
            if (b) acc += b[n];
            if (gelu) acc = 0.5 * acc * (1.0 + erf(acc / sqrt(2.0)));
            if (R) acc += R[m * N + n];
            Y[m * N + n] = acc;
        }
    }
    return 0;
}
