/*
 * WKV7 oracle: plain fp64 CPU definition of the RWKV-7 time-mix recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header or constant with the
 * CUDA library.
 *
 * The recurrence (per batch b, head h; S is N x N, row i = value index,
 * column j = key index):
 *
 *     S_t = S_{t-1} (diag(w_t) + a_t b_t^T) + v_t k_t^T
 *     y_t = S_t r_t                    (read after the write of token t)
 *
 * Sources: the state is updated by a "diagonal plus rank one" transition
 * (Paper Review: RWKV-7 "Goose" with Expressive Dynamic State Evolution,
 * section "Architecture"), combining decay, selective forgetting and value
 * insertion per head (same review, section "The approach"), then read out by
 * the receptance vector (same section).  The vector decay, the in-context
 * learning rate and the separate removal / write keys come from the Elamur
 * Research summary of RWKV-7 "Goose" (section "Summary").  None of the pages
 * prints the equation: the form above is the reading of those passages with
 * the transition applied from the right (it acts on the key axis).
 *
 * Row i of S evolves on its own, given the shared per-token vectors:
 *     p     = sum_j S[i,j] a[j]                      (S_{t-1} a_t, row i)
 *     S[i,j] = S[i,j] w[j] + p b[j] + v[i] k[j]
 *     y[i]  = sum_j S[i,j] r[j]
 * The oracle is written that way: one scalar loop per row, fp64 throughout.
 *
 * Layouts (all contiguous, row-major):
 *     r, w, k, v, a, b, y, dy and the matching gradients: [B, T, H, N]
 *     s0, sT, dsT, ds0: [B, H, N, N]   (state S[b][h][i][j])
 * A NULL s0 means a zero initial state; a NULL dsT means a zero gradient.
 */
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define IDX_TOK(b, t, h, n) ((((size_t)(b) * T + (t)) * H + (h)) * N + (n))
#define IDX_ST(b, h, i, j) ((((size_t)(b) * H + (h)) * N + (i)) * N + (j))

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* Forward: y[B,T,H,N], sT[B,H,N,N] (sT may be NULL). */
void oracle_forward(int B, int T, int H, int N,
                    const double *r, const double *w, const double *k,
                    const double *v, const double *a, const double *b,
                    const double *s0, double *y, double *sT) {
    long nheads = (long)B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < nheads; ++bh) {
        int bb = (int)(bh / H), h = (int)(bh % H);
        double *S = (double *)malloc(sizeof(double) * (size_t)N);
        for (int i = 0; i < N; ++i) {
            for (int j = 0; j < N; ++j)
                S[j] = s0 ? s0[IDX_ST(bb, h, i, j)] : 0.0;
            for (int t = 0; t < T; ++t) {
                const double *at = a + IDX_TOK(bb, t, h, 0);
                const double *bt = b + IDX_TOK(bb, t, h, 0);
                const double *wt = w + IDX_TOK(bb, t, h, 0);
                const double *kt = k + IDX_TOK(bb, t, h, 0);
                const double *rt = r + IDX_TOK(bb, t, h, 0);
                double vi = v[IDX_TOK(bb, t, h, i)];
                double p = 0.0;
                for (int j = 0; j < N; ++j) p += S[j] * at[j];
                double acc = 0.0;
                for (int j = 0; j < N; ++j) {
                    S[j] = S[j] * wt[j] + p * bt[j] + vi * kt[j];
                    acc += S[j] * rt[j];
                }
                y[IDX_TOK(bb, t, h, i)] = acc;
            }
            if (sT)
                for (int j = 0; j < N; ++j) sT[IDX_ST(bb, h, i, j)] = S[j];
        }
        free(S);
    }
}

/*
 * Backward of L = sum(dy * y) + sum(dsT * sT) with respect to every input
 * and s0, by reverse-time accumulation.  With g = dL/dS_t (row i):
 *
 *   g += dy_t[i] r_t                  (y_t = S_t r_t)
 *   dr_t[j] += dy_t[i] S_t[i,j]
 *   dv_t[i]  = sum_j g[j] k_t[j]
 *   dk_t[j] += v_t[i] g[j]
 *   dw_t[j] += S_{t-1}[i,j] g[j]
 *   db_t[j] += p_t g[j],      p_t = sum_j S_{t-1}[i,j] a_t[j]
 *   dp       = sum_j g[j] b_t[j]
 *   da_t[j] += dp S_{t-1}[i,j]
 *   g        = g * w_t + dp a_t          (dL/dS_{t-1} through S_t)
 *
 * and ds0[i,:] = g after token 0.  The states S_t of row i are recomputed
 * by the forward loop above and kept for every t (fp64, T*N per row).
 * Gradient outputs are overwritten, not accumulated into.
 */
void oracle_backward(int B, int T, int H, int N,
                     const double *r, const double *w, const double *k,
                     const double *v, const double *a, const double *b,
                     const double *s0, const double *dy, const double *dsT,
                     double *dr, double *dw, double *dk, double *dv,
                     double *da, double *db, double *ds0) {
    long nheads = (long)B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < nheads; ++bh) {
        int bb = (int)(bh / H), h = (int)(bh % H);
        /* hist[t+1] = S_t of the current row; hist[0] = S_{-1} = s0 row. */
        double *hist = (double *)malloc(sizeof(double) * (size_t)(T + 1) * N);
        double *g = (double *)malloc(sizeof(double) * (size_t)N);
        for (int t = 0; t < T; ++t)
            for (int j = 0; j < N; ++j) {
                size_t o = IDX_TOK(bb, t, h, j);
                dr[o] = dw[o] = dk[o] = da[o] = db[o] = 0.0;
            }
        for (int i = 0; i < N; ++i) {
            double *S = hist;
            for (int j = 0; j < N; ++j) S[j] = s0 ? s0[IDX_ST(bb, h, i, j)] : 0.0;
            for (int t = 0; t < T; ++t) {
                const double *prev = hist + (size_t)t * N;
                double *cur = hist + (size_t)(t + 1) * N;
                const double *at = a + IDX_TOK(bb, t, h, 0);
                double p = 0.0;
                for (int j = 0; j < N; ++j) p += prev[j] * at[j];
                double vi = v[IDX_TOK(bb, t, h, i)];
                for (int j = 0; j < N; ++j)
                    cur[j] = prev[j] * w[IDX_TOK(bb, t, h, j)] + p * b[IDX_TOK(bb, t, h, j)] +
                             vi * k[IDX_TOK(bb, t, h, j)];
            }
            for (int j = 0; j < N; ++j) g[j] = dsT ? dsT[IDX_ST(bb, h, i, j)] : 0.0;
            for (int t = T - 1; t >= 0; --t) {
                const double *prev = hist + (size_t)t * N;
                const double *cur = hist + (size_t)(t + 1) * N;
                const double *rt = r + IDX_TOK(bb, t, h, 0);
                const double *wt = w + IDX_TOK(bb, t, h, 0);
                const double *kt = k + IDX_TOK(bb, t, h, 0);
                const double *at = a + IDX_TOK(bb, t, h, 0);
                const double *bt = b + IDX_TOK(bb, t, h, 0);
                double dyi = dy[IDX_TOK(bb, t, h, i)];
                double vi = v[IDX_TOK(bb, t, h, i)];
                for (int j = 0; j < N; ++j) {
                    g[j] += dyi * rt[j];
                    dr[IDX_TOK(bb, t, h, j)] += dyi * cur[j];
                }
                double dvi = 0.0, p = 0.0, dp = 0.0;
                for (int j = 0; j < N; ++j) {
                    dvi += g[j] * kt[j];
                    p += prev[j] * at[j];
                    dp += g[j] * bt[j];
                }
                dv[IDX_TOK(bb, t, h, i)] = dvi;
                for (int j = 0; j < N; ++j) {
                    size_t o = IDX_TOK(bb, t, h, j);
                    dk[o] += vi * g[j];
                    dw[o] += prev[j] * g[j];
                    db[o] += p * g[j];
                    da[o] += dp * prev[j];
                }
                for (int j = 0; j < N; ++j) g[j] = g[j] * wt[j] + dp * at[j];
            }
            for (int j = 0; j < N; ++j) ds0[IDX_ST(bb, h, i, j)] = g[j];
        }
        free(hist);
        free(g);
    }
}
