/*
 * lnq_oracle.c -- plain FP64 CPU oracle for the GuidedQuant + LNQ hot path.
 *
 * TEST INFRASTRUCTURE ONLY. The test suite, the smoke check and the CPU-baseline leg of the
 * benchmark are the only callers. The CUDA library never links, loads or calls this file, and
 * this file includes nothing from the CUDA library.
 *
 * Every routine is a loop-by-loop transcription of a definition on the source pages, in FP64:
 *
 *   [GQ-eq3]    "GuidedQuant" (jinukkim.me blog), GuidedQuant section, third equation: the
 *               gradient-weighted output error  ||dL/dZ (.) (XW - XW^)||_F^2
 *               = n sum_j (w_j - w^_j)^T F_j (w_j - w^_j), with the sentence after it: the
 *               Fisher blocks are grouped and averaged within each group.
 *   [LNQ-prob]  same post, LNQ section, first equation: per output row j, minimise
 *               ||X w_j - X P c||^2 over a one-hot assignment P (d_in x m) and a codebook c (m).
 *   [LNQ-alg]   same post, LNQ section, second equation: repeat { codebook c <- (P^T H P)^-1 P^T H w;
 *               for i = 1..d_in: assign coordinate i the codeword minimising (w^-w)^T H (w^-w) }.
 *   [GQ-abs]    aitopics "squeezellm" tag page, GuidedQuant abstract: the non-uniform scalar
 *               quantiser decreases its objective monotonically.
 *   [LUT]       same post, LNQ section, last sentence (LNQ runs on the same CUDA kernel as
 *               SqueezeLLM), with the aitopics "squeezellm" tag page, SqueezeLLM abstract
 *               (single-batch inference is memory-bound; weights stored as low-bit indices) and
 *               GANQ abstract (lookup-table based mixed-precision GEMM): the consumer of (C, Q)
 *               multiplies activations by W^ = C[Q] read through each row's codebook.
 *   [GANQ]      scime.ai summary of GANQ (GPU-adaptive non-uniform quantization), Approach
 *               paragraph: the same per-row problem, solved by alternating a Cholesky /
 *               back-substitution assignment of the codebook indices with the closed-form
 *               least-squares codebook update, batched on the GPU. Prior art, here only as a
 *               comparison solver.
 *
 * READINGS (the pages leave these open; each routine below states the one it takes):
 *   R1 groups are contiguous, equal slices of output rows; s_g is the plain mean of squared
 *      gradients over the slice; G absent means every gradient equals 1 (then F = X^T X).
 *   R2 F_g = alpha * X^T diag(s_g) X; alpha = 1 reproduces X^T X when G == 1, alpha = 1/n gives
 *      the F_j of [GQ-eq3].
 *   R3 initial codebook: c_q = sort(w)[floor((2q+1) d / (2m))]; initial assignment: nearest
 *      codeword, ties to the lower index. An iteration starts with the codebook step.
 *   R4 assignment: move coordinate i only if the best candidate strictly lowers the objective;
 *      among equal best candidates take the lowest index; coordinates are visited in natural order.
 *   R5 codebook: solve over non-empty codewords only, empty codewords keep their value, no
 *      damping; a non-positive Cholesky pivot keeps the old codebook and flags the row singular.
 *   R6 packed codes (the pages fix no format): bits = log2(m); each row is a run of 32-bit words
 *      holding floor(32 / bits) codes each, code i of the row in word i / floor(32 / bits) at bit
 *      (i mod floor(32 / bits)) * bits; unused high bits and the tail of the last word are zero.
 *   R7 GANQ-style assignment: the Cholesky factor is lower, F = L L^T, so with r = c[q] - w the
 *      objective is ||L^T r||^2 = sum_i z_i^2, z_i = sum_{k >= i} L[k][i] r_k. Back-substitution
 *      visits i = d-1 down to 0 and gives coordinate i the codeword nearest to
 *      t_i = w_i - (sum_{k > i} L[k][i] r_k) / L[i][i] (the smallest |z_i| given the later
 *      coordinates; ties to the lower index). No damping or preconditioning. An iteration is the
 *      codebook step (R5) followed by this assignment. A non-positive pivot of the factorisation
 *      means the group is not positive definite: its rows keep their codes and report
 *      ORC_ROW_NOT_PD.
 *
 * Build:  gcc -O2 -fopenmp -shared -fPIC lnq_oracle.c -o liblnq_oracle.so -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_ROW_OK 0
#define ORC_ROW_SINGULAR 1
#define ORC_ROW_NOT_PD 2

/* ------------------------------------------------------------------------------------------ */
/* Fisher blocks [GQ-eq3], readings R1, R2                                                      */
/* ------------------------------------------------------------------------------------------ */

/* S[g*n + t] = (1/R) * sum_{j in group g} G[t*d_out + j]^2 with R = d_out / groups (R1).
 * G == NULL means all gradients are 1, so S == 1 (only meaningful with groups == 1). */
void orc_group_scales(const double *G, int64_t n, int64_t d_out, int64_t groups, double *S)
{
    int64_t R = d_out / groups;
    for (int64_t g = 0; g < groups; ++g) {
        for (int64_t t = 0; t < n; ++t) {
            double acc = 0.0;
            if (G == NULL) {
                acc = 1.0;
            } else {
                for (int64_t j = g * R; j < (g + 1) * R; ++j) {
                    double v = G[t * d_out + j];
                    acc += v * v;
                }
                acc /= (double)R;
            }
            S[g * n + t] = acc;
        }
    }
}

/* A block of F = alpha * X^T diag(s) X (R2):
 *   out[a*nb + b] = alpha * sum_t s[t] * XA[t*na + a] * XB[t*nb + b]
 * XA (n x na) and XB (n x nb) are column subsets of X, each row-major and contiguous.
 * Passing XA == XB == X gives the whole matrix. */
void orc_fisher_block(const double *XA, int64_t na, const double *XB, int64_t nb,
                      const double *s, int64_t n, double alpha, double *out)
{
    for (int64_t a = 0; a < na; ++a)
        for (int64_t b = 0; b < nb; ++b)
            out[a * nb + b] = 0.0;
    for (int64_t t = 0; t < n; ++t) {
        const double st = s[t];
        for (int64_t a = 0; a < na; ++a) {
            const double xa = st * XA[t * na + a];
            for (int64_t b = 0; b < nb; ++b)
                out[a * nb + b] += xa * XB[t * nb + b];
        }
    }
    for (int64_t a = 0; a < na; ++a)
        for (int64_t b = 0; b < nb; ++b)
            out[a * nb + b] *= alpha;
}

/* Diagonal of F = alpha * X^T diag(s) X:  out[i] = alpha * sum_t s[t] X[t*d + i]^2. */
void orc_fisher_diag(const double *X, int64_t n, int64_t d, const double *s, double alpha,
                     double *out)
{
    for (int64_t i = 0; i < d; ++i)
        out[i] = 0.0;
    for (int64_t t = 0; t < n; ++t)
        for (int64_t i = 0; i < d; ++i)
            out[i] += s[t] * X[t * d + i] * X[t * d + i];
    for (int64_t i = 0; i < d; ++i)
        out[i] *= alpha;
}

/* ------------------------------------------------------------------------------------------ */
/* LNQ per row [LNQ-prob], [LNQ-alg]                                                           */
/* ------------------------------------------------------------------------------------------ */

/* Row objective J = r^T F r with r = c[q] - w  (the per-row term of [LNQ-prob] written with
 * H = F, as in [GQ-eq3]). */
double orc_objective_row(const double *F, int64_t d, const double *w, const double *c,
                         const uint8_t *q)
{
    double J = 0.0;
    for (int64_t i = 0; i < d; ++i) {
        double ri = c[q[i]] - w[i];
        double acc = 0.0;
        for (int64_t k = 0; k < d; ++k)
            acc += F[i * d + k] * (c[q[k]] - w[k]);
        J += ri * acc;
    }
    return J;
}

static int cmp_double(const void *a, const void *b)
{
    double x = *(const double *)a, y = *(const double *)b;
    return (x > y) - (x < y);
}

/* Initial codebook and assignment (reading R3). */
void orc_init_row(const double *w, int64_t d, int m, double *c, uint8_t *q)
{
    double *sorted = (double *)malloc((size_t)d * sizeof(double));
    memcpy(sorted, w, (size_t)d * sizeof(double));
    qsort(sorted, (size_t)d, sizeof(double), cmp_double);
    for (int j = 0; j < m; ++j)
        c[j] = sorted[((int64_t)(2 * j + 1) * d) / (2 * (int64_t)m)];
    free(sorted);
    for (int64_t i = 0; i < d; ++i) {
        int best = 0;
        double bestdist = fabs(w[i] - c[0]);
        for (int j = 1; j < m; ++j) {
            double dist = fabs(w[i] - c[j]);
            if (dist < bestdist) {
                bestdist = dist;
                best = j;
            }
        }
        q[i] = (uint8_t)best;
    }
}

/* Codebook step of [LNQ-alg]:  c <- (P^T F P)^-1 P^T F w, restricted to the non-empty codewords
 * (reading R5). M and b are formed from their definitions
 *   M[a][b] = sum_{i: q_i=a} sum_{k: q_k=b} F[i][k],   b[a] = sum_{i: q_i=a} sum_k F[i][k] w[k],
 * and the system is solved by an FP64 Cholesky factorisation M = L L^T.
 * Returns ORC_ROW_OK, or ORC_ROW_SINGULAR (codebook left unchanged). */
int orc_codebook_row(const double *F, int64_t d, const double *w, int m, const uint8_t *q,
                     double *c)
{
    double *M = (double *)calloc((size_t)m * m, sizeof(double));
    double *b = (double *)calloc((size_t)m, sizeof(double));
    int *idx = (int *)malloc((size_t)m * sizeof(int));
    int64_t *count = (int64_t *)calloc((size_t)m, sizeof(int64_t));
    for (int64_t i = 0; i < d; ++i) {
        count[q[i]] += 1;
        double fw = 0.0;
        for (int64_t k = 0; k < d; ++k) {
            M[q[i] * m + q[k]] += F[i * d + k];
            fw += F[i * d + k] * w[k];
        }
        b[q[i]] += fw;
    }
    /* Non-empty codewords, in index order. */
    int nn = 0;
    for (int a = 0; a < m; ++a)
        if (count[a] > 0)
            idx[nn++] = a;
    /* Cholesky of the nn x nn principal submatrix, L stored in place (lower triangle). */
    double *L = (double *)calloc((size_t)m * m, sizeof(double));
    int status = ORC_ROW_OK;
    for (int a = 0; a < nn && status == ORC_ROW_OK; ++a) {
        for (int bb = 0; bb <= a; ++bb) {
            double sum = M[idx[a] * m + idx[bb]];
            for (int k = 0; k < bb; ++k)
                sum -= L[a * nn + k] * L[bb * nn + k];
            if (a == bb) {
                if (!(sum > 0.0)) {
                    status = ORC_ROW_SINGULAR;
                    break;
                }
                L[a * nn + a] = sqrt(sum);
            } else {
                L[a * nn + bb] = sum / L[bb * nn + bb];
            }
        }
    }
    if (status == ORC_ROW_OK) {
        double *y = (double *)calloc((size_t)m, sizeof(double));
        for (int a = 0; a < nn; ++a) { /* L y = b */
            double sum = b[idx[a]];
            for (int k = 0; k < a; ++k)
                sum -= L[a * nn + k] * y[k];
            y[a] = sum / L[a * nn + a];
        }
        for (int a = nn - 1; a >= 0; --a) { /* L^T x = y */
            double sum = y[a];
            for (int k = a + 1; k < nn; ++k)
                sum -= L[k * nn + a] * y[k];
            y[a] = sum / L[a * nn + a];
        }
        for (int a = 0; a < nn; ++a)
            c[idx[a]] = y[a];
        free(y);
    }
    free(L);
    free(M);
    free(b);
    free(idx);
    free(count);
    return status;
}

/* Assignment sweep of [LNQ-alg], readings R4, in eager form.
 *
 * With r = c[q] - w and u = F r kept exact, changing coordinate i from its codeword to c_a
 * (delta = c_a - c[q_i]) changes J by  Delta_a = delta * (2 u_i + delta F_ii); this is the exact
 * expansion of (r + delta e_i)^T F (r + delta e_i) - r^T F r, so choosing the argmin of Delta_a is
 * choosing the argmin of the objective in [LNQ-alg]. After a move u += delta * F[:, i].
 *
 * Follow mode: when `hint` is not NULL it holds another solver's assignment after the same sweep.
 * Where the hint differs from this sweep's choice and the hinted candidate's Delta is within
 * max(tie_rel * J_current, tie_abs) of the best Delta, the hint is adopted and counted as a
 * tie-follow; otherwise this sweep's choice is kept and the coordinate is counted as a mismatch.
 * The absolute floor tie_abs matters only for rows whose objective reaches (nearly) zero: there
 * duplicate codewords make many assignments equally good, and the candidates differ only by
 * rounding noise, far below any fraction of J.
 *
 * stats (may be NULL): [0] moves, [1] tie-follows, [2] mismatches, [3] smallest gap
 * (second-best minus best Delta, over all coordinates, in units of J_current) encoded as a
 * double bit pattern.  J_trace (may be NULL, length d+1): J before the sweep and after each
 * coordinate.  Returns J after the sweep (tracked incrementally from J before the sweep). */
double orc_sweep_row(const double *F, int64_t d, const double *w, int m, const double *c,
                     uint8_t *q, const uint8_t *hint, double tie_rel, double tie_abs,
                     int64_t *stats, double *J_trace)
{
    double *u = (double *)malloc((size_t)d * sizeof(double));
    double *delta = (double *)malloc((size_t)m * sizeof(double));
    for (int64_t i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int64_t k = 0; k < d; ++k)
            acc += F[i * d + k] * (c[q[k]] - w[k]);
        u[i] = acc;
    }
    double J = 0.0;
    for (int64_t i = 0; i < d; ++i)
        J += (c[q[i]] - w[i]) * u[i];
    if (J_trace)
        J_trace[0] = J;
    int64_t moves = 0, follows = 0, mismatches = 0;
    double min_gap = INFINITY;
    for (int64_t i = 0; i < d; ++i) {
        const double Fii = F[i * d + i];
        const double cur = c[q[i]];
        /* Staying costs nothing (delta[q_i] == 0 exactly). A candidate replaces the current
         * best only when strictly lower, and indices are scanned upwards, so the result is q_i
         * unless some Delta is negative, and then the lowest index among the minima. */
        int best = q[i];
        double bestD = 0.0;
        for (int a = 0; a < m; ++a) {
            delta[a] = (c[a] - cur) * (2.0 * u[i] + (c[a] - cur) * Fii);
            if (delta[a] < bestD) {
                bestD = delta[a];
                best = a;
            }
        }
        double second = INFINITY;
        for (int a = 0; a < m; ++a)
            if (a != best && delta[a] < second)
                second = delta[a];
        const double band = fmax(tie_rel * fabs(J), tie_abs);
        double gap = (second - bestD) / (fabs(J) > 0.0 ? fabs(J) : 1.0);
        if (gap < min_gap)
            min_gap = gap;
        int chosen = best;
        double chosenD = bestD;
        if (hint != NULL && hint[i] != best) {
            double hD = hint[i] < m ? delta[hint[i]] : INFINITY;
            if (hD - bestD <= band) {
                chosen = hint[i];
                chosenD = hD;
                ++follows;
            } else {
                ++mismatches;
            }
        }
        if (chosen != q[i]) {
            const double dlt = c[chosen] - cur;
            for (int64_t k = 0; k < d; ++k)
                u[k] += dlt * F[k * d + i];
            q[i] = (uint8_t)chosen;
            J += chosenD;
            ++moves;
        }
        if (J_trace)
            J_trace[i + 1] = J;
    }
    if (stats) {
        stats[0] = moves;
        stats[1] = follows;
        stats[2] = mismatches;
        memcpy(&stats[3], &min_gap, sizeof(double));
    }
    free(u);
    free(delta);
    return J;
}

/* Whole LNQ for `nrows` rows that share one F (one Fisher group), [LNQ-alg]:
 *   if init != 0: initial codebook and assignment (R3);
 *   then `iters` times: codebook step, assignment sweep.
 * C (nrows x m) and Q (nrows x d) are in/out. J_hist (nrows x 2*iters, may be NULL) receives the
 * objective after each codebook step and after each sweep, recomputed from its definition.
 * status (nrows, may be NULL) receives ORC_ROW_SINGULAR if any codebook step was singular.
 * Rows run in parallel on `nthreads` OpenMP threads (<= 0: the OpenMP default). */
void orc_lnq_rows(const double *F, int64_t d, const double *W, int64_t nrows, int m, int iters,
                  int init, double *C, uint8_t *Q, double *J_hist, int32_t *status, int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int64_t j = 0; j < nrows; ++j) {
        const double *w = W + j * d;
        double *c = C + j * m;
        uint8_t *q = Q + j * d;
        int32_t st = ORC_ROW_OK;
        if (init)
            orc_init_row(w, d, m, c, q);
        for (int it = 0; it < iters; ++it) {
            if (orc_codebook_row(F, d, w, m, q, c) != ORC_ROW_OK)
                st = ORC_ROW_SINGULAR;
            if (J_hist)
                J_hist[j * 2 * iters + 2 * it] = orc_objective_row(F, d, w, c, q);
            orc_sweep_row(F, d, w, m, c, q, NULL, 0.0, 0.0, NULL, NULL);
            if (J_hist)
                J_hist[j * 2 * iters + 2 * it + 1] = orc_objective_row(F, d, w, c, q);
        }
        if (status)
            status[j] = st;
    }
}

/* One LNQ iteration in follow mode for `nrows` rows sharing F.
 * In:  C_start, Q_start (another solver's state at the start of the iteration) and Q_hint (that
 *      solver's assignment at the end of the iteration); tie_abs (nrows, may be NULL) the
 *      per-row absolute floor of the tie band.
 * Out: C_out = this oracle's codebook step applied to (C_start, Q_start); Q_out = this oracle's
 *      sweep from Q_start with C_out, following the hint inside the tie band; J_out = objective of
 *      (C_out, Q_out) from its definition; stats (nrows x 4) as in orc_sweep_row;
 *      status (nrows) the codebook status. */
void orc_follow_iteration(const double *F, int64_t d, const double *W, int64_t nrows, int m,
                          const double *C_start, const uint8_t *Q_start, const uint8_t *Q_hint,
                          double tie_rel, const double *tie_abs, double *C_out, uint8_t *Q_out,
                          double *J_out,
                          int64_t *stats, int32_t *status, int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int64_t j = 0; j < nrows; ++j) {
        const double *w = W + j * d;
        double *c = C_out + j * m;
        uint8_t *q = Q_out + j * d;
        memcpy(c, C_start + j * m, (size_t)m * sizeof(double));
        memcpy(q, Q_start + j * d, (size_t)d);
        status[j] = orc_codebook_row(F, d, w, m, q, c);
        orc_sweep_row(F, d, w, m, c, q, Q_hint + j * d, tie_rel, tie_abs ? tie_abs[j] : 0.0,
                      stats + 4 * j, NULL);
        J_out[j] = orc_objective_row(F, d, w, c, q);
    }
}

/* ------------------------------------------------------------------------------------------ */
/* GANQ-style comparison solver [GANQ], reading R7                                              */
/* ------------------------------------------------------------------------------------------ */

/* Cholesky factor F = L L^T (Cholesky-Banachiewicz, row by row, FP64); L is d x d row-major,
 * lower, zero above the diagonal. Returns 0, or 1 at the first non-positive pivot (L partial). */
int orc_cholesky(const double *F, int64_t d, double *L)
{
    for (int64_t i = 0; i < d * d; ++i)
        L[i] = 0.0;
    for (int64_t i = 0; i < d; ++i) {
        for (int64_t j = 0; j <= i; ++j) {
            double sum = F[i * d + j];
            for (int64_t k = 0; k < j; ++k)
                sum -= L[i * d + k] * L[j * d + k];
            if (i == j) {
                if (!(sum > 0.0))
                    return 1;
                L[i * d + i] = sqrt(sum);
            } else {
                L[i * d + j] = sum / L[j * d + j];
            }
        }
    }
    return 0;
}

/* Back-substitution assignment of one row (R7): i = d-1 down to 0, coordinate i takes the codeword
 * nearest to t_i = w_i - (sum_{k > i} L[k][i] r_k) / L[i][i], with r_k = c[q_k] - w_k of the
 * coordinates already visited; the cost of candidate a is L[i][i]^2 (c_a - t_i)^2 = z_i^2.
 * Follow mode (hint != NULL): where the hint differs and its cost is within `band` of the best
 * cost, the hint is taken (a tie-follow); otherwise this choice stays (a mismatch).
 * stats (may be NULL): [0] codes changed from the input, [1] tie-follows, [2] mismatches. */
void orc_ganq_assign_row(const double *L, int64_t d, const double *w, int m, const double *c,
                         uint8_t *q, const uint8_t *hint, double band, int64_t *stats)
{
    double *r = (double *)calloc((size_t)d, sizeof(double));
    int64_t changed = 0, follows = 0, mismatches = 0;
    for (int64_t i = d - 1; i >= 0; --i) {
        double s = 0.0;
        for (int64_t k = i + 1; k < d; ++k)
            s += L[k * d + i] * r[k];
        const double lii = L[i * d + i];
        const double t = w[i] - s / lii;
        int best = 0;
        double bcost = lii * lii * (c[0] - t) * (c[0] - t);
        for (int a = 1; a < m; ++a) {
            const double cost = lii * lii * (c[a] - t) * (c[a] - t);
            if (cost < bcost) {
                bcost = cost;
                best = a;
            }
        }
        if (hint != NULL && hint[i] != best) {
            const double hc = lii * lii * (c[hint[i]] - t) * (c[hint[i]] - t);
            if (hc - bcost <= band) {
                best = hint[i];
                follows += 1;
            } else {
                mismatches += 1;
            }
        }
        if (best != q[i])
            changed += 1;
        q[i] = (uint8_t)best;
        r[i] = c[best] - w[i];
    }
    if (stats) {
        stats[0] = changed;
        stats[1] = follows;
        stats[2] = mismatches;
    }
    free(r);
}

/* One GANQ-style iteration for `nrows` rows sharing F (and its factor L, from orc_cholesky):
 * the codebook step (R5) from (C_start, Q_start), then the back-substitution assignment (R7),
 * following Q_hint inside the band (Q_hint may be NULL). band (nrows, may be NULL): per-row
 * absolute tie band. Out: C_out, Q_out, J_out (objective from its definition), stats (nrows x 3),
 * status (nrows: codebook status). */
void orc_ganq_iteration(const double *F, const double *L, int64_t d, const double *W,
                        int64_t nrows, int m, const double *C_start, const uint8_t *Q_start,
                        const uint8_t *Q_hint, const double *band, double *C_out,
                        uint8_t *Q_out, double *J_out, int64_t *stats, int32_t *status,
                        int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int64_t j = 0; j < nrows; ++j) {
        const double *w = W + j * d;
        double *c = C_out + j * m;
        uint8_t *q = Q_out + j * d;
        memcpy(c, C_start + j * m, (size_t)m * sizeof(double));
        memcpy(q, Q_start + j * d, (size_t)d);
        status[j] = orc_codebook_row(F, d, w, m, q, c);
        orc_ganq_assign_row(L, d, w, m, c, q, Q_hint ? Q_hint + j * d : NULL,
                            band ? band[j] : 0.0, stats ? stats + 3 * j : NULL);
        J_out[j] = orc_objective_row(F, d, w, c, q);
    }
}

/* ------------------------------------------------------------------------------------------ */
/* Packed codes and the lookup-table product [LUT], reading R6                                  */
/* ------------------------------------------------------------------------------------------ */

/* P[j*words + w] for rows j < d_out, words = ceil(d_in / floor(32 / bits)) (R6). */
void orc_pack_codes(const uint8_t *Q, int64_t d_out, int64_t d_in, int bits, uint32_t *P)
{
    const int64_t per = 32 / bits;
    const int64_t words = (d_in + per - 1) / per;
    for (int64_t j = 0; j < d_out; ++j) {
        for (int64_t w = 0; w < words; ++w)
            P[j * words + w] = 0u;
        for (int64_t i = 0; i < d_in; ++i) {
            const uint32_t code = (uint32_t)Q[j * d_in + i];
            P[j * words + i / per] |= code << ((i % per) * bits);
        }
    }
}

/* The inverse of orc_pack_codes. */
void orc_unpack_codes(const uint32_t *P, int64_t d_out, int64_t d_in, int bits, uint8_t *Q)
{
    const int64_t per = 32 / bits;
    const int64_t words = (d_in + per - 1) / per;
    const uint32_t mask = (1u << bits) - 1u;
    for (int64_t j = 0; j < d_out; ++j)
        for (int64_t i = 0; i < d_in; ++i)
            Q[j * d_in + i] = (uint8_t)((P[j * words + i / per] >> ((i % per) * bits)) & mask);
}

/* y[b*d_out + j] = sum_i x[b*d_in + i] * C[j*m + Q[j*d_in + i]] for b < nb: the activations times
 * the quantised weights W^[j][i] = c_j[q_ji], read through each row's codebook [LUT]. */
void orc_lut_gemv(const double *x, int64_t nb, const double *C, int m, const uint8_t *Q,
                  int64_t d_out, int64_t d_in, double *y)
{
    for (int64_t b = 0; b < nb; ++b)
        for (int64_t j = 0; j < d_out; ++j) {
            double acc = 0.0;
            for (int64_t i = 0; i < d_in; ++i)
                acc += x[b * d_in + i] * C[j * m + Q[j * d_in + i]];
            y[b * d_out + j] = acc;
        }
}
