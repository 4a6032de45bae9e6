/*
 * gauss_oracle.c -- plain, slow, double-precision CPU oracle for the fused
 * Gaussian kernel reductions.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test-suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no source, header, table or helper
 * with the CUDA library; the two meet only through the seeded input arrays.
 *
 * What it computes is the plain definition, written as the double loop that
 * defines a reduction over the column index j ("Kernel matrix reduction",
 * Implementation sketch, eq. 2: row i reduces the formula over every column j)
 * applied to the Gaussian kernel of the same page's eq. 1 sketch:
 *
 *   sum : out[b,i,c] = sum_j exp(-tau/2 * |x[b,i,:] - y[b,j,:]|^2) * w[b,j,c]
 *   lse : out[b,i,c] = log sum_j w[b,j,c] * exp(-tau/2 * |x_i - y_j|^2)
 *   bwd : the gradient of L = sum_{i,c} g[b,i,c] * sum_out[b,i,c] with respect
 *         to x and to w (the weights are called b on the pages; here w, so as
 *         not to clash with the batch index b).
 *
 * tau is the bandwidth parameter of "Fast Gauss Sums via Flash Attention",
 * Algorithm 1 (input tau > 0); the same kernel is exp(-d^2 / (2 sigma^2)) with
 * tau = 1/sigma^2 in the eq. 1 sketch of "Kernel matrix reduction".
 *
 * Every inner sum over j (or over i, for the weight gradient) is carried out
 * with Neumaier's compensated summation in double, so the oracle's own error
 * stays far below the 1e-5 relative bar it is used to check.  The squared
 * distance is formed in the direct difference form sum_k (x_k - y_k)^2, never
 * through the expanded |x|^2 + |y|^2 - 2 x.y.
 *
 * All arrays are row-major and contiguous:
 *   x [B, M, D], y [B, N, D], w [B, N, C], g [B, M, C],
 *   out [B, R, C] where R = M, or R = n_rows when a row subset is given.
 * rows (optional, may be NULL): indices of the rows i to evaluate, the same
 * subset in every batch.  Rows are evaluated independently in parallel
 * (OpenMP); the arithmetic of one row never depends on the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Neumaier's improvement of Kahan summation: s carries the sum, c the
 * running compensation; the value is s + c. */
typedef struct {
    double s;
    double c;
} comp_sum;

static void cs_add(comp_sum *a, double v)
{
    double t = a->s + v;
    if (fabs(a->s) >= fabs(v))
        a->c += (a->s - t) + v;
    else
        a->c += (v - t) + a->s;
    a->s = t;
}

static double cs_value(const comp_sum *a) { return a->s + a->c; }

/* |p - q|^2 over D coordinates, direct difference form. */
static double sq_dist(const double *p, const double *q, int64_t D)
{
    double acc = 0.0;
    for (int64_t k = 0; k < D; ++k) {
        double d = p[k] - q[k];
        acc += d * d;
    }
    return acc;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Gaussian kernel sum ("Kernel matrix reduction", eq. 1 sketch; output s_m of
 * "Fast Gauss Sums via Flash Attention", Algorithm 1, step 2). */
int oracle_gauss_sum(const double *x, const double *y, const double *w,
                     double *out, int64_t B, int64_t M, int64_t N, int64_t D,
                     int64_t C, double tau, const int64_t *rows,
                     int64_t n_rows)
{
    int64_t R = rows ? n_rows : M;
    if (B < 0 || M < 0 || N < 0 || D < 1 || C < 1 || R < 0 || !(tau > 0.0))
        return 1;
    int bad = 0;
#pragma omp parallel
    {
        comp_sum *acc = (comp_sum *)malloc((size_t)C * sizeof(comp_sum));
        if (!acc) {
#pragma omp atomic write
            bad = 1;
        }
#pragma omp for schedule(dynamic, 4)
        for (int64_t t = 0; t < B * R; ++t) {
            if (!acc)
                continue;
            int64_t bb = t / R;
            int64_t r = t % R;
            int64_t i = rows ? rows[r] : r;
            const double *xi = x + (bb * M + i) * D;
            for (int64_t c = 0; c < C; ++c) {
                acc[c].s = 0.0;
                acc[c].c = 0.0;
            }
            for (int64_t j = 0; j < N; ++j) {
                const double *yj = y + (bb * N + j) * D;
                double k = exp(-0.5 * tau * sq_dist(xi, yj, D));
                const double *wj = w + (bb * N + j) * C;
                for (int64_t c = 0; c < C; ++c)
                    cs_add(&acc[c], k * wj[c]);
            }
            for (int64_t c = 0; c < C; ++c)
                out[(bb * R + r) * C + c] = cs_value(&acc[c]);
        }
        free(acc);
    }
    return bad ? 2 : 0;
}

/* Log-sum-exp reduction ("Kernel matrix reduction", Overview: the reductions
 * covered include log-sum-exp; the .logsumexp() reduction of the LazyTensor
 * API).  The weights enter as log w, so the result is the logarithm of the
 * Gauss sum: out = log sum_j w_j exp(F_ij), F_ij = -tau/2 |x_i - y_j|^2.
 * It is evaluated in two passes, m = max_j F_ij first and then
 * m + log sum_j w_j exp(F_ij - m), so that rows whose every kernel value
 * underflows a double still get their finite logarithm.  N == 0 gives -inf;
 * a non-positive weight sum gives what log gives (-inf or NaN). */
int oracle_gauss_lse(const double *x, const double *y, const double *w,
                     double *out, int64_t B, int64_t M, int64_t N, int64_t D,
                     int64_t C, double tau, const int64_t *rows,
                     int64_t n_rows)
{
    int64_t R = rows ? n_rows : M;
    if (B < 0 || M < 0 || N < 0 || D < 1 || C < 1 || R < 0 || !(tau > 0.0))
        return 1;
    int bad = 0;
#pragma omp parallel
    {
        comp_sum *acc = (comp_sum *)malloc((size_t)C * sizeof(comp_sum));
        if (!acc) {
#pragma omp atomic write
            bad = 1;
        }
#pragma omp for schedule(dynamic, 4)
        for (int64_t t = 0; t < B * R; ++t) {
            if (!acc)
                continue;
            int64_t bb = t / R;
            int64_t r = t % R;
            int64_t i = rows ? rows[r] : r;
            const double *xi = x + (bb * M + i) * D;
            if (N == 0) {
                for (int64_t c = 0; c < C; ++c)
                    out[(bb * R + r) * C + c] = -INFINITY;
                continue;
            }
            double m = -INFINITY;
            for (int64_t j = 0; j < N; ++j) {
                double f = -0.5 * tau * sq_dist(xi, y + (bb * N + j) * D, D);
                if (f > m)
                    m = f;
            }
            for (int64_t c = 0; c < C; ++c) {
                acc[c].s = 0.0;
                acc[c].c = 0.0;
            }
            for (int64_t j = 0; j < N; ++j) {
                double f = -0.5 * tau * sq_dist(xi, y + (bb * N + j) * D, D);
                double e = exp(f - m);
                const double *wj = w + (bb * N + j) * C;
                for (int64_t c = 0; c < C; ++c)
                    cs_add(&acc[c], wj[c] * e);
            }
            for (int64_t c = 0; c < C; ++c)
                out[(bb * R + r) * C + c] = m + log(cs_value(&acc[c]));
        }
        free(acc);
    }
    return bad ? 2 : 0;
}

/* Gradient of L = sum_{i,c} g[i,c] * s[i,c] with s the Gauss sum ("Kernel
 * matrix reduction", Variants: gradients through the same reduction; the
 * torch.autograd.grad example of the LazyTensor API).  Differentiating
 * exp(-tau/2 |x_i - y_j|^2) w_j by hand:
 *
 *   dL/dw[j,c] = sum_i K_ij g[i,c]
 *   dL/dx[i,k] = -tau * sum_j K_ij (sum_c g[i,c] w[j,c]) (x[i,k] - y[j,k])
 *
 * grad_x is [B, R, D] (R = M or n_rows, rows as for the forward); grad_w is
 * [B, Rw, C] over the weight rows wrows (NULL = all N).  Either output may be
 * NULL to skip it. */
int oracle_gauss_sum_bwd(const double *x, const double *y, const double *w,
                         const double *g, double *grad_x, double *grad_w,
                         int64_t B, int64_t M, int64_t N, int64_t D, int64_t C,
                         double tau, const int64_t *rows, int64_t n_rows,
                         const int64_t *wrows, int64_t n_wrows)
{
    int64_t R = rows ? n_rows : M;
    int64_t Rw = wrows ? n_wrows : N;
    if (B < 0 || M < 0 || N < 0 || D < 1 || C < 1 || R < 0 || Rw < 0 ||
        !(tau > 0.0))
        return 1;
    int bad = 0;
    if (grad_x) {
#pragma omp parallel
        {
            comp_sum *acc = (comp_sum *)malloc((size_t)D * sizeof(comp_sum));
            if (!acc) {
#pragma omp atomic write
                bad = 1;
            }
#pragma omp for schedule(dynamic, 4)
            for (int64_t t = 0; t < B * R; ++t) {
                if (!acc)
                    continue;
                int64_t bb = t / R;
                int64_t r = t % R;
                int64_t i = rows ? rows[r] : r;
                const double *xi = x + (bb * M + i) * D;
                const double *gi = g + (bb * M + i) * C;
                for (int64_t k = 0; k < D; ++k) {
                    acc[k].s = 0.0;
                    acc[k].c = 0.0;
                }
                for (int64_t j = 0; j < N; ++j) {
                    const double *yj = y + (bb * N + j) * D;
                    const double *wj = w + (bb * N + j) * C;
                    double kv = exp(-0.5 * tau * sq_dist(xi, yj, D));
                    double gw = 0.0;
                    for (int64_t c = 0; c < C; ++c)
                        gw += gi[c] * wj[c];
                    for (int64_t k = 0; k < D; ++k)
                        cs_add(&acc[k], kv * gw * (xi[k] - yj[k]));
                }
                for (int64_t k = 0; k < D; ++k)
                    grad_x[(bb * R + r) * D + k] = -tau * cs_value(&acc[k]);
            }
            free(acc);
        }
    }
    if (grad_w) {
#pragma omp parallel
        {
            comp_sum *acc = (comp_sum *)malloc((size_t)C * sizeof(comp_sum));
            if (!acc) {
#pragma omp atomic write
                bad = 1;
            }
#pragma omp for schedule(dynamic, 4)
            for (int64_t t = 0; t < B * Rw; ++t) {
                if (!acc)
                    continue;
                int64_t bb = t / Rw;
                int64_t r = t % Rw;
                int64_t j = wrows ? wrows[r] : r;
                const double *yj = y + (bb * N + j) * D;
                for (int64_t c = 0; c < C; ++c) {
                    acc[c].s = 0.0;
                    acc[c].c = 0.0;
                }
                for (int64_t i = 0; i < M; ++i) {
                    const double *xi = x + (bb * M + i) * D;
                    const double *gi = g + (bb * M + i) * C;
                    double kv = exp(-0.5 * tau * sq_dist(xi, yj, D));
                    for (int64_t c = 0; c < C; ++c)
                        cs_add(&acc[c], kv * gi[c]);
                }
                for (int64_t c = 0; c < C; ++c)
                    grad_w[(bb * Rw + r) * C + c] = cs_value(&acc[c]);
            }
            free(acc);
        }
    }
    return bad ? 2 : 0;
}

/* Full vector-Jacobian product of L = sum_{i,c} g[i,c] * s[i,c], s the Gauss
 * sum, extending oracle_gauss_sum_bwd with the source points and the bandwidth
 * ("Kernel matrix reduction", Variants: derivatives of any order through the
 * fused reduction; here the first order in every input):
 *
 *   dL/dy[j,k] = -tau * sum_i K_ij (sum_c g[i,c] w[j,c]) (y[j,k] - x[i,k])
 *   dL/dtau    = -1/2 * sum_b sum_i sum_j K_ij |x_i - y_j|^2 (sum_c g[i,c] w[j,c])
 *
 * grad_y is [B, Rw, D] over the source rows yrows (NULL = all N); grad_tau is
 * one double (NULL to skip).  Either may be NULL. */
int oracle_gauss_sum_vjp_y_tau(const double *x, const double *y, const double *w,
                               const double *g, double *grad_y, double *grad_tau, int64_t B,
                               int64_t M, int64_t N, int64_t D, int64_t C, double tau,
                               const int64_t *yrows, int64_t n_yrows)
{
    int64_t Rw = yrows ? n_yrows : N;
    if (B < 0 || M < 0 || N < 0 || D < 1 || C < 1 || Rw < 0 || !(tau > 0.0))
        return 1;
    int bad = 0;
    if (grad_y) {
#pragma omp parallel
        {
            comp_sum *acc = (comp_sum *)malloc((size_t)D * sizeof(comp_sum));
            if (!acc) {
#pragma omp atomic write
                bad = 1;
            }
#pragma omp for schedule(dynamic, 4)
            for (int64_t t = 0; t < B * Rw; ++t) {
                if (!acc)
                    continue;
                int64_t bb = t / Rw;
                int64_t r = t % Rw;
                int64_t j = yrows ? yrows[r] : r;
                const double *yj = y + (bb * N + j) * D;
                const double *wj = w + (bb * N + j) * C;
                for (int64_t k = 0; k < D; ++k) {
                    acc[k].s = 0.0;
                    acc[k].c = 0.0;
                }
                for (int64_t i = 0; i < M; ++i) {
                    const double *xi = x + (bb * M + i) * D;
                    const double *gi = g + (bb * M + i) * C;
                    double kv = exp(-0.5 * tau * sq_dist(xi, yj, D));
                    double gw = 0.0;
                    for (int64_t c = 0; c < C; ++c)
                        gw += gi[c] * wj[c];
                    for (int64_t k = 0; k < D; ++k)
                        cs_add(&acc[k], kv * gw * (yj[k] - xi[k]));
                }
                for (int64_t k = 0; k < D; ++k)
                    grad_y[(bb * Rw + r) * D + k] = -tau * cs_value(&acc[k]);
            }
            free(acc);
        }
    }
    if (grad_tau) {
        comp_sum total = {0.0, 0.0};
        for (int64_t bb = 0; bb < B; ++bb) {
            for (int64_t i = 0; i < M; ++i) {
                const double *xi = x + (bb * M + i) * D;
                const double *gi = g + (bb * M + i) * C;
                comp_sum row = {0.0, 0.0};
                for (int64_t j = 0; j < N; ++j) {
                    const double *yj = y + (bb * N + j) * D;
                    const double *wj = w + (bb * N + j) * C;
                    double d2 = sq_dist(xi, yj, D);
                    double gw = 0.0;
                    for (int64_t c = 0; c < C; ++c)
                        gw += gi[c] * wj[c];
                    cs_add(&row, exp(-0.5 * tau * d2) * d2 * gw);
                }
                cs_add(&total, cs_value(&row));
            }
        }
        *grad_tau = -0.5 * cs_value(&total);
    }
    return bad ? 2 : 0;
}

/* Gradient of L = sum_{i,c} g[i,c] * lse[i,c], lse the log-sum-exp of
 * oracle_gauss_lse.  With the normalised weights
 *   p_ijc = w[j,c] K_ij / sum_j' w[j',c] K_ij'   (computed max-shifted),
 *   dL/dx[i,k] = -tau * sum_c g[i,c] sum_j p_ijc (x[i,k] - y[j,k])
 *   dL/dy[j,k] = -tau * sum_i sum_c g[i,c] p_ijc (y[j,k] - x[i,k])
 *   dL/dw[j,c] = sum_i g[i,c] p_ijc / w[j,c]  ( = sum_i g[i,c] K_ij / S_ic )
 *   dL/dtau    = -1/2 * sum_i sum_c g[i,c] sum_j p_ijc |x_i - y_j|^2
 * Outputs over all rows ([B,M,D], [B,N,D], [B,N,C], one double); any may be
 * NULL.  Requires w > 0.  Plain triple loops, small sizes only. */
int oracle_gauss_lse_bwd(const double *x, const double *y, const double *w, const double *g,
                         double *grad_x, double *grad_y, double *grad_w, double *grad_tau,
                         int64_t B, int64_t M, int64_t N, int64_t D, int64_t C, double tau)
{
    if (B < 0 || M < 0 || N < 0 || D < 1 || C < 1 || !(tau > 0.0))
        return 1;
    if (grad_x)
        memset(grad_x, 0, (size_t)(B * M * D) * sizeof(double));
    if (grad_y)
        memset(grad_y, 0, (size_t)(B * N * D) * sizeof(double));
    if (grad_w)
        memset(grad_w, 0, (size_t)(B * N * C) * sizeof(double));
    double tau_acc = 0.0;
    double *f = (double *)malloc((size_t)(N > 0 ? N : 1) * sizeof(double));
    if (!f)
        return 2;
    for (int64_t bb = 0; bb < B; ++bb) {
        for (int64_t i = 0; i < M; ++i) {
            const double *xi = x + (bb * M + i) * D;
            double m = -INFINITY;
            for (int64_t j = 0; j < N; ++j) {
                f[j] = -0.5 * tau * sq_dist(xi, y + (bb * N + j) * D, D);
                if (f[j] > m)
                    m = f[j];
            }
            for (int64_t c = 0; c < C; ++c) {
                double gic = g[(bb * M + i) * C + c];
                comp_sum z = {0.0, 0.0};
                for (int64_t j = 0; j < N; ++j)
                    cs_add(&z, w[(bb * N + j) * C + c] * exp(f[j] - m));
                double zs = cs_value(&z);
                for (int64_t j = 0; j < N; ++j) {
                    const double *yj = y + (bb * N + j) * D;
                    double e = exp(f[j] - m);
                    double p = w[(bb * N + j) * C + c] * e / zs;
                    double d2 = sq_dist(xi, yj, D);
                    for (int64_t k = 0; k < D; ++k) {
                        double diff = xi[k] - yj[k];
                        if (grad_x)
                            grad_x[(bb * M + i) * D + k] += -tau * gic * p * diff;
                        if (grad_y)
                            grad_y[(bb * N + j) * D + k] += tau * gic * p * diff;
                    }
                    if (grad_w)
                        grad_w[(bb * N + j) * C + c] += gic * e / zs;
                    tau_acc += -0.5 * gic * p * d2;
                }
            }
        }
    }
    free(f);
    if (grad_tau)
        *grad_tau = tau_acc;
    return 0;
}

/* K-nearest reduction ("Kernel matrix reduction", Overview: the reductions
 * covered include minima and the indices of the K smallest entries per row;
 * the .argmin() reduction of the LazyTensor API).  For each row i the K
 * smallest squared distances |x_i - y_j|^2 over j, ascending, with their
 * indices j; equal distances are ordered by the lower j.  Rows with fewer than
 * K columns get +inf and index -1 in the missing places.  The maximum of the
 * Gaussian kernel over j is exp(-tau/2 * out_d[...,0]), at out_idx[...,0].
 *
 * Two precisions.  oracle_knn computes the distances in double (the plain
 * definition).  oracle_knn_f32 takes float inputs and computes every distance
 * in float with one fixed order of operations -- e_k = x_k - y_k, then
 * d = e_0 * e_0, then d = fma(e_k, e_k, d) for k = 1 .. D-1, each rounded to
 * nearest -- so that an integer result decided by floating point (which index
 * is nearer) is decided in float, the precision of the device kernel.
 * Selection is a plain insertion into a sorted list of K. */
static void knn_insert(double d, int64_t j, double *bd, int64_t *bj, int64_t K)
{
    if (!(d < bd[K - 1] || (d == bd[K - 1] && j < bj[K - 1])))
        return;
    int64_t p = K - 1;
    while (p > 0 && (d < bd[p - 1] || (d == bd[p - 1] && j < bj[p - 1]))) {
        bd[p] = bd[p - 1];
        bj[p] = bj[p - 1];
        --p;
    }
    bd[p] = d;
    bj[p] = j;
}

int oracle_knn(const double *x, const double *y, double *out_d, int64_t *out_idx, int64_t B,
               int64_t M, int64_t N, int64_t D, int64_t K, const int64_t *rows, int64_t n_rows)
{
    int64_t R = rows ? n_rows : M;
    if (B < 0 || M < 0 || N < 0 || D < 1 || K < 1 || R < 0)
        return 1;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t t = 0; t < B * R; ++t) {
        int64_t bb = t / R;
        int64_t r = t % R;
        int64_t i = rows ? rows[r] : r;
        const double *xi = x + (bb * M + i) * D;
        double *bd = out_d + (bb * R + r) * K;
        int64_t *bj = out_idx + (bb * R + r) * K;
        for (int64_t k = 0; k < K; ++k) {
            bd[k] = INFINITY;
            bj[k] = -1;
        }
        for (int64_t j = 0; j < N; ++j)
            knn_insert(sq_dist(xi, y + (bb * N + j) * D, D), j, bd, bj, K);
    }
    return 0;
}

int oracle_knn_f32(const float *x, const float *y, float *out_d, int64_t *out_idx, int64_t B,
                   int64_t M, int64_t N, int64_t D, int64_t K, const int64_t *rows,
                   int64_t n_rows)
{
    int64_t R = rows ? n_rows : M;
    if (B < 0 || M < 0 || N < 0 || D < 1 || K < 1 || R < 0)
        return 1;
    int bad = 0;
#pragma omp parallel
    {
        double *bd = (double *)malloc((size_t)K * sizeof(double));
        if (!bd) {
#pragma omp atomic write
            bad = 1;
        }
#pragma omp for schedule(dynamic, 4)
        for (int64_t t = 0; t < B * R; ++t) {
            if (!bd)
                continue;
            int64_t bb = t / R;
            int64_t r = t % R;
            int64_t i = rows ? rows[r] : r;
            const float *xi = x + (bb * M + i) * D;
            int64_t *bj = out_idx + (bb * R + r) * K;
            for (int64_t k = 0; k < K; ++k) {
                bd[k] = INFINITY;
                bj[k] = -1;
            }
            for (int64_t j = 0; j < N; ++j) {
                const float *yj = y + (bb * N + j) * D;
                float e = xi[0] - yj[0];
                float d = e * e;
                for (int64_t k = 1; k < D; ++k) {
                    e = xi[k] - yj[k];
                    d = fmaf(e, e, d);
                }
                knn_insert((double)d, j, bd, bj, K);
            }
            for (int64_t k = 0; k < K; ++k)
                out_d[(bb * R + r) * K + k] = (float)bd[k];
        }
        free(bd);
    }
    return bad ? 2 : 0;
}

/* Diffusion operator of "FlashDiffusion: Fused Tiled Kernel Spectral
 * Decomposition" (section 2.2, XGEMM: the operator diag(s) K diag(s) applied
 * to a block V; the q and d normalisation passes are kernel applications with
 * V replaced by 1 and by q^-alpha).  The page's section 2.1, which defines s,
 * is missing from the extracted text; the reading taken is the alpha-
 * normalised diffusion map those two passes compute:
 *
 *   q_i = sum_j K_ij                              (pass with V = 1)
 *   d_i = q_i^-alpha * sum_j K_ij q_j^-alpha      (pass with V = q^-alpha)
 *   s_i = q_i^-alpha * d_i^-1/2
 *   A   = diag(s) K diag(s)  (the symmetric form of the Markov matrix of
 *         K_ij / (q_i q_j)^alpha)
 *
 * with K_ij = exp(-tau/2 |x_i - x_j|^2) over one point set x [B, N, D].
 * oracle_diffusion_scales writes q, d and s ([B, N] each, any may be NULL);
 * oracle_diffusion_apply writes out = A V for V [B, N, C]. */
int oracle_diffusion_scales(const double *x, double *q, double *d, double *s, int64_t B,
                            int64_t N, int64_t D, double tau, double alpha)
{
    if (B < 0 || N < 0 || D < 1 || !(tau > 0.0))
        return 1;
    double *qq = (double *)malloc((size_t)((B * N) > 0 ? B * N : 1) * sizeof(double));
    if (!qq)
        return 2;
#pragma omp parallel for schedule(dynamic, 8)
    for (int64_t t = 0; t < B * N; ++t) {
        int64_t bb = t / N, i = t % N;
        comp_sum acc = {0.0, 0.0};
        for (int64_t j = 0; j < N; ++j)
            cs_add(&acc, exp(-0.5 * tau * sq_dist(x + (bb * N + i) * D, x + (bb * N + j) * D, D)));
        qq[t] = cs_value(&acc);
    }
#pragma omp parallel for schedule(dynamic, 8)
    for (int64_t t = 0; t < B * N; ++t) {
        int64_t bb = t / N, i = t % N;
        comp_sum acc = {0.0, 0.0};
        for (int64_t j = 0; j < N; ++j) {
            double k = exp(-0.5 * tau * sq_dist(x + (bb * N + i) * D, x + (bb * N + j) * D, D));
            cs_add(&acc, k * pow(qq[bb * N + j], -alpha));
        }
        double di = pow(qq[t], -alpha) * cs_value(&acc);
        if (q)
            q[t] = qq[t];
        if (d)
            d[t] = di;
        if (s)
            s[t] = pow(qq[t], -alpha) / sqrt(di);
    }
    free(qq);
    return 0;
}

int oracle_diffusion_apply(const double *x, const double *s, const double *v, double *out,
                           int64_t B, int64_t N, int64_t D, int64_t C, double tau)
{
    if (B < 0 || N < 0 || D < 1 || C < 1 || !(tau > 0.0))
        return 1;
    int bad = 0;
#pragma omp parallel
    {
        comp_sum *acc = (comp_sum *)malloc((size_t)C * sizeof(comp_sum));
        if (!acc) {
#pragma omp atomic write
            bad = 1;
        }
#pragma omp for schedule(dynamic, 8)
        for (int64_t t = 0; t < B * N; ++t) {
            if (!acc)
                continue;
            int64_t bb = t / N, i = t % N;
            for (int64_t c = 0; c < C; ++c) {
                acc[c].s = 0.0;
                acc[c].c = 0.0;
            }
            for (int64_t j = 0; j < N; ++j) {
                double k = exp(-0.5 * tau * sq_dist(x + (bb * N + i) * D, x + (bb * N + j) * D, D));
                double ksj = k * s[bb * N + j];
                for (int64_t c = 0; c < C; ++c)
                    cs_add(&acc[c], ksj * v[(bb * N + j) * C + c]);
            }
            for (int64_t c = 0; c < C; ++c)
                out[t * C + c] = s[t] * cs_value(&acc[c]);
        }
        free(acc);
    }
    return bad ? 2 : 0;
}
