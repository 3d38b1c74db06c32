/*
 * kan_oracle.c -- plain, slow, fp64 CPU oracle for the B-spline
 * Kolmogorov-Arnold (KAN) layer, forward and backward.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and
 * the benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or constant with the CUDA path, and the CUDA path never
 * calls it.
 *
 * What it computes (sources):
 *   - KAN layer y_j = sum_i phi_ji(x_i), one learnable univariate function per
 *     edge: InKAN landing page, "What is a KAN?" section.
 *   - phi_ji is a cubic B-spline with local support (~4 knot intervals):
 *     same page and section.
 *   - phi_ji(x) = sum_m coef[j,i,m] B_m(x) on a uniform grid of G intervals on
 *     [lo,hi], extended by k knots each side (G+k basis functions), plus an
 *     optional SiLU base branch sum_i w_base[j,i] silu(x_i): the plainest
 *     reading of the "predefined, bounded grids" of the UKAN abstract ("Want
 *     to train KANS at scale? Now UKAN!", Abstract) and of the layer the task
 *     statement defines.
 *   - B_m evaluated by the Cox-de Boor recursion, k sequential passes for
 *     degree k: FlashKAN abstract (mlsift "GPU kernel" listing).  The
 *     recursion itself is not printed on any page; the textbook form
 *     (de Boor, "A Practical Guide to Splines", ch. IX) is used:
 *         N_{j,0}(x) = 1 if t_j <= x < t_{j+1} else 0          (half-open)
 *         N_{j,p}(x) = (x - t_j)/(t_{j+p} - t_j) N_{j,p-1}(x)
 *                    + (t_{j+p+1} - x)/(t_{j+p+1} - t_{j+1}) N_{j+1,p-1}(x)
 *         N'_{j,k}(x) = k/(t_{j+k} - t_j) N_{j,k-1}(x)
 *                     - k/(t_{j+k+1} - t_{j+1}) N_{j+1,k-1}(x)
 *   - gradients: dcoef[j,i,m] = sum_b B_m(x_bi) dY_bj,
 *     dw_base[j,i] = sum_b silu(x_bi) dY_bj,
 *     dx_bi = sum_j dY_bj (sum_m coef[j,i,m] B'_m(x_bi) + w_base[j,i] silu'(x_bi)).
 *
 * Every sum runs in fp64 in ascending index order.  Terms whose basis value is
 * exactly 0 are skipped (adding an exact 0 does not change an fp64 sum).
 * Work is split over batch rows across pthreads; batch-reduced gradients are
 * per-thread partials added in thread order.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_EXPORT __attribute__((visibility("default")))

/* ------------------------------------------------------------------------ */
/* Knots and basis                                                           */
/* ------------------------------------------------------------------------ */

/* Uniform knots t_j = lo + (j - k)(hi - lo)/G, j = 0 .. G+2k, each computed
 * directly from j (no running sum).  t must hold G+2k+1 values. */
ORACLE_EXPORT void kan_oracle_knots(int G, int k, double lo, double hi, double* t)
{
    for (int j = 0; j <= G + 2 * k; ++j)
        t[j] = lo + ((double)(j - k) * (hi - lo)) / (double)G;
}

/* Cox-de Boor evaluation of all G+k degree-k B-splines at x, and their
 * derivatives.  B and dB (either may be NULL) receive G+k values each.
 * work must hold 2*(G+2k) doubles. */
static void basis_eval(double x, int G, int k, const double* t, double* B, double* dB, double* work)
{
    const int nint = G + 2 * k;          /* number of knot intervals */
    double* cur = work;                  /* N_{., p}   */
    double* prev = work + nint;          /* N_{., p-1} */

    /* degree 0: indicator of the half-open interval [t_j, t_{j+1}) */
    for (int j = 0; j < nint; ++j)
        cur[j] = (t[j] <= x && x < t[j + 1]) ? 1.0 : 0.0;

    for (int p = 1; p <= k; ++p) {
        double* tmp = prev; prev = cur; cur = tmp;
        const int n = nint - p;          /* number of degree-p functions */
        if (p == k && dB) {
            /* derivative of the degree-k functions from the degree-(k-1) ones */
            for (int j = 0; j < n; ++j) {
                double a = (double)k / (t[j + k] - t[j]);
                double c = (double)k / (t[j + k + 1] - t[j + 1]);
                dB[j] = a * prev[j] - c * prev[j + 1];
            }
        }
        for (int j = 0; j < n; ++j) {
            /* a term whose lower-degree factor is exactly 0 is 0 (this also
             * keeps x = +-inf, where (x - t_j) is infinite, at 0) */
            double left = prev[j] != 0.0 ? (x - t[j]) / (t[j + p] - t[j]) * prev[j] : 0.0;
            double right = prev[j + 1] != 0.0 ? (t[j + p + 1] - x) / (t[j + p + 1] - t[j + 1]) * prev[j + 1] : 0.0;
            cur[j] = left + right;
        }
    }
    if (k == 0 && dB)
        for (int j = 0; j < nint; ++j) dB[j] = 0.0;
    if (B)
        for (int j = 0; j < G + k; ++j) B[j] = cur[j];
}

/* Public single-point evaluation: B[G+k], dB[G+k] (either may be NULL). */
ORACLE_EXPORT void kan_oracle_basis(double x, int G, int k, double lo, double hi, double* B, double* dB)
{
    double* t = (double*)malloc(sizeof(double) * (size_t)(G + 2 * k + 1));
    double* work = (double*)malloc(sizeof(double) * (size_t)(2 * (G + 2 * k)));
    kan_oracle_knots(G, k, lo, hi, t);
    basis_eval(x, G, k, t, B, dB, work);
    free(t);
    free(work);
}

/* Vector form: x[n] -> B[n, G+k], dB[n, G+k] (either may be NULL). */
ORACLE_EXPORT void kan_oracle_basis_many(const double* x, int64_t n, int G, int k, double lo, double hi,
                                         double* B, double* dB)
{
    const int nb = G + k;
    double* t = (double*)malloc(sizeof(double) * (size_t)(G + 2 * k + 1));
    double* work = (double*)malloc(sizeof(double) * (size_t)(2 * (G + 2 * k)));
    kan_oracle_knots(G, k, lo, hi, t);
    for (int64_t e = 0; e < n; ++e)
        basis_eval(x[e], G, k, t, B ? B + e * nb : NULL, dB ? dB + e * nb : NULL, work);
    free(t);
    free(work);
}

/* SiLU and its derivative, written from the definitions
 * silu(x) = x * sigma(x), sigma(x) = 1/(1+exp(-x)),
 * silu'(x) = sigma(x) (1 + x (1 - sigma(x))). */
static double silu(double x) { return x / (1.0 + exp(-x)); }
static double dsilu(double x)
{
    double s = 1.0 / (1.0 + exp(-x));
    return s * (1.0 + x * (1.0 - s));
}

ORACLE_EXPORT void kan_oracle_silu_many(const double* x, int64_t n, double* y, double* dy)
{
    for (int64_t e = 0; e < n; ++e) {
        if (y) y[e] = silu(x[e]);
        if (dy) dy[e] = dsilu(x[e]);
    }
}

/* ------------------------------------------------------------------------ */
/* Layer forward / backward                                                  */
/* ------------------------------------------------------------------------ */

typedef struct {
    /* problem */
    int64_t batch, in, out;
    int G, k;
    double lo, hi;
    const double *x, *coef, *w_base, *dY;
    double *y, *dx, *dcoef, *dw_base;
    /* thread slice */
    int64_t b0, b1;
    double* dcoef_part;   /* [out, in, nb] partial of this thread (or NULL) */
    double* dwb_part;     /* [out, in] partial of this thread (or NULL) */
} job_t;

static void* forward_worker(void* arg)
{
    job_t* J = (job_t*)arg;
    const int nb = J->G + J->k;
    double* t = (double*)malloc(sizeof(double) * (size_t)(J->G + 2 * J->k + 1));
    double* work = (double*)malloc(sizeof(double) * (size_t)(2 * (J->G + 2 * J->k)));
    double* Brow = (double*)malloc(sizeof(double) * (size_t)(J->in * nb));
    double* Srow = (double*)malloc(sizeof(double) * (size_t)J->in);
    kan_oracle_knots(J->G, J->k, J->lo, J->hi, t);

    for (int64_t b = J->b0; b < J->b1; ++b) {
        for (int64_t i = 0; i < J->in; ++i) {
            basis_eval(J->x[b * J->in + i], J->G, J->k, t, Brow + i * nb, NULL, work);
            Srow[i] = J->w_base ? silu(J->x[b * J->in + i]) : 0.0;
        }
        for (int64_t j = 0; j < J->out; ++j) {
            double acc = 0.0;
            const double* cj = J->coef + j * J->in * nb;
            for (int64_t i = 0; i < J->in; ++i)
                for (int m = 0; m < nb; ++m) {
                    double bv = Brow[i * nb + m];
                    if (bv != 0.0) acc += cj[i * nb + m] * bv;
                }
            if (J->w_base)
                for (int64_t i = 0; i < J->in; ++i) acc += J->w_base[j * J->in + i] * Srow[i];
            J->y[b * J->out + j] = acc;
        }
    }
    free(t); free(work); free(Brow); free(Srow);
    return NULL;
}

static void* backward_worker(void* arg)
{
    job_t* J = (job_t*)arg;
    const int nb = J->G + J->k;
    double* t = (double*)malloc(sizeof(double) * (size_t)(J->G + 2 * J->k + 1));
    double* work = (double*)malloc(sizeof(double) * (size_t)(2 * (J->G + 2 * J->k)));
    double* Brow = (double*)malloc(sizeof(double) * (size_t)(J->in * nb));
    double* dBrow = (double*)malloc(sizeof(double) * (size_t)(J->in * nb));
    double* Srow = (double*)malloc(sizeof(double) * (size_t)J->in);
    double* dSrow = (double*)malloc(sizeof(double) * (size_t)J->in);
    kan_oracle_knots(J->G, J->k, J->lo, J->hi, t);

    for (int64_t b = J->b0; b < J->b1; ++b) {
        for (int64_t i = 0; i < J->in; ++i) {
            double xv = J->x[b * J->in + i];
            basis_eval(xv, J->G, J->k, t, Brow + i * nb, dBrow + i * nb, work);
            Srow[i] = J->w_base ? silu(xv) : 0.0;
            dSrow[i] = J->w_base ? dsilu(xv) : 0.0;
        }
        const double* dy = J->dY + b * J->out;
        /* dcoef / dw_base partials: this thread's rows, ascending b */
        if (J->dcoef_part)
            for (int64_t j = 0; j < J->out; ++j) {
                double g = dy[j];
                double* pj = J->dcoef_part + j * J->in * nb;
                for (int64_t i = 0; i < J->in; ++i)
                    for (int m = 0; m < nb; ++m) {
                        double bv = Brow[i * nb + m];
                        if (bv != 0.0) pj[i * nb + m] += bv * g;
                    }
            }
        if (J->dwb_part && J->w_base)
            for (int64_t j = 0; j < J->out; ++j)
                for (int64_t i = 0; i < J->in; ++i) J->dwb_part[j * J->in + i] += Srow[i] * dy[j];
        /* dx: sum over j ascending of dY_bj * phi'_ji(x_bi) */
        if (J->dx)
            for (int64_t i = 0; i < J->in; ++i) {
                double acc = 0.0;
                for (int64_t j = 0; j < J->out; ++j) {
                    const double* cji = J->coef + (j * J->in + i) * nb;
                    double d = 0.0;
                    for (int m = 0; m < nb; ++m) {
                        double dbv = dBrow[i * nb + m];
                        if (dbv != 0.0) d += cji[m] * dbv;
                    }
                    if (J->w_base) d += J->w_base[j * J->in + i] * dSrow[i];
                    acc += dy[j] * d;
                }
                J->dx[b * J->in + i] = acc;
            }
    }
    free(t); free(work); free(Brow); free(dBrow); free(Srow); free(dSrow);
    return NULL;
}

static int run_jobs(job_t* proto, int nthreads, void* (*fn)(void*), int with_partials)
{
    if (nthreads < 1) nthreads = 1;
    if ((int64_t)nthreads > proto->batch) nthreads = proto->batch > 0 ? (int)proto->batch : 1;
    const int nb = proto->G + proto->k;
    job_t* jobs = (job_t*)calloc((size_t)nthreads, sizeof(job_t));
    pthread_t* th = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !th) { free(jobs); free(th); return -1; }
    for (int w = 0; w < nthreads; ++w) {
        jobs[w] = *proto;
        jobs[w].b0 = proto->batch * w / nthreads;
        jobs[w].b1 = proto->batch * (w + 1) / nthreads;
        jobs[w].dcoef_part = NULL;
        jobs[w].dwb_part = NULL;
        if (with_partials && proto->dcoef)
            jobs[w].dcoef_part = (double*)calloc((size_t)(proto->out * proto->in * nb), sizeof(double));
        if (with_partials && proto->dw_base && proto->w_base)
            jobs[w].dwb_part = (double*)calloc((size_t)(proto->out * proto->in), sizeof(double));
    }
    for (int w = 1; w < nthreads; ++w) pthread_create(&th[w], NULL, fn, &jobs[w]);
    fn(&jobs[0]);
    for (int w = 1; w < nthreads; ++w) pthread_join(th[w], NULL);

    if (with_partials) {
        /* fixed-order combination: thread 0, 1, 2, ... */
        if (proto->dcoef) {
            int64_t n = proto->out * proto->in * nb;
            for (int64_t e = 0; e < n; ++e) {
                double s = 0.0;
                for (int w = 0; w < nthreads; ++w) s += jobs[w].dcoef_part[e];
                proto->dcoef[e] = s;
            }
        }
        if (proto->dw_base && proto->w_base) {
            int64_t n = proto->out * proto->in;
            for (int64_t e = 0; e < n; ++e) {
                double s = 0.0;
                for (int w = 0; w < nthreads; ++w) s += jobs[w].dwb_part[e];
                proto->dw_base[e] = s;
            }
        }
        for (int w = 0; w < nthreads; ++w) { free(jobs[w].dcoef_part); free(jobs[w].dwb_part); }
    }
    free(jobs);
    free(th);
    return 0;
}

/* y[batch,out] = sum_i sum_m coef[j,i,m] B_m(x[b,i]) (+ sum_i w_base[j,i] silu(x[b,i])).
 * w_base may be NULL (no base branch).  Returns 0 on success. */
ORACLE_EXPORT int kan_oracle_forward(int64_t batch, int64_t in, int64_t out, int G, int k, double lo, double hi,
                                     const double* x, const double* coef, const double* w_base, double* y,
                                     int nthreads)
{
    if (batch < 0 || in < 1 || out < 1 || G < 1 || k < 0 || !(hi > lo)) return -1;
    if (batch == 0) return 0;
    job_t J;
    memset(&J, 0, sizeof(J));
    J.batch = batch; J.in = in; J.out = out; J.G = G; J.k = k; J.lo = lo; J.hi = hi;
    J.x = x; J.coef = coef; J.w_base = w_base; J.y = y;
    return run_jobs(&J, nthreads, forward_worker, 0);
}

/* Gradients of the layer for upstream gradient dY[batch,out].  Any of dx,
 * dcoef, dw_base may be NULL to skip it; dw_base is skipped when w_base is
 * NULL.  Outputs are overwritten.  Returns 0 on success. */
ORACLE_EXPORT int kan_oracle_backward(int64_t batch, int64_t in, int64_t out, int G, int k, double lo, double hi,
                                      const double* x, const double* coef, const double* w_base, const double* dY,
                                      double* dx, double* dcoef, double* dw_base, int nthreads)
{
    if (batch < 0 || in < 1 || out < 1 || G < 1 || k < 0 || !(hi > lo)) return -1;
    const int nb = G + k;
    if (batch == 0) {
        if (dcoef) memset(dcoef, 0, sizeof(double) * (size_t)(out * in * nb));
        if (dw_base && w_base) memset(dw_base, 0, sizeof(double) * (size_t)(out * in));
        return 0;
    }
    job_t J;
    memset(&J, 0, sizeof(J));
    J.batch = batch; J.in = in; J.out = out; J.G = G; J.k = k; J.lo = lo; J.hi = hi;
    J.x = x; J.coef = coef; J.w_base = w_base; J.dY = dY;
    J.dx = dx; J.dcoef = dcoef; J.dw_base = dw_base;
    return run_jobs(&J, nthreads, backward_worker, 1);
}

/* Dense basis matrix A[batch, in*(G+k)] with A[b, i*(G+k)+m] = B_m(x[b,i]):
 * the "dense K-basis" expansion, used by the tests to check the contraction
 * against a library matmul. */
ORACLE_EXPORT void kan_oracle_dense_basis(int64_t batch, int64_t in, int G, int k, double lo, double hi,
                                          const double* x, double* A)
{
    kan_oracle_basis_many(x, batch * in, G, k, lo, hi, A, NULL);
}
