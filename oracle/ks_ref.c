/*
 * Plain CPU oracle for multiplication by a Kronecker-sparse (KS) matrix.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call this file:
 * only the tests, the smoke check and the benchmark's CPU-baseline leg do.  It
 * shares no code, header, table or helper with the CUDA library.
 *
 * What it follows
 *   The taxoreview.com page on Kronecker-sparse matrix multiplication (its
 *   first abstract): a KS matrix is one whose support is a Kronecker product of
 *   identity and all-ones blocks, and butterfly / Monarch matrices are products
 *   of such factors.  The pages print no index formula; the reading used here
 *   is the textbook Kronecker product (A (x) B)[(p,q),(r,s)] = A[p,r] B[q,s]
 *   with row index p*rows(B)+q, applied to I_a (x) 1_{b x c} (x) I_d:
 *
 *     K is (a*b*d) x (a*c*d),
 *     K[i*b*d + k*d + l][i*c*d + j*d + l] = values[i][l][k][j]
 *     (i<a, k<b, j<c, l<d), every other entry zero,
 *
 *   and the product computed is Y = X * K^T over a batch of N rows:
 *
 *     Y[n][i*b*d + k*d + l] = sum_{j<c} values[i][l][k][j] * X[n][i*c*d + j*d + l].
 *
 * Everything is double precision; inputs are converted exactly by the caller
 * (fp32 and bf16 values are exactly representable in double).  The loops are
 * the definition written out: no blocking, no reordering, no fusion.  Rows of
 * the batch are independent, so the outer loop over n may run on OpenMP
 * threads; that changes nothing in the arithmetic of any one output.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Number of OpenMP threads the next call may use (<= 0: the runtime's default). */
static int g_threads = 0;

void ks_ref_set_threads(int n) { g_threads = n; }

int ks_ref_get_threads(void)
{
#ifdef _OPENMP
    return g_threads > 0 ? g_threads : omp_get_max_threads();
#else
    return 1;
#endif
}

/* Y = X * K^T for one KS factor, K given by its pattern (a,b,c,d) and
 * values[a][d][b][c].  X is N x (a*c*d), Y is N x (a*b*d), both row-major. */
void ks_ref_matmul(const double *X, const double *values,
                   int64_t a, int64_t b, int64_t c, int64_t d,
                   int64_t N, double *Y)
{
    const int64_t in_f = a * c * d;
    const int64_t out_f = a * b * d;
    int nt = ks_ref_get_threads();
    (void)nt;
#pragma omp parallel for schedule(static) num_threads(nt)
    for (int64_t n = 0; n < N; ++n) {
        const double *x = X + n * in_f;
        double *y = Y + n * out_f;
        for (int64_t i = 0; i < a; ++i)
            for (int64_t k = 0; k < b; ++k)
                for (int64_t l = 0; l < d; ++l) {
                    double acc = 0.0;
                    for (int64_t j = 0; j < c; ++j)
                        acc += values[((i * d + l) * b + k) * c + j] *
                               x[i * c * d + j * d + l];
                    y[i * b * d + k * d + l] = acc;
                }
    }
}

/* The dense (a*b*d) x (a*c*d) matrix K of one factor (row-major, zero off the
 * support). */
void ks_ref_densify(const double *values, int64_t a, int64_t b, int64_t c,
                    int64_t d, double *K)
{
    const int64_t rows = a * b * d, cols = a * c * d;
    memset(K, 0, (size_t)(rows * cols) * sizeof(double));
    for (int64_t i = 0; i < a; ++i)
        for (int64_t l = 0; l < d; ++l)
            for (int64_t k = 0; k < b; ++k)
                for (int64_t j = 0; j < c; ++j)
                    K[(i * b * d + k * d + l) * cols + (i * c * d + j * d + l)] =
                        values[((i * d + l) * b + k) * c + j];
}

/* Y = X * K^T for a dense K (rows x cols), by the naive triple loop. */
void ks_ref_dense_matmul(const double *X, const double *K, int64_t N,
                         int64_t rows, int64_t cols, double *Y)
{
    int nt = ks_ref_get_threads();
    (void)nt;
#pragma omp parallel for schedule(static) num_threads(nt)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t r = 0; r < rows; ++r) {
            double acc = 0.0;
            for (int64_t q = 0; q < cols; ++q)
                acc += K[r * cols + q] * X[n * cols + q];
            Y[n * rows + r] = acc;
        }
}

/* A chain of KS factors applied in order: factor 0 first, so
 * Y = X * (K_{n-1} ... K_1 K_0)^T.  patterns holds 4 int64 per factor
 * (a,b,c,d); factor t's output width a*b*d must equal factor t+1's input width
 * a*c*d.  Intermediates stay in double.  Returns 0, or -1 on a width mismatch
 * or an allocation failure (Y untouched). */
int ks_ref_chain(const double *X, const double *const *factors,
                 const int64_t *patterns, int n_factors, int64_t N, double *Y)
{
    if (n_factors <= 0) return -1;
    int64_t widest = 0;
    for (int t = 0; t < n_factors; ++t) {
        const int64_t *p = patterns + 4 * t;
        int64_t in_f = p[0] * p[2] * p[3], out_f = p[0] * p[1] * p[3];
        if (t > 0) {
            const int64_t *q = patterns + 4 * (t - 1);
            if (q[0] * q[1] * q[3] != in_f) return -1;
        }
        if (in_f > widest) widest = in_f;
        if (out_f > widest) widest = out_f;
    }
    double *buf[2];
    buf[0] = (double *)malloc((size_t)(N * widest) * sizeof(double));
    buf[1] = (double *)malloc((size_t)(N * widest) * sizeof(double));
    if (!buf[0] || !buf[1]) {
        free(buf[0]);
        free(buf[1]);
        return -1;
    }
    const double *src = X;
    for (int t = 0; t < n_factors; ++t) {
        const int64_t *p = patterns + 4 * t;
        double *dst = (t == n_factors - 1) ? Y : buf[t & 1];
        ks_ref_matmul(src, factors[t], p[0], p[1], p[2], p[3], N, dst);
        src = dst;
    }
    free(buf[0]);
    free(buf[1]);
    return 0;
}

/* Backward of Y = X * K^T (the page's KSLinear layer is trained by gradient
 * descent; these are the two gradients of that product, written from the
 * definition of K above).
 *
 * Input gradient: dX = dY * K, i.e. for every n, i, j, l
 *     dX[n][i*c*d + j*d + l] = sum_{k<b} values[i][l][k][j] * dY[n][i*b*d + k*d + l].
 * dY is N x (a*b*d), dX is N x (a*c*d). */
void ks_ref_dx(const double *dY, const double *values,
               int64_t a, int64_t b, int64_t c, int64_t d,
               int64_t N, double *dX)
{
    const int64_t in_f = a * c * d;
    const int64_t out_f = a * b * d;
    int nt = ks_ref_get_threads();
    (void)nt;
#pragma omp parallel for schedule(static) num_threads(nt)
    for (int64_t n = 0; n < N; ++n) {
        const double *g = dY + n * out_f;
        double *h = dX + n * in_f;
        for (int64_t i = 0; i < a; ++i)
            for (int64_t j = 0; j < c; ++j)
                for (int64_t l = 0; l < d; ++l) {
                    double acc = 0.0;
                    for (int64_t k = 0; k < b; ++k)
                        acc += g[i * b * d + k * d + l] *
                               values[(i * d + l) * b * c + k * c + j];
                    h[i * c * d + j * d + l] = acc;
                }
    }
}

/* Gradient of the values: for every i, l, k, j
 *     dV[i][l][k][j] = sum_{n<N} dY[n][i*b*d + k*d + l] * X[n][i*c*d + j*d + l],
 * the entries of dY^T * X at K's support, in the values layout [a][d][b][c].
 * The sum over n runs in order n = 0..N-1. */
void ks_ref_dv(const double *dY, const double *X,
               int64_t a, int64_t b, int64_t c, int64_t d,
               int64_t N, double *dV)
{
    const int64_t in_f = a * c * d;
    const int64_t out_f = a * b * d;
    int nt = ks_ref_get_threads();
    (void)nt;
#pragma omp parallel for schedule(static) num_threads(nt)
    for (int64_t il = 0; il < a * d; ++il) {
        const int64_t i = il / d, l = il % d;
        for (int64_t k = 0; k < b; ++k)
            for (int64_t j = 0; j < c; ++j) {
                double acc = 0.0;
                for (int64_t n = 0; n < N; ++n)
                    acc += dY[n * out_f + i * b * d + k * d + l] *
                           X[n * in_f + i * c * d + j * d + l];
                dV[((i * d + l) * b + k) * c + j] = acc;
            }
    }
}
