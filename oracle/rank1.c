/*
 * O3: marginal coding rate by a rank-1 Cholesky recursion, plain C, float64.
 *
 * Method (ByteFlow, arXiv 2603.03583; paper.rainbus.top summary,
 * "Prerequisites: lossy coding rate" and "Method steps", stage 2):
 *   R_eps(H) = 1/2 logdet(I + c H H^T), c = d / eps^2,
 *   dR_t = R_eps(h_{1:t}) - R_eps(h_{1:t-1}).
 * With M_t = I_d + c sum_{i<=t} h_i h_i^T, Sylvester's identity gives
 * R_eps(h_{1:t}) = 1/2 logdet M_t, and the matrix determinant lemma gives
 * det M_t = det M_{t-1} (1 + c h_t^T M_{t-1}^{-1} h_t), hence
 *   dR_t = 1/2 log(1 + c q_t),  q_t = |L_{t-1}^{-1} h_t|^2,  M_{t-1} = L L^T.
 * The incremental update of the factor is the one the summary's
 * "independent weaknesses" paragraph suggests (Sherman-Morrison-Woodbury
 * style), done on the Cholesky factor: the textbook rank-1 Cholesky update
 * (Golub & Van Loan, Matrix Computations, "updating a Cholesky
 * factorization"): for k = 0..d-1 with v = sqrt(c) h,
 *   r = hypot(L_kk, v_k), cs = r / L_kk, sn = v_k / L_kk, L_kk = r,
 *   L_ik = (L_ik + sn v_i) / cs,  v_i = cs v_i - sn L_ik   (i > k).
 *
 * Positions are 0-based; position 0 sees M_{-1} = I.  One row (sequence) is
 * processed by one thread; rows are handed out through an atomic counter.
 *
 * Test infrastructure only: used by the test-suite, the smoke check and the
 * benchmark's CPU-baseline leg; never by the product path.
 */
#include <math.h>
#include <pthread.h>
#include <stdatomic.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    const float *H;           /* [N, d] values (fp32 or widened bf16) */
    const int64_t *offsets;   /* [rows + 1] */
    int64_t rows, d;
    double c;
    double *dR;               /* [N] */
    atomic_long next;
    int status;
} job_t;

/* U holds L^T row-major: U[k*d + i] = L[i][k] for i >= k, so column k of L
 * is contiguous. */
static void row_dR(const float *H, int64_t T, int64_t d, double c, double *dR,
                   double *U, double *w, double *v)
{
    memset(U, 0, sizeof(double) * (size_t)(d * d));
    for (int64_t k = 0; k < d; ++k) U[k * d + k] = 1.0;
    const double sc = sqrt(c);
    for (int64_t t = 0; t < T; ++t) {
        const float *h = H + t * d;
        /* forward substitution L y = h, column oriented; y overwrites w */
        for (int64_t i = 0; i < d; ++i) w[i] = (double)h[i];
        double q = 0.0;
        for (int64_t k = 0; k < d; ++k) {
            const double *Lk = U + k * d;
            double yk = w[k] / Lk[k];
            w[k] = yk;
            q += yk * yk;
            for (int64_t i = k + 1; i < d; ++i) w[i] -= Lk[i] * yk;
        }
        dR[t] = 0.5 * log1p(c * q);
        /* rank-1 update L L^T + v v^T, v = sqrt(c) h */
        for (int64_t i = 0; i < d; ++i) v[i] = sc * (double)h[i];
        for (int64_t k = 0; k < d; ++k) {
            double *Lk = U + k * d;
            double r = hypot(Lk[k], v[k]);
            double cs = r / Lk[k];
            double sn = v[k] / Lk[k];
            Lk[k] = r;
            for (int64_t i = k + 1; i < d; ++i) {
                double l = (Lk[i] + sn * v[i]) / cs;
                v[i] = cs * v[i] - sn * l;
                Lk[i] = l;
            }
        }
    }
}

static void *worker(void *arg)
{
    job_t *J = (job_t *)arg;
    int64_t d = J->d;
    double *U = (double *)malloc(sizeof(double) * (size_t)(d * d));
    double *w = (double *)malloc(sizeof(double) * (size_t)d);
    double *v = (double *)malloc(sizeof(double) * (size_t)d);
    if (!U || !w || !v) { J->status = -1; free(U); free(w); free(v); return NULL; }
    for (;;) {
        long r = atomic_fetch_add(&J->next, 1);
        if (r >= J->rows) break;
        int64_t a = J->offsets[r], b = J->offsets[r + 1];
        row_dR(J->H + a * d, b - a, d, J->c, J->dR + a, U, w, v);
    }
    free(U); free(w); free(v);
    return NULL;
}

/* dR for every position of every row.  Returns 0 on success. */
int oracle_dR_rank1(const float *H, const int64_t *offsets, int64_t rows,
                    int64_t d, double c, double *dR, int nthreads)
{
    if (!H || !offsets || !dR || rows < 0 || d < 1 || !(c > 0.0)) return -2;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > rows) nthreads = rows > 0 ? (int)rows : 1;
    job_t J;
    J.H = H; J.offsets = offsets; J.rows = rows; J.d = d; J.c = c; J.dR = dR;
    atomic_init(&J.next, 0);
    J.status = 0;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!th) return -1;
    int started = 0;
    for (int i = 0; i < nthreads; ++i)
        if (pthread_create(&th[i], NULL, worker, &J) == 0) ++started;
    if (started == 0) worker(&J);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    free(th);
    return J.status;
}
