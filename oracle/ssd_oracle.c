/*
 * ssd_oracle.c -- plain fp64 CPU oracle of the SSD layer forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  It shares
 * no code, header, table or helper with the CUDA path and includes nothing from
 * it.
 *
 * What it computes (the plain definition, no blocking or reordering):
 *
 *   "Transformers are SSMs" analysis page, section "The SSM as a Matrix
 *   Transformation", equation (2): h_t = A_t h_{t-1} + B_t x_t,
 *   y_t = C_t^T h_t, restricted (section "The Scalar-Identity SSM") to
 *   A_t = a_t I.  With a head dimension P, the state of one head is an
 *   (N x P) matrix (stored here as [P][N]) and every one of the P input
 *   channels runs the same scalar recurrence ("SSD Layer: Formal
 *   Definition": Y = M X broadcast over the P dimension of X).
 *
 *   The pages never write the discretisation.  This oracle takes the reading
 *   used throughout the build: a_t = exp(dt_t * A_h), the input term is
 *   B_t x_t^T with no dt factor, a skip term D_h * x_t is added to y_t, the
 *   initial state h_{-1} is init_state (zero when absent) so that a_0 does
 *   multiply the initial state, and heads map to B/C groups contiguously,
 *   g = h / (H / G).
 *
 * Layouts (row-major, all fp64):
 *   x [b][T][H][P], dt [b][T][H], A [H], B, C [b][T][G][N], D [H],
 *   init_state [b][H][P][N] (may be NULL), y [b][T][H][P],
 *   final_state [b][H][P][N] (may be NULL).
 *
 * Heads are independent, so the (batch, head) pairs are spread over POSIX
 * threads; each pair is still a plain token-by-token loop.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

typedef struct {
    const double *x, *dt, *A, *B, *C, *D, *init;
    double *y, *fin;
    long batch, T, H, P, G, N;
    const long *pairs; /* optional list of (b, h) pairs, 2 entries each */
    long npairs;
    long next; /* work counter, guarded by mu */
    pthread_mutex_t mu;
} job_t;

/* One (batch, head) sequence: the recurrence, token by token. */
static void run_pair(const job_t *j, long b, long h) {
    const long T = j->T, H = j->H, P = j->P, G = j->G, N = j->N;
    const long g = h / (H / G);
    double *S = (double *)calloc((size_t)(P * N), sizeof(double));
    if (!S) return;
    if (j->init) memcpy(S, j->init + (b * H + h) * P * N, sizeof(double) * (size_t)(P * N));
    for (long t = 0; t < T; ++t) {
        const double a = exp(j->dt[(b * T + t) * H + h] * j->A[h]);
        const double *xt = j->x + ((b * T + t) * H + h) * P;
        const double *Bt = j->B + ((b * T + t) * G + g) * N;
        const double *Ct = j->C + ((b * T + t) * G + g) * N;
        double *yt = j->y + ((b * T + t) * H + h) * P;
        for (long p = 0; p < P; ++p) {
            double *Sp = S + p * N;
            const double xv = xt[p];
            double acc = 0.0;
            for (long n = 0; n < N; ++n) {
                Sp[n] = a * Sp[n] + xv * Bt[n];
                acc += Sp[n] * Ct[n];
            }
            yt[p] = acc + j->D[h] * xv;
        }
    }
    if (j->fin) memcpy(j->fin + (b * H + h) * P * N, S, sizeof(double) * (size_t)(P * N));
    free(S);
}

static void *worker(void *arg) {
    job_t *j = (job_t *)arg;
    const long total = j->pairs ? j->npairs : j->batch * j->H;
    for (;;) {
        pthread_mutex_lock(&j->mu);
        const long k = j->next++;
        pthread_mutex_unlock(&j->mu);
        if (k >= total) break;
        const long b = j->pairs ? j->pairs[2 * k] : k / j->H;
        const long h = j->pairs ? j->pairs[2 * k + 1] : k % j->H;
        run_pair(j, b, h);
    }
    return NULL;
}

/*
 * Returns 0 on success, 1 on invalid arguments.  nthreads <= 0 means one
 * thread per online core.  When pairs != NULL only the listed (b, h) pairs are
 * computed and only their slices of y / final_state are written.
 */
int ssd_ref_fwd_f64(const double *x, const double *dt, const double *A, const double *B,
                    const double *C, const double *D, const double *init_state, double *y,
                    double *final_state, long batch, long T, long H, long P, long G, long N,
                    const long *pairs, long npairs, int nthreads) {
    if (!x || !dt || !A || !B || !C || !D || !y) return 1;
    if (batch <= 0 || T < 0 || H <= 0 || P <= 0 || G <= 0 || N <= 0 || H % G != 0) return 1;
    if (pairs && npairs < 0) return 1;
    job_t j;
    memset(&j, 0, sizeof j);
    j.x = x; j.dt = dt; j.A = A; j.B = B; j.C = C; j.D = D; j.init = init_state;
    j.y = y; j.fin = final_state;
    j.batch = batch; j.T = T; j.H = H; j.P = P; j.G = G; j.N = N;
    j.pairs = pairs; j.npairs = npairs;
    pthread_mutex_init(&j.mu, NULL);
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    pthread_t th[256];
    int started = 0;
    for (int i = 1; i < nthreads; ++i)
        if (pthread_create(&th[started], NULL, worker, &j) == 0) ++started;
    worker(&j);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    pthread_mutex_destroy(&j.mu);
    return 0;
}

/* Number of threads ssd_ref_fwd_f64 uses when nthreads <= 0. */
int ssd_ref_default_threads(void) {
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    if (n < 1) n = 1;
    if (n > 256) n = 256;
    return (int)n;
}
