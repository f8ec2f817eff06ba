/*
 * KDA oracle: the token-by-token recurrence in FP64.
 *
 * TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline / reference leg may load this library. The product path never does.
 * It shares no code, header or constant with the CUDA library.
 *
 * What it computes (one sequence b, one head h, tokens t = 0..T-1), with the state
 * S laid out [key channel i][value channel j] (Glm5NextKdaWorkspace page: the
 * recurrent state is carried per head as head_dim x head_dim FP32):
 *
 *   S'  = diag(exp(g_t)) S            per-channel log-decay gate g_t <= 0 (field `gate`)
 *   u   = beta_t (v_t - S'^T k_t)     delta rule with the sigmoid beta (field `beta`)
 *   S   = S' + k_t u^T
 *   o_t = scale * S^T q_t             read-out after the update (field `core`)
 *
 * q and k arrive already L2-normalised; they are used as given (Glm5NextKdaLayer
 * page, `decode`: kda_recurrent takes pre-normalised q/k). Only the T valid rows are
 * passed in: the oracle never sees padding.
 *
 * Layouts (row-major, doubles): q,k,v,g [B,T,H,D]; beta [B,T,H]; S [B,H,D,D]
 * (updated in place); o [B,T,H,D].
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>

typedef struct {
    int B, T, H, D;
    double scale;
    const double *q, *k, *v, *g, *beta;
    double *S, *o;
    int next_unit;
    pthread_mutex_t lock;
} job_t;

static void one_head(const job_t *J, int b, int h, double *y, double *u)
{
    const int T = J->T, H = J->H, D = J->D;
    double *S = J->S + ((size_t)b * H + h) * D * D;
    for (int t = 0; t < T; ++t) {
        const size_t row = ((size_t)b * T + t) * H + h;
        const double *q = J->q + row * D, *k = J->k + row * D;
        const double *v = J->v + row * D, *g = J->g + row * D;
        const double beta = J->beta[row];
        /* S' = diag(exp(g)) S : row i (key channel i) decays by exp(g_i) */
        for (int i = 0; i < D; ++i) {
            const double a = exp(g[i]);
            for (int j = 0; j < D; ++j) S[i * D + j] *= a;
        }
        /* y = S'^T k */
        for (int j = 0; j < D; ++j) y[j] = 0.0;
        for (int i = 0; i < D; ++i)
            for (int j = 0; j < D; ++j) y[j] += S[i * D + j] * k[i];
        /* u = beta (v - y) ; S = S' + k u^T */
        for (int j = 0; j < D; ++j) u[j] = beta * (v[j] - y[j]);
        for (int i = 0; i < D; ++i)
            for (int j = 0; j < D; ++j) S[i * D + j] += k[i] * u[j];
        /* o = scale S^T q */
        double *o = J->o + row * D;
        for (int j = 0; j < D; ++j) y[j] = 0.0;
        for (int i = 0; i < D; ++i)
            for (int j = 0; j < D; ++j) y[j] += S[i * D + j] * q[i];
        for (int j = 0; j < D; ++j) o[j] = J->scale * y[j];
    }
}

static void *worker(void *arg)
{
    job_t *J = (job_t *)arg;
    double *y = (double *)malloc(sizeof(double) * J->D);
    double *u = (double *)malloc(sizeof(double) * J->D);
    for (;;) {
        pthread_mutex_lock(&J->lock);
        const int unit = J->next_unit++;
        pthread_mutex_unlock(&J->lock);
        if (unit >= J->B * J->H) break;
        one_head(J, unit / J->H, unit % J->H, y, u);
    }
    free(y);
    free(u);
    return NULL;
}

/* Returns 0 on success, -1 on bad arguments. nthreads <= 0 means 1. */
int oracle_recurrence(int B, int T, int H, int D, double scale,
                      const double *q, const double *k, const double *v,
                      const double *g, const double *beta, double *S, double *o,
                      int nthreads)
{
    if (B < 0 || T < 0 || H <= 0 || D <= 0) return -1;
    if (B == 0 || T == 0) return 0;
    job_t J = {B, T, H, D, scale, q, k, v, g, beta, S, o, 0};
    pthread_mutex_init(&J.lock, NULL);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > B * H) nthreads = B * H;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
    for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, worker, &J);
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J.lock);
    return 0;
}
