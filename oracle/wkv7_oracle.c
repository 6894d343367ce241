/*
 * Plain fp64 C statement of the WKV-7 recurrence (RWKV-7 "Goose") and its
 * group_norm + bonus epilogue.
 *
 * TEST INFRASTRUCTURE ONLY: loaded by the tests, the graft smoke check and the
 * benchmark's CPU-baseline leg. It shares no code, header or constant with the
 * CUDA library and is never linked into it.
 *
 * Definition followed (rebuttal page, numpy time_mixing listing; ARWKV verdict
 * page, key_machinery): per batch element b and head h, with S an N x N matrix
 * whose row i is a value channel and column j a key channel,
 *     removed[i] = sum_j S[i][j] * kk[j]                     (state before update)
 *     S[i][j]    = S[i][j]*w[j] - removed[i]*kk[j]*a[j] + v[i]*k[j]
 *     y[i]       = sum_j S[i][j] * r[j]                      (state after update)
 * Epilogue (same listing): population-variance group_norm over the N channels of
 * a head with eps inside the square root, per-channel affine, then
 * + (sum_j r[j]*k[j]*r_k[h][j]) * v[i].
 *
 * Layouts: token tensors [B][T][H][N]; S0 / S_T [B][H][N][N]; snapshots
 * [B][T/snap_every][H][N][N]; epilogue parameters [H][N]. All fp64.
 * Units (b, h) are independent and are spread over POSIX threads; within a unit
 * the token loop runs in order, so the result does not depend on the thread count.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

typedef struct {
    int B, T, H, N;
    const double *r, *w, *k, *v, *kk, *a, *S0;
    double *y, *S_T, *snaps;
    int snap_every;
    int next_unit;
    pthread_mutex_t lock;
    int failed;
} job_t;

static int take_unit(job_t *j) {
    pthread_mutex_lock(&j->lock);
    int u = j->next_unit < j->B * j->H ? j->next_unit++ : -1;
    pthread_mutex_unlock(&j->lock);
    return u;
}

static void run_unit(job_t *j, int u, double *S, double *removed) {
    const int T = j->T, H = j->H, N = j->N;
    const int b = u / H, h = u % H;
    const int n_snap = j->snap_every > 0 ? T / j->snap_every : 0;
    if (j->S0)
        memcpy(S, j->S0 + (size_t)u * N * N, sizeof(double) * N * N);
    else
        memset(S, 0, sizeof(double) * N * N);
    for (int t = 0; t < T; ++t) {
        const size_t base = (((size_t)b * T + t) * H + h) * N;
        const double *w = j->w + base, *k = j->k + base, *v = j->v + base;
        const double *kk = j->kk + base, *a = j->a + base, *r = j->r + base;
        for (int i = 0; i < N; ++i) {
            double acc = 0.0;
            for (int jj = 0; jj < N; ++jj) acc += S[i * N + jj] * kk[jj];
            removed[i] = acc;
        }
        for (int i = 0; i < N; ++i)
            for (int jj = 0; jj < N; ++jj)
                S[i * N + jj] = S[i * N + jj] * w[jj] - removed[i] * (kk[jj] * a[jj]) + v[i] * k[jj];
        for (int i = 0; i < N; ++i) {
            double acc = 0.0;
            for (int jj = 0; jj < N; ++jj) acc += S[i * N + jj] * r[jj];
            j->y[base + i] = acc;
        }
        if (n_snap && (t + 1) % j->snap_every == 0) {
            const int m = (t + 1) / j->snap_every - 1;
            double *dst = j->snaps + ((((size_t)b * n_snap + m) * H + h) * N) * N;
            memcpy(dst, S, sizeof(double) * N * N);
        }
    }
    if (j->S_T) memcpy(j->S_T + (size_t)u * N * N, S, sizeof(double) * N * N);
}

static void *worker(void *arg) {
    job_t *j = (job_t *)arg;
    double *S = (double *)malloc(sizeof(double) * j->N * j->N);
    double *removed = (double *)malloc(sizeof(double) * j->N);
    if (!S || !removed) {
        pthread_mutex_lock(&j->lock);
        j->failed = 1;
        pthread_mutex_unlock(&j->lock);
    } else {
        for (int u; (u = take_unit(j)) >= 0;) run_unit(j, u, S, removed);
    }
    free(S);
    free(removed);
    return NULL;
}

/* Returns 0 on success, -1 on bad arguments, -2 on allocation failure. */
int wkv7_oracle_forward(int B, int T, int H, int N,
                        const double *r, const double *w, const double *k,
                        const double *v, const double *kk, const double *a,
                        const double *S0, double *y, double *S_T,
                        int snap_every, double *snaps, int nthreads) {
    if (B < 0 || T < 0 || H < 0 || N <= 0 || !r || !w || !k || !v || !kk || !a || !y) return -1;
    if (snap_every < 0 || (snap_every > 0 && !snaps)) return -1;
    job_t j = {B, T, H, N, r, w, k, v, kk, a, S0, y, S_T, snaps, snap_every, 0,
               PTHREAD_MUTEX_INITIALIZER, 0};
    const int units = B * H;
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads > units) nthreads = units;
    if (nthreads <= 1) {
        worker(&j);
        return j.failed ? -2 : 0;
    }
    pthread_t *tid = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
    if (!tid) return -2;
    int started = 0;
    for (int i = 0; i < nthreads; ++i)
        if (pthread_create(&tid[i], NULL, worker, &j) == 0) ++started;
    if (started == 0) worker(&j);
    for (int i = 0; i < started; ++i) pthread_join(tid[i], NULL);
    free(tid);
    return j.failed ? -2 : 0;
}

/* out may alias y. Returns 0, or -1 on bad arguments. */
int wkv7_oracle_epilogue(int B, int T, int H, int N, const double *y,
                         const double *r, const double *k, const double *v,
                         const double *ln_w, const double *ln_b, const double *r_k,
                         double eps, double *out) {
    if (B < 0 || T < 0 || H < 0 || N <= 0 || !y || !r || !k || !v || !ln_w || !ln_b || !r_k || !out)
        return -1;
    for (size_t row = 0; row < (size_t)B * T * H; ++row) {
        const int h = (int)(row % H);
        const size_t base = row * N;
        double mean = 0.0;
        for (int i = 0; i < N; ++i) mean += y[base + i];
        mean /= N;
        double var = 0.0;
        for (int i = 0; i < N; ++i) var += (y[base + i] - mean) * (y[base + i] - mean);
        var /= N;
        const double inv = 1.0 / sqrt(var + eps);
        double bonus = 0.0;
        for (int jj = 0; jj < N; ++jj) bonus += r[base + jj] * k[base + jj] * r_k[h * N + jj];
        for (int i = 0; i < N; ++i)
            out[base + i] = (y[base + i] - mean) * inv * ln_w[h * N + i] + ln_b[h * N + i] +
                            bonus * v[base + i];
    }
    return 0;
}
