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
 * wkv7_oracle_layer (at the end) is a second, independent transcription of the whole
 * time-mixing layer, against which the numpy layer is checked.
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

/*
 * One RWKV-7 time-mixing layer, a second transcription independent of the numpy oracle:
 * the rebuttal page's numpy time_mixing listing taken one token at a time with plain loops,
 * every vector 1-D of length C = H * N and every step in the listing's order:
 *   token-shift mixes x_m = x + m (x_prev - x);
 *   r = Wr x_r (W stored [out][in]);
 *   w = exp(-sigmoid(tanh(x_w Ww1) Ww2 + w_bias) / sqrt(e)) (low-rank factors [in][out]);
 *   k = Wk x_k, v = Wv x_v;
 *   first layer: v0 = v; later layers: v += (v0 - v) sigmoid(x_v Wv1 Wv2 + v_bias);
 *   a = sigmoid(x_a Wa1 Wa2 + a_bias); g = sigmoid(x_g Wg1) Wg2;
 *   kk = k * k_k; k += k (a - 1) k_a; kk normalised per head (floor 1e-12 on the norm);
 *   S = S diag(w) - (S kk)(kk a)^T + v k^T per head; y = S r;
 *   group_norm per head (population variance, eps inside the root), * ln_w + ln_b;
 *   y += (sum_j r_j k_j r_k_j) v per head; out = Wo (y * g).
 * Layouts: x, v0, out, v0_out [B][T][C]; last_x, last_out [B][C]; S0, S_T [B][H][N][N];
 * square projections [C][C]; Ww1 [C][dw], Ww2 [dw][C] and likewise for a, v, g;
 * mixes and biases [C]; r_k, k_k, k_a, ln_w, ln_b [H][N] (= [C]). last_x, v0, S0 may be NULL
 * (zeros / first layer / zero state; Wv1, Wv2, v_bias are then unused). Single-threaded.
 * Returns 0, -1 on bad arguments, -2 on allocation failure.
 */
static double sigm(double z) { return 1.0 / (1.0 + exp(-z)); }

int wkv7_oracle_layer(int B, int T, int H, int N, int dw, int da, int dv, int dg,
                      const double *x, const double *last_x, const double *v0, const double *S0,
                      const double *mr, const double *mw, const double *mk, const double *mv,
                      const double *ma, const double *mg, const double *w_bias, const double *a_bias,
                      const double *v_bias, const double *r_k, const double *k_k, const double *k_a,
                      const double *ln_w, const double *ln_b, const double *Wr, const double *Wk,
                      const double *Wv, const double *Wo, const double *Ww1, const double *Ww2,
                      const double *Wa1, const double *Wa2, const double *Wv1, const double *Wv2,
                      const double *Wg1, const double *Wg2, double eps,
                      double *out, double *v0_out, double *last_out, double *S_T) {
    if (B < 0 || T < 0 || H <= 0 || N <= 0 || dw <= 0 || da <= 0 || dv <= 0 || dg <= 0 || !x || !out ||
        !v0_out || !last_out || !S_T)
        return -1;
    const int C = H * N;
    const int dmax = dw > da ? (dw > dv ? (dw > dg ? dw : dg) : (dv > dg ? dv : dg))
                             : (da > dv ? (da > dg ? da : dg) : (dv > dg ? dv : dg));
    double *buf = (double *)malloc(sizeof(double) * ((size_t)C * 17 + dmax));
    if (!buf) return -2;
    double *xp = buf, *xr = xp + C, *xw = xr + C, *xk = xw + C, *xv = xk + C, *xa = xv + C, *xg = xa + C;
    double *r = xg + C, *w = r + C, *k = w + C, *v = k + C, *a = v + C, *g = a + C, *kk = g + C;
    double *y = kk + C, *tmp = y + C, *sk = tmp + C, *hid = sk + C;
    const double *mixes[6] = {mr, mw, mk, mv, ma, mg};
    double *xs[6] = {xr, xw, xk, xv, xa, xg};
    for (int b = 0; b < B; ++b) {
        double *Sb = S_T + (size_t)b * H * N * N;
        for (size_t e = 0; e < (size_t)H * N * N; ++e) Sb[e] = S0 ? S0[(size_t)b * H * N * N + e] : 0.0;
        for (int c = 0; c < C; ++c) xp[c] = last_x ? last_x[(size_t)b * C + c] : 0.0;
        for (int t = 0; t < T; ++t) {
            const double *xt = x + ((size_t)b * T + t) * C;
            for (int m = 0; m < 6; ++m)
                for (int c = 0; c < C; ++c) xs[m][c] = xt[c] + mixes[m][c] * (xp[c] - xt[c]);
            for (int o = 0; o < C; ++o) {   /* square projections: W @ x */
                double sr = 0.0, sk2 = 0.0, sv = 0.0;
                for (int i = 0; i < C; ++i) {
                    sr += Wr[(size_t)o * C + i] * xr[i];
                    sk2 += Wk[(size_t)o * C + i] * xk[i];
                    sv += Wv[(size_t)o * C + i] * xv[i];
                }
                r[o] = sr;
                k[o] = sk2;
                v[o] = sv;
            }
            /* decay: hidden = tanh(x_w @ Ww1), logit = hidden @ Ww2 + w_bias */
            for (int d = 0; d < dw; ++d) {
                double s = 0.0;
                for (int c = 0; c < C; ++c) s += xw[c] * Ww1[(size_t)c * dw + d];
                hid[d] = tanh(s);
            }
            for (int c = 0; c < C; ++c) {
                double s = w_bias[c];
                for (int d = 0; d < dw; ++d) s += hid[d] * Ww2[(size_t)d * C + c];
                w[c] = exp(-sigm(s) / sqrt(exp(1.0)));
            }
            double *v0t = v0_out + ((size_t)b * T + t) * C;
            if (!v0) {
                for (int c = 0; c < C; ++c) v0t[c] = v[c];
            } else {
                const double *v0i = v0 + ((size_t)b * T + t) * C;
                for (int d = 0; d < dv; ++d) {
                    double s = 0.0;
                    for (int c = 0; c < C; ++c) s += xv[c] * Wv1[(size_t)c * dv + d];
                    hid[d] = s;
                }
                for (int c = 0; c < C; ++c) {
                    double s = v_bias[c];
                    for (int d = 0; d < dv; ++d) s += hid[d] * Wv2[(size_t)d * C + c];
                    v[c] += (v0i[c] - v[c]) * sigm(s);
                    v0t[c] = v0i[c];
                }
            }
            for (int d = 0; d < da; ++d) {   /* rate: no activation between the two factors */
                double s = 0.0;
                for (int c = 0; c < C; ++c) s += xa[c] * Wa1[(size_t)c * da + d];
                hid[d] = s;
            }
            for (int c = 0; c < C; ++c) {
                double s = a_bias[c];
                for (int d = 0; d < da; ++d) s += hid[d] * Wa2[(size_t)d * C + c];
                a[c] = sigm(s);
            }
            for (int d = 0; d < dg; ++d) {   /* gate: sigmoid on the hidden value, then Wg2 */
                double s = 0.0;
                for (int c = 0; c < C; ++c) s += xg[c] * Wg1[(size_t)c * dg + d];
                hid[d] = sigm(s);
            }
            for (int c = 0; c < C; ++c) {
                double s = 0.0;
                for (int d = 0; d < dg; ++d) s += hid[d] * Wg2[(size_t)d * C + c];
                g[c] = s;
            }
            for (int c = 0; c < C; ++c) kk[c] = k[c] * k_k[c];
            for (int c = 0; c < C; ++c) k[c] += k[c] * (a[c] - 1.0) * k_a[c];
            for (int h = 0; h < H; ++h) {
                double ss = 0.0;
                for (int j = 0; j < N; ++j) ss += kk[h * N + j] * kk[h * N + j];
                double nrm = sqrt(ss);
                if (nrm < 1e-12) nrm = 1e-12;
                for (int j = 0; j < N; ++j) kk[h * N + j] /= nrm;
            }
            for (int h = 0; h < H; ++h) {
                double *Sh = Sb + (size_t)h * N * N;
                const double *wh = w + h * N, *kh = k + h * N, *vh = v + h * N, *kkh = kk + h * N;
                const double *ah = a + h * N, *rh = r + h * N;
                for (int i = 0; i < N; ++i) {
                    double s = 0.0;
                    for (int j = 0; j < N; ++j) s += Sh[i * N + j] * kkh[j];
                    sk[i] = s;
                }
                for (int i = 0; i < N; ++i)
                    for (int j = 0; j < N; ++j)
                        Sh[i * N + j] = Sh[i * N + j] * wh[j] - sk[i] * (kkh[j] * ah[j]) + vh[i] * kh[j];
                for (int i = 0; i < N; ++i) {
                    double s = 0.0;
                    for (int j = 0; j < N; ++j) s += Sh[i * N + j] * rh[j];
                    y[h * N + i] = s;
                }
                double mean = 0.0, var = 0.0, bonus = 0.0;
                for (int i = 0; i < N; ++i) mean += y[h * N + i];
                mean /= N;
                for (int i = 0; i < N; ++i) var += (y[h * N + i] - mean) * (y[h * N + i] - mean);
                var /= N;
                for (int i = 0; i < N; ++i)
                    y[h * N + i] = (y[h * N + i] - mean) / sqrt(var + eps) * ln_w[h * N + i] + ln_b[h * N + i];
                for (int j = 0; j < N; ++j) bonus += rh[j] * kh[j] * r_k[h * N + j];
                for (int i = 0; i < N; ++i) y[h * N + i] += bonus * vh[i];
            }
            for (int c = 0; c < C; ++c) tmp[c] = y[c] * g[c];
            double *ot = out + ((size_t)b * T + t) * C;
            for (int o = 0; o < C; ++o) {
                double s = 0.0;
                for (int i = 0; i < C; ++i) s += Wo[(size_t)o * C + i] * tmp[i];
                ot[o] = s;
            }
            for (int c = 0; c < C; ++c) xp[c] = xt[c];
        }
        for (int c = 0; c < C; ++c) last_out[(size_t)b * C + c] = xp[c];
    }
    free(buf);
    return 0;
}
