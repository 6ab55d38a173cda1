/*
 * ssd_oracle.c — plain, slow, fp64 CPU oracle for the Mamba-2 SSD layer.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or
 * load this file: only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark do. It shares no code, header or table with the CUDA library.
 *
 * What it computes (citations name the web page and the section on it):
 *
 *  - ssd_oracle_forward: the sequential recurrence, one (batch, head) at a time,
 *      a_t = exp(dt[t,h] * A[h])
 *      h   = a_t * h + dt[t,h] * x_t B_t^T          (state h is P x N)
 *      y_t = h C_t + D[h] * x_t
 *    "Mamba-2" (docsaid.org), sections "Writing the SSM as one matrix"
 *    (h_t = A_t h_{t-1} + B_t x_t, y_t = C_t^T h_t) and "Simplifying A to one
 *    number" (A_t = a_t I, scalar a_t in [0,1]); the discretisation
 *    a = exp(dt A), B-bar = dt B follows the simplified selective-scan code of
 *    "Mamba paper review" (youngju.dev), section 3.3 "Hardware-aware
 *    algorithm". Multi-head with B, C shared by a group of heads: "Mamba-2",
 *    section "Mamba-2 block", item 2 (multi-head).
 *
 *  - ssd_oracle_mask / ssd_oracle_quadratic: the quadratic ("attention") form
 *    y = (L o C B^T)(dt o x) + D x, with L_ji = a_j * ... * a_{i+1} for j >= i
 *    and 0 above the diagonal; "Mamba-2" (docsaid.org), section "Simplifying A
 *    to one number", the equation for M = L o (C B^T); "Mamba-2 SSD note"
 *    (0h-n0.github.io), section "SSD layer: equivalence under the scalar
 *    constraint". The mask is built as a literal product of the a_k, not from
 *    cumulative sums, so it does not share a single step with the recurrence.
 *
 *  - ssd_oracle_scan_core: the recurrence on given per-step decays a_t and
 *    input scales s_t for one head, as in the four-token hand calculation of
 *    "Mamba-2", section "Computing with four tokens" (there s_t = 1, P = 1).
 *
 *  - ssd_oracle_step: one decode step from a given state, the recurrent form
 *    used for generation ("Mamba-2", section "Computing with four tokens",
 *    closing remarks on the recurrent route having constant memory).
 *
 * Layouts (row-major, contiguous, all fp64):
 *   x[B][L][H][P], dt[B][L][H], A[H], Bm[B][L][G][N], Cm[B][L][G][N], D[H],
 *   y[B][L][H][P], state / final_state[B][H][P][N]. Head h reads group
 *   g = h / (H / G).
 *
 * Return value: 0 on success, -1 on an invalid argument.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

static int dims_ok(int B, int L, int H, int P, int G, int N)
{
    if (B < 0 || L < 0 || H <= 0 || P <= 0 || G <= 0 || N <= 0) return 0;
    if (H % G != 0) return 0;
    return 1;
}

/* One (batch, head) pair of the sequential recurrence. */
static void forward_one(const double* x, const double* dt, const double* A,
                        const double* Bm, const double* Cm, const double* D,
                        const double* init_state, double* y, double* final_state,
                        int b, int h, int L, int H, int P, int G, int N, double* hs)
{
    const int g = h / (H / G);
    const double Dh = D ? D[h] : 0.0;
    if (init_state)
        memcpy(hs, init_state + ((size_t)b * H + h) * P * N, sizeof(double) * P * N);
    else
        memset(hs, 0, sizeof(double) * P * N);

    for (int t = 0; t < L; ++t) {
        const double d = dt[((size_t)b * L + t) * H + h];
        const double a = exp(d * A[h]);
        const double* xt = x + (((size_t)b * L + t) * H + h) * P;
        const double* Bt = Bm + (((size_t)b * L + t) * G + g) * N;
        const double* Ct = Cm + (((size_t)b * L + t) * G + g) * N;
        double* yt = y + (((size_t)b * L + t) * H + h) * P;
        for (int p = 0; p < P; ++p) {
            double* hp = hs + (size_t)p * N;
            const double u = d * xt[p];
            double acc = 0.0;
            for (int n = 0; n < N; ++n) {
                hp[n] = a * hp[n] + u * Bt[n];
                acc += hp[n] * Ct[n];
            }
            yt[p] = acc + Dh * xt[p];
        }
    }
    if (final_state)
        memcpy(final_state + ((size_t)b * H + h) * P * N, hs, sizeof(double) * P * N);
}

typedef struct {
    const double *x, *dt, *A, *Bm, *Cm, *D, *init_state;
    double *y, *final_state;
    int B, L, H, P, G, N;
    int first, stride;
} fwd_job;

static void* fwd_worker(void* arg)
{
    fwd_job* j = (fwd_job*)arg;
    double* hs = (double*)malloc(sizeof(double) * (size_t)j->P * j->N);
    if (!hs) return (void*)1;
    for (int bh = j->first; bh < j->B * j->H; bh += j->stride)
        forward_one(j->x, j->dt, j->A, j->Bm, j->Cm, j->D, j->init_state, j->y,
                    j->final_state, bh / j->H, bh % j->H, j->L, j->H, j->P, j->G,
                    j->N, hs);
    free(hs);
    return NULL;
}

int ssd_oracle_forward(const double* x, const double* dt, const double* A,
                       const double* Bm, const double* Cm, const double* D,
                       const double* init_state, double* y, double* final_state,
                       int B, int L, int H, int P, int G, int N, int nthreads)
{
    if (!dims_ok(B, L, H, P, G, N)) return -1;
    if (!x || !dt || !A || !Bm || !Cm || !y) return -1;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > B * H) nthreads = B * H > 0 ? B * H : 1;
    fwd_job* jobs = (fwd_job*)calloc((size_t)nthreads, sizeof(fwd_job));
    pthread_t* tids = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !tids) { free(jobs); free(tids); return -1; }
    int rc = 0;
    for (int i = 0; i < nthreads; ++i) {
        fwd_job j = {x, dt, A, Bm, Cm, D, init_state, y, final_state,
                     B, L, H, P, G, N, i, nthreads};
        jobs[i] = j;
    }
    if (nthreads == 1) {
        rc = fwd_worker(&jobs[0]) ? -1 : 0;
    } else {
        int started = 0;
        for (int i = 0; i < nthreads; ++i) {
            if (pthread_create(&tids[i], NULL, fwd_worker, &jobs[i]) != 0) { rc = -1; break; }
            ++started;
        }
        for (int i = 0; i < started; ++i) {
            void* r = NULL;
            pthread_join(tids[i], &r);
            if (r) rc = -1;
        }
    }
    free(jobs);
    free(tids);
    return rc;
}

/* L[j][i] = a[j] * a[j-1] * ... * a[i+1] for j >= i (empty product = 1), else 0. */
int ssd_oracle_mask(const double* a, int L, double* Lmat)
{
    if (!a || !Lmat || L < 0) return -1;
    for (int j = 0; j < L; ++j) {
        for (int i = 0; i < L; ++i) {
            double v = 0.0;
            if (j >= i) {
                v = 1.0;
                for (int k = i + 1; k <= j; ++k) v *= a[k];
            }
            Lmat[(size_t)j * L + i] = v;
        }
    }
    return 0;
}

/* Brute-force quadratic form, O(L^2 (N + P)) per (b, h): tiny inputs only. */
int ssd_oracle_quadratic(const double* x, const double* dt, const double* A,
                         const double* Bm, const double* Cm, const double* D,
                         double* y, int B, int L, int H, int P, int G, int N)
{
    if (!dims_ok(B, L, H, P, G, N)) return -1;
    if (!x || !dt || !A || !Bm || !Cm || !y) return -1;
    double* a = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    double* Lm = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1) * (L > 0 ? L : 1));
    if (!a || !Lm) { free(a); free(Lm); return -1; }
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            const int g = h / (H / G);
            const double Dh = D ? D[h] : 0.0;
            for (int t = 0; t < L; ++t) a[t] = exp(dt[((size_t)b * L + t) * H + h] * A[h]);
            ssd_oracle_mask(a, L, Lm);
            for (int j = 0; j < L; ++j) {
                const double* Cj = Cm + (((size_t)b * L + j) * G + g) * N;
                double* yj = y + (((size_t)b * L + j) * H + h) * P;
                const double* xj = x + (((size_t)b * L + j) * H + h) * P;
                for (int p = 0; p < P; ++p) yj[p] = Dh * xj[p];
                for (int i = 0; i <= j; ++i) {
                    const double* Bi = Bm + (((size_t)b * L + i) * G + g) * N;
                    double cb = 0.0;
                    for (int n = 0; n < N; ++n) cb += Cj[n] * Bi[n];
                    const double m = Lm[(size_t)j * L + i] * cb * dt[((size_t)b * L + i) * H + h];
                    const double* xi = x + (((size_t)b * L + i) * H + h) * P;
                    for (int p = 0; p < P; ++p) yj[p] += m * xi[p];
                }
            }
        }
    }
    free(a);
    free(Lm);
    return 0;
}

/* Recurrence on given decays a[t] and input scales s[t], one head:
 * h = a_t h + s_t x_t B_t^T, y_t = h C_t.  x[L][P], Bm/Cm[L][N], y[L][P], h[P][N]. */
int ssd_oracle_scan_core(const double* a, const double* s, const double* x,
                         const double* Bm, const double* Cm, double* y, double* h,
                         int L, int P, int N)
{
    if (!a || !s || !x || !Bm || !Cm || !y || !h || L < 0 || P <= 0 || N <= 0) return -1;
    memset(h, 0, sizeof(double) * (size_t)P * N);
    for (int t = 0; t < L; ++t) {
        for (int p = 0; p < P; ++p) {
            double acc = 0.0;
            for (int n = 0; n < N; ++n) {
                double* hv = h + (size_t)p * N + n;
                *hv = a[t] * *hv + s[t] * x[(size_t)t * P + p] * Bm[(size_t)t * N + n];
                acc += *hv * Cm[(size_t)t * N + n];
            }
            y[(size_t)t * P + p] = acc;
        }
    }
    return 0;
}

/* One decode step: x[B][H][P], dt[B][H], Bm/Cm[B][G][N], state[B][H][P][N] in/out,
 * y[B][H][P]. */
int ssd_oracle_step(const double* x, const double* dt, const double* A,
                    const double* Bm, const double* Cm, const double* D,
                    double* state, double* y, int B, int H, int P, int G, int N)
{
    if (!dims_ok(B, 1, H, P, G, N)) return -1;
    if (!x || !dt || !A || !Bm || !Cm || !state || !y) return -1;
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            const int g = h / (H / G);
            const double d = dt[(size_t)b * H + h];
            const double a = exp(d * A[h]);
            const double Dh = D ? D[h] : 0.0;
            const double* xt = x + ((size_t)b * H + h) * P;
            const double* Bt = Bm + ((size_t)b * G + g) * N;
            const double* Ct = Cm + ((size_t)b * G + g) * N;
            double* hs = state + ((size_t)b * H + h) * P * N;
            for (int p = 0; p < P; ++p) {
                double acc = 0.0;
                for (int n = 0; n < N; ++n) {
                    double* hv = hs + (size_t)p * N + n;
                    *hv = a * *hv + d * xt[p] * Bt[n];
                    acc += *hv * Ct[n];
                }
                y[(size_t)b * H * P + (size_t)h * P + p] = acc + Dh * xt[p];
            }
        }
    }
    return 0;
}
