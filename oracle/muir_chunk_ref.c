/*
 * muir_chunk_ref.c -- chunked (WY / UT form) fp64 oracle of the Muir forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and
 * bench.py's cpu_baseline leg may load it.  It shares nothing with the CUDA
 * library, and it shares no code with muir_ref.c either: the two are
 * independent statements of the same recurrence, and the tests check each
 * against the other (results must not depend on the chunk size).
 *
 * Source: "Muir: Linear Attention with Sensitivity-Allocated Gating and
 * Matched-Filter Readout" (arXiv 2611.08376), wolonglab.org page, section
 * "Methodology": the training implementation writes each chunk as a triangular
 * system.  The page gives no equations; the chunk equations here are derived
 * from the token recurrence
 *     S_t = D_t S_{t-1} - (e_t*k_t)(k_t^T D_t S_{t-1}) + k_t (w_t*v_t)^T,
 *     o_t = S_t^T (gamma_t*q_t),   D_t = diag(exp g_t)
 * by unrolling it over one chunk of C tokens with chunk-start state S:
 *
 *   Gam_t = sum_{i<=t} g_i (inside the chunk),  gbar = Gam_C
 *   [X (*) Z]_{ts} = sum_j X_tj Z_sj exp(Gam_tj - Gam_sj)       (s <= t)
 *   L_A = strict lower part of K (*) A,  L_K = strict lower of K (*) K
 *   M_QK = lower incl. diagonal of Qh (*) K,  M_QA = same of Qh (*) A
 *   (I + L_A) Y = (K * e^Gam) S + L_K U            (y_t = k_t^T D_t S_{t-1})
 *   O  = (Qh * e^Gam) S + M_QK U - M_QA Y
 *   S' = diag(e^gbar) S + (K * e^{gbar-Gam})^T U - (A * e^{gbar-Gam})^T Y
 * with A = e*K, U = w*V, Qh = gamma*Q.  Every decay factor is formed from an
 * exact exponent difference (no pivots, no clamps); the triangular system is
 * solved by plain forward substitution.  W = (I+L_A)^{-1}(K*e^Gam) and
 * U' = (I+L_A)^{-1} L_K U are formed explicitly so that Y = W S + U'.
 * A last chunk shorter than C is allowed.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int B, T, H, dk, dv, C;
    const double *q, *k, *v, *g, *e, *w, *gam, *S0;
    double *o, *S_out, *S_chunks;
    int next;
    pthread_mutex_t lock;
} cref_job;

static size_t at(const cref_job* J, int b, int t, int h, int d) {
    return (((size_t)b * J->T + t) * J->H + h) * (size_t)d;
}

static void chunk_head(cref_job* J, int b, int h) {
    const int dk = J->dk, dv = J->dv, Cmax = J->C;
    const size_t sz = (size_t)dk * dv;
    double* S = (double*)calloc(sz, sizeof(double));
    double* Gam = (double*)malloc(sizeof(double) * (size_t)Cmax * dk);
    double* LA = (double*)malloc(sizeof(double) * (size_t)Cmax * Cmax);
    double* LK = (double*)malloc(sizeof(double) * (size_t)Cmax * Cmax);
    double* MQK = (double*)malloc(sizeof(double) * (size_t)Cmax * Cmax);
    double* MQA = (double*)malloc(sizeof(double) * (size_t)Cmax * Cmax);
    double* W = (double*)malloc(sizeof(double) * (size_t)Cmax * dk);
    double* Up = (double*)malloc(sizeof(double) * (size_t)Cmax * dv);
    double* Y = (double*)malloc(sizeof(double) * (size_t)Cmax * dv);
    double* Sn = (double*)malloc(sizeof(double) * sz);
    if (J->S0) memcpy(S, J->S0 + ((size_t)b * J->H + h) * sz, sizeof(double) * sz);

    int n_chunks = (J->T + Cmax - 1) / Cmax;
    for (int n = 0; n < n_chunks; ++n) {
        int t0 = n * Cmax;
        int C = J->T - t0 < Cmax ? J->T - t0 : Cmax;
        if (J->S_chunks)
            memcpy(J->S_chunks + (((size_t)b * J->H + h) * n_chunks + n) * sz, S,
                   sizeof(double) * sz);
#define Kv(t, j) (J->k[at(J, b, t0 + (t), h, dk) + (j)])
#define Qv(t, j) (J->q[at(J, b, t0 + (t), h, dk) + (j)] * (J->gam ? J->gam[at(J, b, t0 + (t), h, dk) + (j)] : 1.0))
#define Av(t, j) (J->e[at(J, b, t0 + (t), h, dk) + (j)] * Kv(t, j))
#define Uv(t, c) (J->w[at(J, b, t0 + (t), h, dv) + (c)] * J->v[at(J, b, t0 + (t), h, dv) + (c)])
        /* cumulative log decay inside the chunk */
        for (int j = 0; j < dk; ++j) {
            double run = 0.0;
            for (int t = 0; t < C; ++t) {
                run += J->g[at(J, b, t0 + t, h, dk) + j];
                Gam[(size_t)t * dk + j] = run;
            }
        }
        const double* gbar = Gam + (size_t)(C - 1) * dk;
        /* decay-masked products */
        for (int t = 0; t < C; ++t)
            for (int s = 0; s < C; ++s) {
                double la = 0, lk = 0, mqk = 0, mqa = 0;
                if (s <= t) {
                    for (int j = 0; j < dk; ++j) {
                        double f = exp(Gam[(size_t)t * dk + j] - Gam[(size_t)s * dk + j]);
                        double kt = Kv(t, j), qt = Qv(t, j), ks = Kv(s, j), as = Av(s, j);
                        la += kt * as * f;
                        lk += kt * ks * f;
                        mqk += qt * ks * f;
                        mqa += qt * as * f;
                    }
                }
                size_t i = (size_t)t * C + s;
                LA[i] = s < t ? la : 0.0;
                LK[i] = s < t ? lk : 0.0;
                MQK[i] = mqk;
                MQA[i] = mqa;
            }
        /* forward substitution: (I + L_A) [W | U'] = [K e^Gam | L_K U] */
        for (int t = 0; t < C; ++t) {
            for (int j = 0; j < dk; ++j) {
                double r = Kv(t, j) * exp(Gam[(size_t)t * dk + j]);
                for (int s = 0; s < t; ++s) r -= LA[(size_t)t * C + s] * W[(size_t)s * dk + j];
                W[(size_t)t * dk + j] = r;
            }
            for (int c = 0; c < dv; ++c) {
                double r = 0.0;
                for (int s = 0; s < t; ++s) r += LK[(size_t)t * C + s] * Uv(s, c);
                for (int s = 0; s < t; ++s) r -= LA[(size_t)t * C + s] * Up[(size_t)s * dv + c];
                Up[(size_t)t * dv + c] = r;
            }
        }
        /* Y = W S + U' */
        for (int t = 0; t < C; ++t)
            for (int c = 0; c < dv; ++c) {
                double acc = Up[(size_t)t * dv + c];
                for (int j = 0; j < dk; ++j) acc += W[(size_t)t * dk + j] * S[(size_t)j * dv + c];
                Y[(size_t)t * dv + c] = acc;
            }
        /* O = (Qh e^Gam) S + M_QK U - M_QA Y */
        if (J->o)
            for (int t = 0; t < C; ++t)
                for (int c = 0; c < dv; ++c) {
                    double acc = 0.0;
                    for (int j = 0; j < dk; ++j)
                        acc += Qv(t, j) * exp(Gam[(size_t)t * dk + j]) * S[(size_t)j * dv + c];
                    for (int s = 0; s <= t; ++s)
                        acc += MQK[(size_t)t * C + s] * Uv(s, c) - MQA[(size_t)t * C + s] * Y[(size_t)s * dv + c];
                    J->o[at(J, b, t0 + t, h, dv) + c] = acc;
                }
        /* S' = diag(e^gbar) S + (K e^{gbar-Gam})^T U - (A e^{gbar-Gam})^T Y */
        for (int j = 0; j < dk; ++j)
            for (int c = 0; c < dv; ++c) {
                double acc = exp(gbar[j]) * S[(size_t)j * dv + c];
                for (int t = 0; t < C; ++t) {
                    double f = exp(gbar[j] - Gam[(size_t)t * dk + j]);
                    acc += Kv(t, j) * f * Uv(t, c) - Av(t, j) * f * Y[(size_t)t * dv + c];
                }
                Sn[(size_t)j * dv + c] = acc;
            }
        memcpy(S, Sn, sizeof(double) * sz);
#undef Kv
#undef Qv
#undef Av
#undef Uv
    }
    if (J->S_out) memcpy(J->S_out + ((size_t)b * J->H + h) * sz, S, sizeof(double) * sz);
    free(Sn); free(Y); free(Up); free(W); free(MQA); free(MQK); free(LK); free(LA);
    free(Gam); free(S);
}

static void* cref_worker(void* arg) {
    cref_job* J = (cref_job*)arg;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int u = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (u >= J->B * J->H) break;
        chunk_head(J, u / J->H, u % J->H);
    }
    return NULL;
}

/* Chunked forward.  S_chunks (may be NULL) receives the chunk-start state of
 * every chunk, [B][H][ceil(T/C)][dk][dv]. */
int muir_chunk_ref_fwd(int B, int T, int H, int dk, int dv, int C, const double* q,
                       const double* k, const double* v, const double* g, const double* e,
                       const double* w, const double* gamma, const double* S0, double* o,
                       double* S_out, double* S_chunks, int n_threads) {
    if (B <= 0 || T <= 0 || H <= 0 || dk <= 0 || dv <= 0 || C <= 0) return 1;
    cref_job J;
    J.B = B; J.T = T; J.H = H; J.dk = dk; J.dv = dv; J.C = C;
    J.q = q; J.k = k; J.v = v; J.g = g; J.e = e; J.w = w; J.gam = gamma; J.S0 = S0;
    J.o = o; J.S_out = S_out; J.S_chunks = S_chunks;
    J.next = 0;
    pthread_mutex_init(&J.lock, NULL);
    if (n_threads < 1) n_threads = 1;
    if (n_threads > B * H) n_threads = B * H;
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)n_threads);
    for (int i = 0; i < n_threads; ++i) pthread_create(&th[i], NULL, cref_worker, &J);
    for (int i = 0; i < n_threads; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J.lock);
    return 0;
}
