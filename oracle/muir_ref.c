/*
 * muir_ref.c -- token-by-token fp64 oracle for the Muir gated delta rule.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously correct CPU
 * definition that the CUDA path is checked against.  Only tests/,
 * __graft_entry__.smoke() and bench.py's cpu_baseline leg may load it.  It
 * shares no code, header, table or helper with the CUDA library, and the
 * CUDA library never calls it.
 *
 * Source of the arithmetic: "Muir: Linear Attention with Sensitivity-Allocated
 * Gating and Matched-Filter Readout" (arXiv 2611.08376), as summarised on the
 * wolonglab.org page, section "Methodology", equations eq:gdn2 and eq:ours.
 * The page prints only the labels; its prose says the state is decayed
 * row-wise, the prediction for the current key is erased, a gated value is
 * written, and a fifth gate gamma_t scales the normalised query only at
 * readout.  The formula written out below is that prose made explicit:
 *
 *     P_t   = diag(exp(g_t)) S_{t-1}                 (row-wise decay)
 *     y_t   = P_t^T k_t                              (prediction for k_t)
 *     S_t   = P_t - (e_t * k_t) y_t^T + k_t (w_t * v_t)^T   (erase, write)
 *     o_t   = S_t^T (gamma_t * q_t)                  (readout after update)
 *
 * S is d_k x d_v with rows indexed by key channels.  g, e, gamma, q, k live on
 * key channels; v, w on value channels.  No 1/sqrt(d_k) scaling, no output
 * gate: those are outside the recurrence.
 *
 * Layout: token-major [B][T][H][d] for per-token inputs, [B][H][d_k][d_v] for
 * states, all double.  Work is split over (b, h) pairs with pthreads.
 *
 * Backward: plain back-propagation through time of the four lines above, one
 * token at a time in reverse, recomputing S_{t-1} from checkpoints.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int B, T, H, dk, dv;
} ref_dims;

/* index of element (b, t, h, j) in a [B][T][H][d] array */
static inline size_t tok_idx(const ref_dims* D, int b, int t, int h, int j, int d) {
    return (((size_t)b * D->T + t) * D->H + h) * (size_t)d + j;
}

/* ---------------------------------------------------------------- threads */

typedef void (*unit_fn)(void* ctx, int unit);

typedef struct {
    unit_fn fn;
    void* ctx;
    int n_units;
    int next;
    pthread_mutex_t lock;
} pool_t;

static void* pool_worker(void* arg) {
    pool_t* p = (pool_t*)arg;
    for (;;) {
        pthread_mutex_lock(&p->lock);
        int u = p->next++;
        pthread_mutex_unlock(&p->lock);
        if (u >= p->n_units) break;
        p->fn(p->ctx, u);
    }
    return NULL;
}

static void run_units(unit_fn fn, void* ctx, int n_units, int n_threads) {
    if (n_threads < 1) n_threads = 1;
    if (n_threads > n_units) n_threads = n_units;
    pool_t p;
    p.fn = fn;
    p.ctx = ctx;
    p.n_units = n_units;
    p.next = 0;
    pthread_mutex_init(&p.lock, NULL);
    if (n_threads <= 1) {
        pool_worker(&p);
    } else {
        pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)n_threads);
        for (int i = 0; i < n_threads; ++i) pthread_create(&th[i], NULL, pool_worker, &p);
        for (int i = 0; i < n_threads; ++i) pthread_join(th[i], NULL);
        free(th);
    }
    pthread_mutex_destroy(&p.lock);
}

/* ------------------------------------------------------------ one token */

/* Advance one state by one token.  Sp (dk x dv) is S_{t-1} on entry and S_t
 * on exit.  y (dv) receives y_t, P (dk x dv, may be NULL) receives P_t. */
static void token_update(int dk, int dv, double* S, const double* q, const double* k,
                         const double* v, const double* g, const double* e,
                         const double* w, const double* gam, double* o, double* y,
                         double* P) {
    /* P = diag(exp g) S ;  y = P^T k */
    for (int c = 0; c < dv; ++c) y[c] = 0.0;
    for (int j = 0; j < dk; ++j) {
        double dj = exp(g[j]);
        double* row = S + (size_t)j * dv;
        for (int c = 0; c < dv; ++c) {
            row[c] *= dj;
            y[c] += row[c] * k[j];
        }
        if (P) memcpy(P + (size_t)j * dv, row, sizeof(double) * (size_t)dv);
    }
    /* S = P - (e*k) y^T + k (w*v)^T */
    for (int j = 0; j < dk; ++j) {
        double aj = e[j] * k[j];
        double kj = k[j];
        double* row = S + (size_t)j * dv;
        for (int c = 0; c < dv; ++c) row[c] = row[c] - aj * y[c] + kj * (w[c] * v[c]);
    }
    /* o = S^T (gamma * q) */
    if (o) {
        for (int c = 0; c < dv; ++c) o[c] = 0.0;
        for (int j = 0; j < dk; ++j) {
            double qj = gam ? gam[j] * q[j] : q[j];
            const double* row = S + (size_t)j * dv;
            for (int c = 0; c < dv; ++c) o[c] += row[c] * qj;
        }
    }
}

/* ---------------------------------------------------------------- forward */

typedef struct {
    ref_dims D;
    const double *q, *k, *v, *g, *e, *w, *gam, *S0;
    double *o, *S_out;
} fwd_ctx;

static void gather_tok(const ref_dims* D, const double* src, int b, int t, int h, int d,
                       double* dst) {
    memcpy(dst, src + tok_idx(D, b, t, h, 0, d), sizeof(double) * (size_t)d);
}

static void fwd_unit(void* vctx, int unit) {
    fwd_ctx* C = (fwd_ctx*)vctx;
    const ref_dims* D = &C->D;
    int b = unit / D->H, h = unit % D->H;
    int dk = D->dk, dv = D->dv;
    size_t sz = (size_t)dk * dv;
    double* S = (double*)malloc(sizeof(double) * sz);
    double* buf = (double*)malloc(sizeof(double) * (size_t)(6 * dk + 4 * dv));
    double *q = buf, *k = q + dk, *g = k + dk, *e = g + dk, *gm = e + dk, *pad = gm + dk;
    double *v = pad + dk, *w = v + dv, *o = w + dv, *y = o + dv;
    (void)pad;
    if (C->S0)
        memcpy(S, C->S0 + ((size_t)b * D->H + h) * sz, sizeof(double) * sz);
    else
        memset(S, 0, sizeof(double) * sz);
    for (int t = 0; t < D->T; ++t) {
        gather_tok(D, C->q, b, t, h, dk, q);
        gather_tok(D, C->k, b, t, h, dk, k);
        gather_tok(D, C->g, b, t, h, dk, g);
        gather_tok(D, C->e, b, t, h, dk, e);
        if (C->gam) gather_tok(D, C->gam, b, t, h, dk, gm);
        gather_tok(D, C->v, b, t, h, dv, v);
        gather_tok(D, C->w, b, t, h, dv, w);
        token_update(dk, dv, S, q, k, v, g, e, w, C->gam ? gm : NULL, o, y, NULL);
        if (C->o) memcpy(C->o + tok_idx(D, b, t, h, 0, dv), o, sizeof(double) * (size_t)dv);
    }
    if (C->S_out) memcpy(C->S_out + ((size_t)b * D->H + h) * sz, S, sizeof(double) * sz);
    free(buf);
    free(S);
}

/* o may be NULL; S_out may be NULL; S0 NULL means zeros; gamma NULL means 1. */
int muir_ref_fwd(int B, int T, int H, int dk, int dv, const double* q, const double* k,
                 const double* v, const double* g, const double* e, const double* w,
                 const double* gamma, const double* S0, double* o, double* S_out,
                 int n_threads) {
    if (B <= 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0) return 1;
    fwd_ctx C = {{B, T, H, dk, dv}, q, k, v, g, e, w, gamma, S0, o, S_out};
    run_units(fwd_unit, &C, B * H, n_threads);
    return 0;
}

/* ---------------------------------------------------------------- backward */

typedef struct {
    ref_dims D;
    const double *q, *k, *v, *g, *e, *w, *gam, *S0, *dO, *dS_final;
    double *dq, *dk, *dv, *dg, *de, *dw, *dgam, *dS0;
    int ckpt;
} bwd_ctx;

static void bwd_unit(void* vctx, int unit) {
    bwd_ctx* C = (bwd_ctx*)vctx;
    const ref_dims* D = &C->D;
    int b = unit / D->H, h = unit % D->H;
    int dk = D->dk, dv = D->dv, T = D->T, L = C->ckpt;
    size_t sz = (size_t)dk * dv;
    int n_seg = (T + L - 1) / L;
    /* checkpoints: state before token s*L */
    double* ck = (double*)malloc(sizeof(double) * sz * (size_t)(n_seg + 1));
    double* seg = (double*)malloc(sizeof(double) * sz * (size_t)(L + 1)); /* S_{t-1} .. */
    double* S = (double*)malloc(sizeof(double) * sz);
    double* G = (double*)malloc(sizeof(double) * sz);
    double* P = (double*)malloc(sizeof(double) * sz);
    double* buf = (double*)malloc(sizeof(double) * (size_t)(12 * dk + 12 * dv));
    double *q = buf, *k = q + dk, *g = k + dk, *e = g + dk, *gm = e + dk;
    double *dqh = gm + dk, *da = dqh + dk, *dkk = da + dk, *dgg = dkk + dk, *a = dgg + dk;
    double *v = a + dk, *w = v + dv, *y = w + dv, *u = y + dv, *dO = u + dv;
    double *dy = dO + dv, *du = dy + dv, *tmp = du + dv;
    (void)tmp;

    if (C->S0)
        memcpy(S, C->S0 + ((size_t)b * D->H + h) * sz, sizeof(double) * sz);
    else
        memset(S, 0, sizeof(double) * sz);
    /* forward pass storing one state per checkpoint */
    for (int t = 0; t < T; ++t) {
        if (t % L == 0) memcpy(ck + (size_t)(t / L) * sz, S, sizeof(double) * sz);
        gather_tok(D, C->q, b, t, h, dk, q);
        gather_tok(D, C->k, b, t, h, dk, k);
        gather_tok(D, C->g, b, t, h, dk, g);
        gather_tok(D, C->e, b, t, h, dk, e);
        gather_tok(D, C->v, b, t, h, dv, v);
        gather_tok(D, C->w, b, t, h, dv, w);
        token_update(dk, dv, S, q, k, v, g, e, w, NULL, NULL, y, NULL);
    }
    /* G carries dL/dS_t from the future; start with dS_final */
    if (C->dS_final)
        memcpy(G, C->dS_final + ((size_t)b * D->H + h) * sz, sizeof(double) * sz);
    else
        memset(G, 0, sizeof(double) * sz);

    for (int s = n_seg - 1; s >= 0; --s) {
        int t0 = s * L, t1 = t0 + L < T ? t0 + L : T;
        /* recompute S_{t0-1} .. S_{t1-1}; seg[i] = S before token t0+i */
        memcpy(seg, ck + (size_t)s * sz, sizeof(double) * sz);
        for (int t = t0; t < t1 - 1; ++t) {
            double* Sn = seg + (size_t)(t - t0 + 1) * sz;
            memcpy(Sn, seg + (size_t)(t - t0) * sz, sizeof(double) * sz);
            gather_tok(D, C->k, b, t, h, dk, k);
            gather_tok(D, C->g, b, t, h, dk, g);
            gather_tok(D, C->e, b, t, h, dk, e);
            gather_tok(D, C->v, b, t, h, dv, v);
            gather_tok(D, C->w, b, t, h, dv, w);
            token_update(dk, dv, Sn, q, k, v, g, e, w, NULL, NULL, y, NULL);
        }
        for (int t = t1 - 1; t >= t0; --t) {
            const double* Sprev = seg + (size_t)(t - t0) * sz;
            gather_tok(D, C->q, b, t, h, dk, q);
            gather_tok(D, C->k, b, t, h, dk, k);
            gather_tok(D, C->g, b, t, h, dk, g);
            gather_tok(D, C->e, b, t, h, dk, e);
            if (C->gam) gather_tok(D, C->gam, b, t, h, dk, gm);
            gather_tok(D, C->v, b, t, h, dv, v);
            gather_tok(D, C->w, b, t, h, dv, w);
            gather_tok(D, C->dO, b, t, h, dv, dO);
            /* recompute P, y and S_t for this token */
            memcpy(S, Sprev, sizeof(double) * sz);
            token_update(dk, dv, S, q, k, v, g, e, w, NULL, NULL, y, P);
            for (int j = 0; j < dk; ++j) a[j] = e[j] * k[j];
            for (int c = 0; c < dv; ++c) u[c] = w[c] * v[c];
            /* readout o = S^T qhat:  dqhat = S dO ; G += qhat dO^T */
            for (int j = 0; j < dk; ++j) {
                double qh = C->gam ? gm[j] * q[j] : q[j];
                const double* row = S + (size_t)j * dv;
                double acc = 0.0;
                double* grow = G + (size_t)j * dv;
                for (int c = 0; c < dv; ++c) {
                    acc += row[c] * dO[c];
                    grow[c] += qh * dO[c];
                }
                dqh[j] = acc;
            }
            /* S = P - a y^T + k u^T, with G = dL/dS_t */
            for (int c = 0; c < dv; ++c) { dy[c] = 0.0; du[c] = 0.0; }
            for (int j = 0; j < dk; ++j) {
                const double* grow = G + (size_t)j * dv;
                double s_gy = 0.0, s_gu = 0.0;
                for (int c = 0; c < dv; ++c) {
                    s_gy += grow[c] * y[c];
                    s_gu += grow[c] * u[c];
                    dy[c] -= grow[c] * a[j];
                    du[c] += grow[c] * k[j];
                }
                da[j] = -s_gy;
                dkk[j] = s_gu;
            }
            /* y = P^T k :  dP = G + k dy^T ; dk += P dy */
            for (int j = 0; j < dk; ++j) {
                double* grow = G + (size_t)j * dv; /* becomes dP in place */
                const double* prow = P + (size_t)j * dv;
                double s_pdy = 0.0, s_pdp = 0.0;
                for (int c = 0; c < dv; ++c) {
                    grow[c] += k[j] * dy[c];
                    s_pdy += prow[c] * dy[c];
                    s_pdp += prow[c] * grow[c];
                }
                dkk[j] += s_pdy;
                dgg[j] = s_pdp; /* P = diag(exp g) S_{t-1}: dg = rowsum(P * dP) */
            }
            /* gates */
            size_t ik = tok_idx(D, b, t, h, 0, dk), iv = tok_idx(D, b, t, h, 0, dv);
            for (int j = 0; j < dk; ++j) {
                double qh_grad = dqh[j];
                if (C->dq) C->dq[ik + j] = C->gam ? qh_grad * gm[j] : qh_grad;
                if (C->dgam) C->dgam[ik + j] = qh_grad * q[j];
                if (C->de) C->de[ik + j] = da[j] * k[j];
                if (C->dk) C->dk[ik + j] = dkk[j] + da[j] * e[j];
                if (C->dg) C->dg[ik + j] = dgg[j];
            }
            for (int c = 0; c < dv; ++c) {
                if (C->dw) C->dw[iv + c] = du[c] * v[c];
                if (C->dv) C->dv[iv + c] = du[c] * w[c];
            }
            /* dS_{t-1} = diag(exp g) dP */
            for (int j = 0; j < dk; ++j) {
                double dj = exp(g[j]);
                double* grow = G + (size_t)j * dv;
                for (int c = 0; c < dv; ++c) grow[c] *= dj;
            }
        }
    }
    if (C->dS0) memcpy(C->dS0 + ((size_t)b * D->H + h) * sz, G, sizeof(double) * sz);
    free(buf);
    free(P);
    free(G);
    free(S);
    free(seg);
    free(ck);
}

/* Gradients of sum(o * dO) + sum(S_T * dS_final) w.r.t. every input.
 * Any output pointer may be NULL.  gamma NULL means 1 (then dgamma is q*dqhat
 * with qhat = q).  ckpt is the recompute segment length (>=1). */
int muir_ref_bwd(int B, int T, int H, int dk, int dv, const double* q, const double* k,
                 const double* v, const double* g, const double* e, const double* w,
                 const double* gamma, const double* S0, const double* dO,
                 const double* dS_final, double* dq, double* dk_, double* dv_, double* dg,
                 double* de, double* dw, double* dgamma, double* dS0, int ckpt,
                 int n_threads) {
    if (B <= 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0) return 1;
    if (ckpt < 1) ckpt = 64;
    bwd_ctx C = {{B, T, H, dk, dv}, q, k, v, g, e, w, gamma, S0, dO, dS_final,
                 dq, dk_, dv_, dg, de, dw, dgamma, dS0, ckpt};
    if (T == 0) {
        size_t sz = (size_t)dk * dv * B * H;
        if (dS0) {
            if (dS_final) memcpy(dS0, dS_final, sizeof(double) * sz);
            else memset(dS0, 0, sizeof(double) * sz);
        }
        return 0;
    }
    run_units(bwd_unit, &C, B * H, n_threads);
    return 0;
}

/* ------------------------------------------------------------ decode step */

/* One token for every (b, h).  Per-token tensors are [B][H][d].  gamma is
 * [B][H][dk] when gamma_static == 0, [H][dk] (shared by every b) when 1, and
 * NULL for gamma = 1.  S [B][H][dk][dv] is updated in place. */
int muir_ref_step(int B, int H, int dk, int dv, const double* q, const double* k,
                  const double* v, const double* g, const double* e, const double* w,
                  const double* gamma, int gamma_static, double* S, double* o) {
    if (B <= 0 || H <= 0 || dk <= 0 || dv <= 0) return 1;
    double* y = (double*)malloc(sizeof(double) * (size_t)dv);
    size_t sz = (size_t)dk * dv;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            size_t ik = ((size_t)b * H + h) * dk, iv = ((size_t)b * H + h) * dv;
            const double* gm = NULL;
            if (gamma) gm = gamma_static ? gamma + (size_t)h * dk : gamma + ik;
            token_update(dk, dv, S + ((size_t)b * H + h) * sz, q + ik, k + ik, v + iv, g + ik,
                         e + ik, w + iv, gm, o ? o + iv : NULL, y, NULL);
        }
    free(y);
    return 0;
}
