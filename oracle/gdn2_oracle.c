/*
 * fp64 CPU oracle for the Gated DeltaNet-2 recurrence.  TEST INFRASTRUCTURE ONLY:
 * the parity tests, the smoke check and the benchmark's CPU-baseline leg call it;
 * the library path never does.  It shares no code with the CUDA path.
 *
 * What it computes (page "NVIDIA представила Gated DeltaNet-2 ...", section
 * "Техническая схема", the state-update equation), per batch element b and head h:
 *
 *     S_t = (I - k_t (b_t ⊙ k_t)^T) Diag(alpha_t) S_{t-1} + k_t (w_t ⊙ v_t)^T
 *     o_t = S_t^T q_t                       (read-out of the post-update state)
 *
 * with S in R^{d_k x d_v}: Diag(alpha_t) scales the key rows, the erase vector
 * b_t ⊙ k_t reads along keys and the write vector w_t ⊙ v_t lives on the value
 * axis.  No 1/sqrt(d_k) scale is applied to q.  The equation is evaluated as
 * written, in this order, one token at a time:
 *
 *     X   = Diag(alpha_t) S_{t-1}              (decay)
 *     r   = X^T (b_t ⊙ k_t)                    (what the erase projector removes)
 *     S_t = X - k_t r^T + k_t (w_t ⊙ v_t)^T    (erase, then write)
 *     o_t = S_t^T q_t
 *
 * Everything is fp64; inputs arrive as fp64 copies of the stored (bf16 / fp32)
 * values.  Layouts: tokens [B, T, H, d] (d fastest), states [B, H, d_k, d_v].
 *
 * Parity is pinned by tests/test_oracle_pins.py (brute-force matrix products,
 * the KDA and Gated DeltaNet collapsed-gate restatements, closed forms and
 * invariants); see the header of that file.
 */
#include <pthread.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    const double *q, *k, *v, *alpha, *b, *w, *S0;
    double *o, *ST;
    int B, H, T, K, V;
    int first_chain, last_chain; /* chains are (b, h) pairs, index b*H + h */
} job_t;

/* One (b, h) chain, tokens 0..T-1. */
static void run_chain(const job_t *J, int chain, double *S, double *r) {
    const int B = J->B, H = J->H, T = J->T, K = J->K, V = J->V;
    const int bb = chain / H, hh = chain % H;
    (void)B;
    if (J->S0)
        memcpy(S, J->S0 + (size_t)chain * K * V, sizeof(double) * (size_t)K * V);
    else
        memset(S, 0, sizeof(double) * (size_t)K * V);

    for (int t = 0; t < T; ++t) {
        const size_t tk = (((size_t)bb * T + t) * H + hh) * (size_t)K;
        const size_t tv = (((size_t)bb * T + t) * H + hh) * (size_t)V;
        const double *qt = J->q + tk, *kt = J->k + tk, *at = J->alpha + tk, *bt = J->b + tk;
        const double *vt = J->v + tv, *wt = J->w + tv;

        /* X = Diag(alpha_t) S_{t-1}: row c of S is scaled by alpha_t[c] */
        for (int c = 0; c < K; ++c)
            for (int j = 0; j < V; ++j) S[(size_t)c * V + j] *= at[c];

        /* r = X^T (b_t ⊙ k_t) */
        for (int j = 0; j < V; ++j) r[j] = 0.0;
        for (int c = 0; c < K; ++c) {
            const double e = bt[c] * kt[c];
            for (int j = 0; j < V; ++j) r[j] += e * S[(size_t)c * V + j];
        }

        /* S_t = X - k_t r^T + k_t (w_t ⊙ v_t)^T */
        for (int c = 0; c < K; ++c)
            for (int j = 0; j < V; ++j)
                S[(size_t)c * V + j] += kt[c] * (wt[j] * vt[j] - r[j]);

        /* o_t = S_t^T q_t */
        if (J->o) {
            double *ot = J->o + tv;
            for (int j = 0; j < V; ++j) ot[j] = 0.0;
            for (int c = 0; c < K; ++c)
                for (int j = 0; j < V; ++j) ot[j] += qt[c] * S[(size_t)c * V + j];
        }
    }
    if (J->ST) memcpy(J->ST + (size_t)chain * K * V, S, sizeof(double) * (size_t)K * V);
}

static void *worker(void *p) {
    const job_t *J = (const job_t *)p;
    double *S = (double *)malloc(sizeof(double) * (size_t)J->K * J->V);
    double *r = (double *)malloc(sizeof(double) * (size_t)J->V);
    if (S && r)
        for (int ch = J->first_chain; ch < J->last_chain; ++ch) run_chain(J, ch, S, r);
    free(S);
    free(r);
    return NULL;
}

/*
 * Sequential recurrence over T tokens for all B*H chains.
 *   S0 may be NULL (zero initial state); o and ST may be NULL (not written).
 *   nthreads host threads split the chains (chains are independent).
 * Returns 0, or -1 on bad arguments.
 */
int gdn2_oracle_recurrence(const double *q, const double *k, const double *v, const double *alpha,
                           const double *b, const double *w, const double *S0, double *o, double *ST,
                           int B, int H, int T, int K, int V, int nthreads) {
    if (!q || !k || !v || !alpha || !b || !w) return -1;
    if (B < 0 || H < 0 || T < 0 || K <= 0 || V <= 0) return -1;
    const int chains = B * H;
    if (chains == 0) return 0;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > chains) nthreads = chains;
    if (nthreads > 256) nthreads = 256;
    job_t jobs[256];
    pthread_t tid[256];
    int per = (chains + nthreads - 1) / nthreads;
    int n = 0;
    for (int i = 0; i < nthreads; ++i) {
        int lo = i * per, hi = lo + per > chains ? chains : lo + per;
        if (lo >= hi) break;
        job_t J = {q, k, v, alpha, b, w, S0, o, ST, B, H, T, K, V, lo, hi};
        jobs[i] = J;
        n = i + 1;
    }
    if (n == 1) {
        worker(&jobs[0]);
        return 0;
    }
    for (int i = 0; i < n; ++i)
        if (pthread_create(&tid[i], NULL, worker, &jobs[i]) != 0) {
            worker(&jobs[i]);
            tid[i] = 0;
        }
    for (int i = 0; i < n; ++i)
        if (tid[i]) pthread_join(tid[i], NULL);
    return 0;
}

/*
 * One decode step: the same update for a single token per chain, state in place.
 *   tokens [B, H, d]; S [B, H, K, V] (in/out); o [B, H, V] (may be NULL).
 */
int gdn2_oracle_decode_step(const double *q, const double *k, const double *v, const double *alpha,
                            const double *b, const double *w, double *S, double *o, int B, int H, int K,
                            int V, int nthreads) {
    if (!S) return -1;
    /* a decode step is the recurrence over T = 1 starting from S, written back to S */
    return gdn2_oracle_recurrence(q, k, v, alpha, b, w, S, o, S, B, H, 1, K, V, nthreads);
}

/*
 * Gradient of a scalar loss L through the same recurrence (test infrastructure, like the rest
 * of this file): given dO = dL/do [B, T, H, d_v] and dST = dL/dS_T [B, H, d_k, d_v] (NULL: zero),
 * writes dq, dk, dalpha, db [B, T, H, d_k], dv, dw [B, T, H, d_v] and dS0 [B, H, d_k, d_v]
 * (NULL: not written).  The same page's chunkwise paragraph says only that the gradients must
 * account for the per-channel gates; this is the chain rule of each step as written above,
 * walked in reverse with every state S_t kept (T+1 states per chain), in the order of
 * oracle/backward.py:
 *
 *     dq_t = S_t dO_t;  G += q_t dO_t^T;  ddelta = G^T k_t;  dk_t = G delta_t
 *     de = -X ddelta (X = Diag(alpha_t) S_{t-1});  dX = G - e ddelta^T
 *     db_t = k_t ⊙ de;  dk_t += b_t ⊙ de;  dw_t = v_t ⊙ ddelta;  dv_t = w_t ⊙ ddelta
 *     dalpha_t = rowsum(dX ⊙ S_{t-1});  G = Diag(alpha_t) dX;   dS0 = G at the end
 */
typedef struct {
    const double *q, *k, *v, *alpha, *b, *w, *S0, *dO, *dST;
    double *dq, *dk, *dv, *dalpha, *db, *dw, *dS0;
    int H, T, K, V;
    int first_chain, last_chain;
} bjob_t;

static void bwd_chain(const bjob_t *J, int chain, double *states, double *deltas, double *G, double *dX,
                      double *dd, double *de) {
    const int H = J->H, T = J->T, K = J->K, V = J->V;
    const int bb = chain / H, hh = chain % H;
    const size_t KV = (size_t)K * V;
    if (J->S0)
        memcpy(states, J->S0 + (size_t)chain * KV, sizeof(double) * KV);
    else
        memset(states, 0, sizeof(double) * KV);
    /* forward, every state kept: states[t+1] = S_t (0-based t) */
    for (int t = 0; t < T; ++t) {
        const size_t tk = (((size_t)bb * T + t) * H + hh) * (size_t)K;
        const size_t tv = (((size_t)bb * T + t) * H + hh) * (size_t)V;
        const double *kt = J->k + tk, *at = J->alpha + tk, *bt = J->b + tk, *vt = J->v + tv, *wt = J->w + tv;
        const double *Sp = states + (size_t)t * KV;
        double *Sn = states + (size_t)(t + 1) * KV;
        double *dl = deltas + (size_t)t * V;
        for (int c = 0; c < K; ++c)
            for (int j = 0; j < V; ++j) Sn[(size_t)c * V + j] = at[c] * Sp[(size_t)c * V + j];
        for (int j = 0; j < V; ++j) dl[j] = 0.0;
        for (int c = 0; c < K; ++c) {
            const double e = bt[c] * kt[c];
            for (int j = 0; j < V; ++j) dl[j] += e * Sn[(size_t)c * V + j];
        }
        for (int j = 0; j < V; ++j) dl[j] = wt[j] * vt[j] - dl[j];
        for (int c = 0; c < K; ++c)
            for (int j = 0; j < V; ++j) Sn[(size_t)c * V + j] += kt[c] * dl[j];
    }
    /* reverse */
    if (J->dST)
        memcpy(G, J->dST + (size_t)chain * KV, sizeof(double) * KV);
    else
        memset(G, 0, sizeof(double) * KV);
    for (int t = T - 1; t >= 0; --t) {
        const size_t tk = (((size_t)bb * T + t) * H + hh) * (size_t)K;
        const size_t tv = (((size_t)bb * T + t) * H + hh) * (size_t)V;
        const double *qt = J->q + tk, *kt = J->k + tk, *at = J->alpha + tk, *bt = J->b + tk;
        const double *vt = J->v + tv, *wt = J->w + tv, *gt = J->dO + tv;
        const double *Sp = states + (size_t)t * KV, *Sn = states + (size_t)(t + 1) * KV;
        const double *dl = deltas + (size_t)t * V;
        double *dqt = J->dq + tk, *dkt = J->dk + tk, *dat = J->dalpha + tk, *dbt = J->db + tk;
        double *dvt = J->dv + tv, *dwt = J->dw + tv;
        /* o_t = S_t^T q_t */
        for (int c = 0; c < K; ++c) {
            double s = 0.0;
            for (int j = 0; j < V; ++j) s += Sn[(size_t)c * V + j] * gt[j];
            dqt[c] = s;
        }
        for (int c = 0; c < K; ++c)
            for (int j = 0; j < V; ++j) G[(size_t)c * V + j] += qt[c] * gt[j];
        /* S_t = X + k_t delta_t^T */
        for (int j = 0; j < V; ++j) dd[j] = 0.0;
        for (int c = 0; c < K; ++c)
            for (int j = 0; j < V; ++j) dd[j] += G[(size_t)c * V + j] * kt[c];
        for (int c = 0; c < K; ++c) {
            double s = 0.0;
            for (int j = 0; j < V; ++j) s += G[(size_t)c * V + j] * dl[j];
            dkt[c] = s;
        }
        /* delta_t = u_t - X^T e_t */
        for (int c = 0; c < K; ++c) {
            double s = 0.0;
            for (int j = 0; j < V; ++j) s += at[c] * Sp[(size_t)c * V + j] * dd[j];
            de[c] = -s;
        }
        for (int c = 0; c < K; ++c) {
            const double e = bt[c] * kt[c];
            for (int j = 0; j < V; ++j) dX[(size_t)c * V + j] = G[(size_t)c * V + j] - e * dd[j];
        }
        /* e_t = b_t ⊙ k_t, u_t = w_t ⊙ v_t */
        for (int c = 0; c < K; ++c) {
            dbt[c] = kt[c] * de[c];
            dkt[c] += bt[c] * de[c];
        }
        for (int j = 0; j < V; ++j) {
            dwt[j] = vt[j] * dd[j];
            dvt[j] = wt[j] * dd[j];
        }
        /* X = Diag(alpha_t) S_{t-1} */
        for (int c = 0; c < K; ++c) {
            double s = 0.0;
            for (int j = 0; j < V; ++j) s += dX[(size_t)c * V + j] * Sp[(size_t)c * V + j];
            dat[c] = s;
        }
        for (int c = 0; c < K; ++c)
            for (int j = 0; j < V; ++j) G[(size_t)c * V + j] = at[c] * dX[(size_t)c * V + j];
    }
    if (J->dS0) memcpy(J->dS0 + (size_t)chain * KV, G, sizeof(double) * KV);
}

static void *bwd_worker(void *p) {
    const bjob_t *J = (const bjob_t *)p;
    const size_t KV = (size_t)J->K * J->V;
    double *states = (double *)malloc(sizeof(double) * (size_t)(J->T + 1) * KV);
    double *deltas = (double *)malloc(sizeof(double) * ((size_t)J->T * J->V + 1));
    double *G = (double *)malloc(sizeof(double) * KV), *dX = (double *)malloc(sizeof(double) * KV);
    double *dd = (double *)malloc(sizeof(double) * (size_t)J->V), *de = (double *)malloc(sizeof(double) * (size_t)J->K);
    int ok = states && deltas && G && dX && dd && de;
    if (ok)
        for (int ch = J->first_chain; ch < J->last_chain; ++ch) bwd_chain(J, ch, states, deltas, G, dX, dd, de);
    free(states);
    free(deltas);
    free(G);
    free(dX);
    free(dd);
    free(de);
    return ok ? NULL : (void *)1;
}

/* Returns 0, -1 on bad arguments, -2 when a thread could not allocate its T+1 states. */
int gdn2_oracle_backward(const double *q, const double *k, const double *v, const double *alpha, const double *b,
                         const double *w, const double *S0, const double *dO, const double *dST, double *dq,
                         double *dk, double *dv, double *dalpha, double *db, double *dw, double *dS0, int B, int H,
                         int T, int K, int V, int nthreads) {
    if (!q || !k || !v || !alpha || !b || !w || !dO || !dq || !dk || !dv || !dalpha || !db || !dw) return -1;
    if (B < 0 || H < 0 || T < 0 || K <= 0 || V <= 0) return -1;
    const int chains = B * H;
    if (chains == 0) return 0;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > chains) nthreads = chains;
    if (nthreads > 256) nthreads = 256;
    bjob_t jobs[256];
    pthread_t tid[256];
    void *ret[256];
    int per = (chains + nthreads - 1) / nthreads, n = 0;
    for (int i = 0; i < nthreads; ++i) {
        int lo = i * per, hi = lo + per > chains ? chains : lo + per;
        if (lo >= hi) break;
        bjob_t J = {q, k, v, alpha, b, w, S0, dO, dST, dq, dk, dv, dalpha, db, dw, dS0, H, T, K, V, lo, hi};
        jobs[i] = J;
        n = i + 1;
    }
    int rc = 0;
    for (int i = 0; i < n; ++i) {
        ret[i] = NULL;
        if (n == 1 || pthread_create(&tid[i], NULL, bwd_worker, &jobs[i]) != 0) {
            ret[i] = bwd_worker(&jobs[i]);
            tid[i] = 0;
        }
    }
    for (int i = 0; i < n; ++i) {
        if (tid[i] && n > 1) pthread_join(tid[i], &ret[i]);
        if (ret[i]) rc = -2;
    }
    return rc;
}
