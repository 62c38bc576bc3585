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
