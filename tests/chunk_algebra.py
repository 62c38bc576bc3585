"""Test-only fp64 chunkwise restatement of the gated delta-rule recurrence.

It restates the sequential update (page "NVIDIA представила Gated DeltaNet-2 ...",
section "Техническая схема") chunk by chunk, in the WY/UT form the same page names
for its chunkwise kernels (chunk size C = 64 there; any C here).  It is used to pin
the oracle (chunk-size invariance: every C must give the sequential result) and to
document the algebra the GPU kernels implement.

Per chunk of L tokens with incoming state S (K x V), positions r, i in 0..L-1:

    g_r  = sum_{j<=r} log alpha_j           (per key channel)
    e_r  = b_r ⊙ k_r,  u_r = w_r ⊙ v_r
    A_ri = sum_c e_rc k_ic exp(g_rc - g_ic)  for i < r   (strictly lower)
    P_ri = sum_c q_rc k_ic exp(g_rc - g_ic)  for i <= r
    T    = (I + A)^-1
    W    = T (exp(g) ⊙ E),   U~ = T U
    Delta = U~ - W S
    O    = (exp(g) ⊙ Q) S + P Delta
    S'   = Diag(exp(g_{L-1})) S + ((exp(g_{L-1} - g) ⊙ K))^T Delta

This follows from writing one step as S_t = D_t S_{t-1} + k_t delta_t^T with
delta_t = u_t - S_{t-1}^T (alpha_t ⊙ e_t).
"""
import numpy as np


def chunk_step(q, k, v, alpha, b, w, S):
    """One chunk: token arrays [L, d] (fp64), S [K, V].  Returns (O [L, V], S')."""
    g = np.cumsum(np.log(alpha), axis=0)                 # [L, K]
    e = b * k
    u = w * v
    L = q.shape[0]
    diff = g[:, None, :] - g[None, :, :]                 # [r, i, c] = g_rc - g_ic
    lower = np.tril(np.ones((L, L), dtype=bool), -1)
    lower_eq = np.tril(np.ones((L, L), dtype=bool), 0)
    dec = np.exp(np.where(lower_eq[:, :, None], diff, -np.inf))
    A = np.einsum("rc,ic,ric->ri", e, k, dec) * lower
    P = np.einsum("rc,ic,ric->ri", q, k, dec) * lower_eq
    Tm = np.linalg.inv(np.eye(L) + A)
    gam = np.exp(g)
    W = Tm @ (gam * e)
    Ut = Tm @ u
    Delta = Ut - W @ S
    O = (gam * q) @ S + P @ Delta
    Khat = np.exp(g[-1][None, :] - g) * k
    S_new = gam[-1][:, None] * S + Khat.T @ Delta
    return O, S_new, Tm, A


def chunked(q, k, v, alpha, b, w, S0, C):
    """Whole sequence of one chain ([T, d] arrays) in chunks of C (last one ragged)."""
    T = q.shape[0]
    K, V = k.shape[1], v.shape[1]
    S = np.zeros((K, V)) if S0 is None else np.array(S0, dtype=np.float64)
    O = np.zeros((T, V))
    for t0 in range(0, T, C):
        t1 = min(T, t0 + C)
        O[t0:t1], S, _, _ = chunk_step(q[t0:t1], k[t0:t1], v[t0:t1], alpha[t0:t1], b[t0:t1], w[t0:t1], S)
    return O, S
