"""fp64 gradient of the Gated DeltaNet-2 recurrence -- TEST INFRASTRUCTURE ONLY.

Only ``tests/`` may import this module; the CUDA backward never calls it and
shares no code with it.

What it computes: for a scalar loss L of the recurrence's outputs, given the
loss's gradients at the outputs, dO_t = dL/do_t and dS_T = dL/dS_T, the
gradients of L with respect to every input of the recurrence (q, k, v, alpha,
b, w and S0).  The recurrence is the state-update equation of the page
"NVIDIA представила Gated DeltaNet-2 ...", section "Техническая схема":

    S_t = (I - k_t (b_t ⊙ k_t)^T) Diag(alpha_t) S_{t-1} + k_t (w_t ⊙ v_t)^T,   o_t = S_t^T q_t.

The same page says only that the backward pass needs gradients that account
for the per-channel gates (the scalar-gate shortcut does not carry over); it
prints no formulas.  So this is the chain rule applied to each step exactly as
the step is written, walked in reverse order, with every intermediate state
kept (no checkpointing, no chunking).  Per step, with Sbar_t = Diag(alpha_t)
S_{t-1}, e_t = b_t ⊙ k_t, u_t = w_t ⊙ v_t, delta_t = u_t - Sbar_t^T e_t and
S_t = Sbar_t + k_t delta_t^T, and G = dL/dS_t:

    o_t = S_t^T q_t          ->  dq_t = S_t dO_t,        G += q_t dO_t^T
    S_t = Sbar_t + k delta^T ->  dk_t += G delta_t,      ddelta = G^T k_t,   dSbar = G
    delta = u - Sbar^T e     ->  du_t = ddelta,          de_t = -Sbar_t ddelta,  dSbar -= e_t ddelta^T
    e = b ⊙ k, u = w ⊙ v     ->  db_t = k ⊙ de, dk_t += b ⊙ de, dw_t = v ⊙ du, dv_t = w ⊙ du
    Sbar = Diag(alpha) S     ->  dalpha_t = rowsum(dSbar ⊙ S_{t-1}),   dL/dS_{t-1} = Diag(alpha_t) dSbar

Pinned by ``tests/test_oracle_backward.py`` (finite differences of the
forward oracle, autograd of an independently written loop, the closed form of
the ungated, erase-free special case) and ``tests/test_oracle_backward_mutants.py``.
"""
from __future__ import annotations

import numpy as np


def chain_backward(q, k, v, alpha, b, w, S0, dO, dST):
    """Gradients of one chain.

    q, k, alpha, b: [T, K]; v, w, dO: [T, V]; S0, dST: [K, V] or None (zero).
    Returns (dq, dk, dv, dalpha, db, dw, dS0) in fp64, shaped like the inputs (dS0 [K, V]).
    """
    q, k, v, alpha, b, w, dO = (np.asarray(a, dtype=np.float64) for a in (q, k, v, alpha, b, w, dO))
    T, K = q.shape
    V = v.shape[1]
    states = np.empty((T + 1, K, V))     # states[t] = S_{t-1} in the page's 1-based count
    states[0] = 0.0 if S0 is None else np.asarray(S0, dtype=np.float64)
    deltas = np.empty((T, V))
    for t in range(T):
        e = b[t] * k[t]
        u = w[t] * v[t]
        Sbar = alpha[t][:, None] * states[t]
        deltas[t] = u - Sbar.T @ e
        states[t + 1] = Sbar + np.outer(k[t], deltas[t])

    dq, dk, dalpha, db = (np.zeros((T, K)) for _ in range(4))
    dv, dw = np.zeros((T, V)), np.zeros((T, V))
    G = np.zeros((K, V)) if dST is None else np.array(dST, dtype=np.float64)
    for t in range(T - 1, -1, -1):
        # o_t = S_t^T q_t
        dq[t] = states[t + 1] @ dO[t]
        G = G + np.outer(q[t], dO[t])
        # S_t = Sbar_t + k_t delta_t^T
        ddelta = G.T @ k[t]
        dk[t] = G @ deltas[t]
        # delta_t = u_t - Sbar_t^T e_t
        e = b[t] * k[t]
        Sbar = alpha[t][:, None] * states[t]
        du = ddelta
        de = -(Sbar @ ddelta)
        dSbar = G - np.outer(e, ddelta)
        # e_t = b_t ⊙ k_t, u_t = w_t ⊙ v_t
        db[t] = k[t] * de
        dk[t] = dk[t] + b[t] * de
        dw[t] = v[t] * du
        dv[t] = w[t] * du
        # Sbar_t = Diag(alpha_t) S_{t-1}
        dalpha[t] = np.sum(dSbar * states[t], axis=1)
        G = alpha[t][:, None] * dSbar
    return dq, dk, dv, dalpha, db, dw, G


def recurrence_backward(q, k, v, alpha, b, w, S0, dO, dST):
    """Gradients for [B, T, H, d] token arrays and [B, H, K, V] states (S0, dST may be None).

    Returns (dq, dk, dv, dalpha, db, dw, dS0) in fp64 with the inputs' layouts.
    """
    q = np.asarray(q)
    B, T, H, K = q.shape
    V = np.asarray(v).shape[-1]
    outs = [np.zeros((B, T, H, K)) for _ in range(2)] + [np.zeros((B, T, H, V))] + \
           [np.zeros((B, T, H, K)) for _ in range(2)] + [np.zeros((B, T, H, V)), np.zeros((B, H, K, V))]
    for bb in range(B):
        for h in range(H):
            g = chain_backward(q[bb, :, h], k[bb, :, h], v[bb, :, h], alpha[bb, :, h], b[bb, :, h],
                               w[bb, :, h], None if S0 is None else S0[bb, h], dO[bb, :, h],
                               None if dST is None else dST[bb, h])
            for i in range(6):
                outs[i][bb, :, h] = g[i]
            outs[6][bb, h] = g[6]
    return tuple(outs)
