"""Pins of the fp64 oracle to facts fixed by the pages and by the mathematics.

The oracle (oracle/gdn2_oracle.c) evaluates the GDN-2 update of page
"NVIDIA представила Gated DeltaNet-2 ...", section "Техническая схема":
S_t = (I - k_t (b_t ⊙ k_t)^T) Diag(alpha_t) S_{t-1} + k_t (w_t ⊙ v_t)^T, o_t = S_t^T q_t.
No page prints a worked numeric example, so the pins are:

1. brute force: the d_k x d_k matrices M_t = (I - k_t e_t^T) D_t multiplied out,
   S_t = M_t...M_1 S_0 + sum_i M_t...M_{i+1} k_i u_i^T (T <= 8, d_k != d_v);
2. collapsed gates (page "NVIDIA улучшила память LLM ...", the quoted sentence
   on special cases; and the GDN-2 page's architecture paragraph): b = w = beta 1
   gives KDA, S = (I - beta k k^T) Diag(alpha) S + beta k v^T; a scalar alpha on
   top gives Gated DeltaNet, S = alpha (I - beta k k^T) S + beta k v^T;
3. erase-then-write: with b = 1 and |k_t| = 1, k_t^T S_t = (w_t ⊙ v_t)^T for any alpha;
4. frozen state: alpha = 1, b = w = 0 gives S_t = S_0;
5. pure decay (b = w = 0) and no-erase (b = 0) closed forms;
6. chunk-size invariance of an independent chunkwise (WY/UT) restatement;
7. split-resume and T = 1 prefill == one decode step.

tests/test_oracle_mutants.py plants single mistakes in copies of the oracle and
checks that these pins catch each one.
"""
import numpy as np
import pytest

import oracle
from tests.chunk_algebra import chunked, chunk_step


def rand_inputs(rng, B, T, H, K, V, unit_k=True, s0=True):
    q = rng.standard_normal((B, T, H, K))
    k = rng.standard_normal((B, T, H, K))
    if unit_k:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, V))
    alpha = np.exp(-np.logaddexp(0, rng.standard_normal((B, T, H, K))))
    b = 1 / (1 + np.exp(-rng.standard_normal((B, T, H, K))))
    w = 1 / (1 + np.exp(-rng.standard_normal((B, T, H, V))))
    S0 = rng.standard_normal((B, H, K, V)) * 0.3 if s0 else None
    return q, k, v, alpha, b, w, S0


def brute_force(q, k, v, alpha, b, w, S0):
    """Single chain, [T, d] arrays: dense products, unrolled sum (independent of the oracle loop)."""
    T, K = k.shape
    V = v.shape[1]
    M = [(np.eye(K) - np.outer(k[t], b[t] * k[t])) @ np.diag(alpha[t]) for t in range(T)]
    S0 = np.zeros((K, V)) if S0 is None else S0
    o = np.zeros((T, V))
    St = None
    for t in range(T):
        prod = np.eye(K)
        for j in range(t, -1, -1):
            prod = prod @ M[j]
        St = prod @ S0
        for i in range(t + 1):
            tail = np.eye(K)
            for j in range(t, i, -1):
                tail = tail @ M[j]
            St = St + tail @ np.outer(k[i], w[i] * v[i])
        o[t] = St.T @ q[t]
    return o, St


@pytest.mark.parametrize("T,K,V", [(1, 4, 3), (2, 3, 5), (5, 6, 4), (8, 5, 7)])
def test_brute_force_products(rng, T, K, V):
    B, H = 2, 3
    q, k, v, alpha, b, w, S0 = rand_inputs(rng, B, T, H, K, V, unit_k=False)
    o, ST = oracle.recurrence(q, k, v, alpha, b, w, S0, threads=2)
    for bb in range(B):
        for hh in range(H):
            ob, Sb = brute_force(q[bb, :, hh], k[bb, :, hh], v[bb, :, hh], alpha[bb, :, hh],
                                 b[bb, :, hh], w[bb, :, hh], S0[bb, hh])
            np.testing.assert_allclose(o[bb, :, hh], ob, rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(ST[bb, hh], Sb, rtol=1e-12, atol=1e-12)


def kda_restatement(q, k, v, alpha, beta, S0):
    """KDA: one scalar beta_t per token for both gates; channel-wise decay."""
    T, K = k.shape
    S = S0.copy()
    o = np.zeros((T, v.shape[1]))
    for t in range(T):
        S = (np.eye(K) - beta[t] * np.outer(k[t], k[t])) @ (alpha[t][:, None] * S) + beta[t] * np.outer(k[t], v[t])
        o[t] = S.T @ q[t]
    return o, S


def gdn_restatement(q, k, v, a, beta, S0):
    """Gated DeltaNet: scalar decay a_t and scalar beta_t per token."""
    T, K = k.shape
    S = S0.copy()
    o = np.zeros((T, v.shape[1]))
    for t in range(T):
        S = a[t] * ((np.eye(K) - beta[t] * np.outer(k[t], k[t])) @ S) + beta[t] * np.outer(k[t], v[t])
        o[t] = S.T @ q[t]
    return o, S


def test_kda_special_case(rng):
    B, T, H, K, V = 2, 40, 2, 8, 6
    q, k, v, alpha, _, _, S0 = rand_inputs(rng, B, T, H, K, V)
    beta = 1 / (1 + np.exp(-rng.standard_normal((B, T, H))))
    b = np.repeat(beta[..., None], K, axis=-1)
    w = np.repeat(beta[..., None], V, axis=-1)
    o, ST = oracle.recurrence(q, k, v, alpha, b, w, S0)
    for bb in range(B):
        for hh in range(H):
            ok, Sk = kda_restatement(q[bb, :, hh], k[bb, :, hh], v[bb, :, hh], alpha[bb, :, hh], beta[bb, :, hh],
                                     S0[bb, hh])
            np.testing.assert_allclose(o[bb, :, hh], ok, rtol=1e-11, atol=1e-12)
            np.testing.assert_allclose(ST[bb, hh], Sk, rtol=1e-11, atol=1e-12)


def test_gated_deltanet_special_case(rng):
    B, T, H, K, V = 2, 40, 2, 8, 6
    q, k, v, _, _, _, S0 = rand_inputs(rng, B, T, H, K, V)
    beta = 1 / (1 + np.exp(-rng.standard_normal((B, T, H))))
    a = np.exp(-np.logaddexp(0, rng.standard_normal((B, T, H)) + 1.0))
    alpha = np.repeat(a[..., None], K, axis=-1)
    b = np.repeat(beta[..., None], K, axis=-1)
    w = np.repeat(beta[..., None], V, axis=-1)
    o, ST = oracle.recurrence(q, k, v, alpha, b, w, S0)
    for bb in range(B):
        for hh in range(H):
            og, Sg = gdn_restatement(q[bb, :, hh], k[bb, :, hh], v[bb, :, hh], a[bb, :, hh], beta[bb, :, hh],
                                     S0[bb, hh])
            np.testing.assert_allclose(o[bb, :, hh], og, rtol=1e-11, atol=1e-12)
            np.testing.assert_allclose(ST[bb, hh], Sg, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("T", [1, 2, 7, 50])
def test_erase_then_write(rng, T):
    B, H, K, V = 2, 2, 8, 5
    q, k, v, alpha, _, w, S0 = rand_inputs(rng, B, T, H, K, V)
    b = np.ones_like(k)
    _, ST = oracle.recurrence(q, k, v, alpha, b, w, S0)
    for bb in range(B):
        for hh in range(H):
            kt = k[bb, -1, hh]
            np.testing.assert_allclose(kt @ ST[bb, hh], w[bb, -1, hh] * v[bb, -1, hh], rtol=1e-12, atol=1e-13)


def test_erase_then_write_every_step(rng):
    """Resume one token at a time and check the identity after every step."""
    B, H, K, V, T = 1, 3, 6, 4, 12
    q, k, v, alpha, _, w, S = rand_inputs(rng, B, T, H, K, V)
    b = np.ones_like(k)
    for t in range(T):
        sl = slice(t, t + 1)
        _, S = oracle.recurrence(q[:, sl], k[:, sl], v[:, sl], alpha[:, sl], b[:, sl], w[:, sl], S)
        for hh in range(H):
            np.testing.assert_allclose(k[0, t, hh] @ S[0, hh], w[0, t, hh] * v[0, t, hh], rtol=1e-12, atol=1e-13)


def test_frozen_state(rng):
    B, T, H, K, V = 2, 30, 2, 7, 5
    q, k, v, _, _, _, S0 = rand_inputs(rng, B, T, H, K, V)
    ones = np.ones_like(k)
    zk, zv = np.zeros_like(k), np.zeros((B, T, H, V))
    o, ST = oracle.recurrence(q, k, v, ones, zk, zv, S0)
    np.testing.assert_array_equal(ST, S0)
    np.testing.assert_allclose(o, np.einsum("bthc,bhcv->bthv", q, S0), rtol=1e-13, atol=1e-14)


def test_pure_decay_closed_form(rng):
    B, T, H, K, V = 2, 30, 2, 7, 5
    q, k, v, alpha, _, _, S0 = rand_inputs(rng, B, T, H, K, V)
    o, ST = oracle.recurrence(q, k, v, alpha, np.zeros_like(k), np.zeros((B, T, H, V)), S0)
    gam = np.cumprod(alpha, axis=1)                      # [B, T, H, K]
    np.testing.assert_allclose(ST, gam[:, -1][..., None] * S0, rtol=1e-12)
    o_ref = np.einsum("bthc,bhcv->bthv", q * gam, S0)
    np.testing.assert_allclose(o, o_ref, rtol=1e-11, atol=1e-14)


def test_no_erase_closed_form(rng):
    B, T, H, K, V = 2, 25, 2, 6, 5
    q, k, v, alpha, _, w, S0 = rand_inputs(rng, B, T, H, K, V)
    o, ST = oracle.recurrence(q, k, v, alpha, np.zeros_like(k), w, S0)
    gam = np.cumprod(alpha, axis=1)
    u = w * v
    for bb in range(B):
        for hh in range(H):
            g = gam[bb, :, hh]
            for t in (0, T // 2, T - 1):
                St = g[t][:, None] * S0[bb, hh]
                for i in range(t + 1):
                    St = St + np.outer((g[t] / g[i]) * k[bb, i, hh], u[bb, i, hh])
                np.testing.assert_allclose(o[bb, t, hh], St.T @ q[bb, t, hh], rtol=1e-10, atol=1e-13)
                if t == T - 1:
                    np.testing.assert_allclose(ST[bb, hh], St, rtol=1e-10, atol=1e-13)


@pytest.mark.parametrize("C", [1, 8, 16, 64])
def test_chunk_size_invariance(rng, C):
    B, T, H, K, V = 1, 150, 2, 16, 12            # ragged last chunk for C in {8, 16, 64}
    q, k, v, alpha, b, w, S0 = rand_inputs(rng, B, T, H, K, V)
    o, ST = oracle.recurrence(q, k, v, alpha, b, w, S0)
    for hh in range(H):
        oc, Sc = chunked(q[0, :, hh], k[0, :, hh], v[0, :, hh], alpha[0, :, hh], b[0, :, hh], w[0, :, hh],
                         S0[0, hh], C)
        np.testing.assert_allclose(oc, o[0, :, hh], rtol=1e-9, atol=1e-11)
        np.testing.assert_allclose(Sc, ST[0, hh], rtol=1e-9, atol=1e-11)


def test_ut_transform_inverse(rng):
    """The chunk's T = (I + A)^-1 is unit lower-triangular and inverts I + A."""
    L, K, V = 64, 16, 8
    q, k, v, alpha, b, w, S0 = rand_inputs(rng, 1, L, 1, K, V)
    _, _, Tm, A = chunk_step(q[0, :, 0], k[0, :, 0], v[0, :, 0], alpha[0, :, 0], b[0, :, 0], w[0, :, 0], S0[0, 0])
    np.testing.assert_allclose(Tm @ (np.eye(L) + A), np.eye(L), atol=1e-10)
    np.testing.assert_allclose(np.triu(Tm, 1), 0, atol=0)
    np.testing.assert_allclose(np.diag(Tm), 1, atol=1e-12)


def test_split_resume(rng):
    B, T, H, K, V = 2, 37, 2, 8, 6
    q, k, v, alpha, b, w, S0 = rand_inputs(rng, B, T, H, K, V)
    o, ST = oracle.recurrence(q, k, v, alpha, b, w, S0)
    cut = 20
    a = lambda x, s: x[:, s]
    o1, S1 = oracle.recurrence(*(a(x, slice(0, cut)) for x in (q, k, v, alpha, b, w)), S0)
    o2, S2 = oracle.recurrence(*(a(x, slice(cut, T)) for x in (q, k, v, alpha, b, w)), S1)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=1), o, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(S2, ST, rtol=1e-13, atol=1e-15)


def test_prefill_T1_equals_decode_step(rng):
    B, H, K, V = 3, 2, 8, 6
    q, k, v, alpha, b, w, S0 = rand_inputs(rng, B, 1, H, K, V)
    o, ST = oracle.recurrence(q, k, v, alpha, b, w, S0)
    S = S0.copy()
    od = oracle.decode_step(q[:, 0], k[:, 0], v[:, 0], alpha[:, 0], b[:, 0], w[:, 0], S)
    np.testing.assert_array_equal(od, o[:, 0])
    np.testing.assert_array_equal(S, ST)


def test_zero_state_default_and_empty(rng):
    B, T, H, K, V = 1, 5, 1, 4, 3
    q, k, v, alpha, b, w, _ = rand_inputs(rng, B, T, H, K, V, s0=False)
    o1, S1 = oracle.recurrence(q, k, v, alpha, b, w, None)
    o2, S2 = oracle.recurrence(q, k, v, alpha, b, w, np.zeros((B, H, K, V)))
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(S1, S2)
    # T = 0: the state passes through unchanged
    S0 = np.ones((B, H, K, V))
    e = lambda d: np.zeros((B, 0, H, d))
    o0, S0out = oracle.recurrence(e(K), e(K), e(V), e(K), e(K), e(V), S0)
    assert o0.shape == (B, 0, H, V)
    np.testing.assert_array_equal(S0out, S0)


def test_threads_do_not_change_results(rng):
    q, k, v, alpha, b, w, S0 = rand_inputs(rng, 3, 20, 5, 8, 6)
    o1, S1 = oracle.recurrence(q, k, v, alpha, b, w, S0, threads=1)
    o4, S4 = oracle.recurrence(q, k, v, alpha, b, w, S0, threads=4)
    np.testing.assert_array_equal(o1, o4)
    np.testing.assert_array_equal(S1, S4)
