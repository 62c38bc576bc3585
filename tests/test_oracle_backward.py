"""Pins of the fp64 backward oracle (oracle/backward.py) to facts other than itself.

The oracle gives the gradient of a scalar loss L through the recurrence of page
"NVIDIA представила Gated DeltaNet-2 ...", section "Техническая схема".  Taking
L = sum_t dO_t . o_t + sum dS_T ⊙ S_T makes dO and dS_T the loss's gradients
at the outputs.  Pins:

1. finite differences: central differences of L evaluated with the FORWARD
   oracle (oracle/gdn2_oracle.c, itself pinned), along random directions, one
   input at a time; the error of a central difference is O(eps^2);
2. autograd: torch's reverse mode (fp64, CPU) through a step loop written here
   from the update equation;
3. closed form: alpha = 1 and b = 0 make the recurrence plain linear attention,
   o_t = S_0^T q_t + sum_{i<=t} (k_i . q_t) u_i, whose gradients are textbook
   sums over the causal mask.
The C version of the same gradient (oracle/gdn2_oracle.c, gdn2_oracle_backward) passes the
finite-difference pin and agrees with the numpy one to rounding.
"""
import numpy as np
import pytest

import oracle
from oracle import backward as ob
from tests.test_oracle_pins import rand_inputs

NAMES = ("q", "k", "v", "alpha", "b", "w", "S0")


def loss(x, dO, dST):
    o, ST = oracle.recurrence(*(x[n] for n in NAMES), threads=1)
    return float(np.sum(dO * o) + np.sum(dST * ST))


def problem(rng, B, T, H, K, V):
    q, k, v, alpha, b, w, S0 = rand_inputs(rng, B, T, H, K, V, unit_k=False)
    x = dict(zip(NAMES, (q, k, v, alpha, b, w, S0)))
    dO = rng.standard_normal((B, T, H, V))
    dST = rng.standard_normal((B, H, K, V))
    return x, dO, dST


def directional_errors(rng, x, dO, dST, grads, eps=1e-5):
    """|central difference - <grad, d>| / scale for a random direction d per input."""
    errs = {}
    for name, g in zip(NAMES, grads):
        d = rng.standard_normal(x[name].shape)
        xp = dict(x)
        xm = dict(x)
        xp[name] = x[name] + eps * d
        xm[name] = x[name] - eps * d
        fd = (loss(xp, dO, dST) - loss(xm, dO, dST)) / (2 * eps)
        an = float(np.sum(g * d))
        errs[name] = abs(fd - an) / max(1.0, abs(an))
    return errs


IMPLS = {"numpy": ob.recurrence_backward, "c": oracle.recurrence_backward_c}


@pytest.mark.parametrize("impl", sorted(IMPLS))
@pytest.mark.parametrize("T,K,V", [(1, 3, 2), (4, 3, 5), (9, 5, 4)])
def test_finite_differences(rng, T, K, V, impl):
    x, dO, dST = problem(rng, 1, T, 2, K, V)
    grads = IMPLS[impl](*(x[n] for n in NAMES), dO, dST)
    errs = directional_errors(rng, x, dO, dST, grads)
    assert max(errs.values()) < 1e-8, errs


def test_finite_differences_without_state_gradient(rng):
    """dS_T = 0 and S_0 = 0 (the defaults): only the outputs o carry gradient."""
    x, dO, _ = problem(rng, 1, 6, 1, 4, 3)
    x["S0"] = np.zeros_like(x["S0"])
    zero = np.zeros((1, 1, 4, 3))
    grads = ob.recurrence_backward(*(x[n] for n in NAMES[:-1]), None, dO, None)
    errs = directional_errors(rng, x, dO, zero, grads)
    assert max(errs.values()) < 1e-8, errs


def test_autograd(rng):
    torch = pytest.importorskip("torch")
    B, T, H, K, V = 1, 12, 2, 6, 5
    x, dO, dST = problem(rng, B, T, H, K, V)
    tx = {n: torch.tensor(x[n], dtype=torch.float64, requires_grad=True) for n in NAMES}
    L = 0.0
    for h in range(H):
        S = tx["S0"][0, h]
        for t in range(T):
            kt, qt = tx["k"][0, t, h], tx["q"][0, t, h]
            et = tx["b"][0, t, h] * kt
            ut = tx["w"][0, t, h] * tx["v"][0, t, h]
            M = torch.eye(K, dtype=torch.float64) - torch.outer(kt, et)
            S = M @ (tx["alpha"][0, t, h][:, None] * S) + torch.outer(kt, ut)
            L = L + torch.dot(torch.tensor(dO[0, t, h]), S.T @ qt)
        L = L + torch.sum(torch.tensor(dST[0, h]) * S)
    L.backward()
    grads = ob.recurrence_backward(*(x[n] for n in NAMES), dO, dST)
    for n, g in zip(NAMES, grads):
        np.testing.assert_allclose(g, tx[n].grad.numpy(), rtol=1e-10, atol=1e-12, err_msg=n)


def test_linear_attention_closed_form(rng):
    """alpha = 1, b = 0: o_t = S0^T q_t + sum_{i<=t} (q_t . k_i) u_i and S_T = S0 + sum_i k_i u_i^T."""
    T, K, V = 7, 4, 3
    x, dO, dST = problem(rng, 1, T, 1, K, V)
    x["alpha"] = np.ones_like(x["alpha"])
    x["b"] = np.zeros_like(x["b"])
    g = ob.recurrence_backward(*(x[n] for n in NAMES), dO, dST)
    q, k, v, w, S0 = (x[n][0, :, 0] if n != "S0" else x[n][0, 0] for n in ("q", "k", "v", "w", "S0"))
    do, dst = dO[0, :, 0], dST[0, 0]
    u = w * v
    mask = np.tril(np.ones((T, T)))                 # mask[t, i] = 1 for i <= t
    qk = (q @ k.T) * mask                            # (q_t . k_i) for i <= t
    du_ref = qk.T @ do + k @ dst                     # du_i = sum_{t>=i} (q_t.k_i) dO_t + dS_T^T k_i
    dk_ref = ((do @ u.T) * mask).T @ q + u @ dst.T   # dk_i = sum_{t>=i} (dO_t.u_i) q_t + dS_T u_i
    dq_ref = ((do @ u.T) * mask) @ k + do @ S0.T     # dq_t = sum_{i<=t} (dO_t.u_i) k_i + S0 dO_t
    dS0_ref = q.T @ do + dst
    np.testing.assert_allclose(g[0][0, :, 0], dq_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g[1][0, :, 0], dk_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g[2][0, :, 0], w * du_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g[5][0, :, 0], v * du_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g[6][0, 0], dS0_ref, rtol=1e-12, atol=1e-12)


def test_empty_sequence(rng):
    """T = 0: S_T = S_0, so dS0 = dS_T and there are no token gradients."""
    x, dO, dST = problem(rng, 1, 1, 1, 3, 2)
    g = ob.chain_backward(*(np.zeros((0, 3)) if n in ("q", "k", "alpha", "b") else np.zeros((0, 2))
                            for n in NAMES[:-1]), x["S0"][0, 0], np.zeros((0, 2)), dST[0, 0])
    assert all(a.shape[0] == 0 for a in g[:6])
    np.testing.assert_array_equal(g[6], dST[0, 0])


@pytest.mark.parametrize("B,T,H,K,V", [(1, 0, 2, 3, 2), (1, 1, 1, 4, 3), (2, 37, 3, 6, 5), (1, 70, 2, 16, 8)])
@pytest.mark.parametrize("with_state", [True, False])
def test_c_oracle_matches_numpy(rng, B, T, H, K, V, with_state):
    """The C backward (oracle/gdn2_oracle.c) and the numpy one take the same steps in the same order:
    they agree to rounding, threads or not."""
    x, dO, dST = problem(rng, B, max(T, 1), H, K, V)
    if T == 0:
        x = {n: (a if n == "S0" else a[:, :0]) for n, a in x.items()}
        dO = dO[:, :0]
    if not with_state:
        x["S0"] = None
        dST = None
    ref = ob.recurrence_backward(*(x[n] for n in NAMES), dO, dST)
    for threads in (1, 3):
        got = oracle.recurrence_backward_c(*(x[n] for n in NAMES), dO, dST, threads=threads)
        for n, r, g in zip(("dq", "dk", "dv", "dalpha", "db", "dw", "dS0"), ref, got):
            np.testing.assert_allclose(g, r, rtol=1e-12, atol=1e-13 * max(1.0, np.max(np.abs(r), initial=0.0)),
                                       err_msg=n)


@pytest.mark.parametrize("impl", sorted(IMPLS))
def test_gradients_linear_in_output_gradients(rng, impl):
    """The gradient is a linear map of (dO, dS_T): grads(a*g1 + g2) = a*grads(g1) + grads(g2)."""
    x, dO1, dST1 = problem(rng, 1, 11, 2, 5, 4)
    _, dO2, dST2 = problem(rng, 1, 11, 2, 5, 4)
    f = lambda dO, dST: IMPLS[impl](*(x[n] for n in NAMES), dO, dST)
    a = 1.7
    lhs = f(a * dO1 + dO2, a * dST1 + dST2)
    g1, g2 = f(dO1, dST1), f(dO2, dST2)
    for n, l, r1, r2 in zip(NAMES, lhs, g1, g2):
        np.testing.assert_allclose(l, a * r1 + r2, rtol=1e-10, atol=1e-12, err_msg=n)


@pytest.mark.parametrize("impl", sorted(IMPLS))
@pytest.mark.parametrize("T,K,V", [(1, 3, 2), (9, 5, 4), (30, 4, 6)])
def test_euler_identities(rng, impl, T, K, V):
    """Homogeneity pins.  L = sum dO.o + sum dS_T⊙S_T is linear in (S0, v) jointly and, through the
    readout alone, in q; by Euler's theorem for degree-1 functions
        <dS0, S0> + <dv, v> = <dS0, S0> + <dw, w> = L      and      <dq, q> = sum dO.o,
    and dq does not depend on dS_T (q never feeds the state)."""
    x, dO, dST = problem(rng, 1, T, 2, K, V)
    g = IMPLS[impl](*(x[n] for n in NAMES), dO, dST)
    o, ST = oracle.recurrence(*(x[n] for n in NAMES), threads=1)
    L_o, L = float(np.sum(dO * o)), float(np.sum(dO * o) + np.sum(dST * ST))
    for grad, name in ((g[2], "v"), (g[5], "w")):   # u = w ⊙ v is linear in each of them
        euler = float(np.sum(g[6] * x["S0"]) + np.sum(grad * x[name]))
        assert abs(euler - L) <= 1e-11 * (1 + abs(L)), (name, euler, L)
    assert abs(float(np.sum(g[0] * x["q"])) - L_o) <= 1e-11 * (1 + abs(L_o))
    g0 = IMPLS[impl](*(x[n] for n in NAMES), dO, np.zeros_like(dST))
    np.testing.assert_allclose(g0[0], g[0], rtol=1e-13, atol=1e-14)
