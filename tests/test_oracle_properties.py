"""Property-based pins of the fp64 oracle (oracle/gdn2_oracle.c), random shapes and inputs drawn by
hypothesis.  Each property follows from the update equation of page "NVIDIA представила Gated
DeltaNet-2 ...", section "Техническая схема", and none re-states the oracle's loop:

1. given q, k, alpha, b, w, the map (S0, v) -> (o, S_T) is linear;
2. o is linear in q alone, and q does not touch the state;
3. chains are independent: permuting batch elements and heads permutes the results;
4. cutting the sequence anywhere and resuming from the carried state changes nothing."""
import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle
from tests.test_oracle_pins import rand_inputs

SETTINGS = settings(max_examples=25, deadline=None, derandomize=True)
shapes = st.tuples(st.integers(1, 2), st.integers(0, 19), st.integers(1, 3), st.integers(1, 6), st.integers(1, 6))


def draw(seed, B, T, H, K, V):
    rng = np.random.default_rng(seed)
    return rng, rand_inputs(rng, B, max(T, 1), H, K, V, unit_k=False)


def run(q, k, v, alpha, b, w, S0):
    return oracle.recurrence(q, k, v, alpha, b, w, S0, threads=1)


def cut(T, x):
    return x[:, :T]


@SETTINGS
@given(shapes, st.integers(0, 2**32 - 1))
def test_linear_in_state_and_values(shape, seed):
    B, T, H, K, V = shape
    rng, (q, k, v, alpha, b, w, S0) = draw(seed, *shape)
    q, k, v, alpha, b, w = (cut(T, x) for x in (q, k, v, alpha, b, w))
    S1, v1 = rng.standard_normal(S0.shape), rng.standard_normal(v.shape)
    c = float(rng.uniform(-2, 2))
    oa, Sa = run(q, k, v, alpha, b, w, S0)
    ob, Sb = run(q, k, v1, alpha, b, w, S1)
    oc, Sc = run(q, k, c * v + v1, alpha, b, w, c * S0 + S1)
    scale = 1.0 + np.abs(oc).max(initial=0.0) + np.abs(Sc).max()
    assert np.abs(oc - (c * oa + ob)).max(initial=0.0) <= 1e-12 * scale
    assert np.abs(Sc - (c * Sa + Sb)).max() <= 1e-12 * scale


@SETTINGS
@given(shapes, st.integers(0, 2**32 - 1))
def test_linear_in_queries_only(shape, seed):
    B, T, H, K, V = shape
    rng, (q, k, v, alpha, b, w, S0) = draw(seed, *shape)
    q, k, v, alpha, b, w = (cut(T, x) for x in (q, k, v, alpha, b, w))
    q1 = rng.standard_normal(q.shape)
    c = float(rng.uniform(-2, 2))
    oa, Sa = run(q, k, v, alpha, b, w, S0)
    ob, Sb = run(q1, k, v, alpha, b, w, S0)
    oc, Sc = run(c * q + q1, k, v, alpha, b, w, S0)
    np.testing.assert_array_equal(Sa, Sb)       # the readout never feeds the state
    np.testing.assert_array_equal(Sa, Sc)
    assert np.abs(oc - (c * oa + ob)).max(initial=0.0) <= 1e-12 * (1.0 + np.abs(oc).max(initial=0.0))


@SETTINGS
@given(shapes, st.integers(0, 2**32 - 1))
def test_chains_are_independent(shape, seed):
    B, T, H, K, V = shape
    rng, (q, k, v, alpha, b, w, S0) = draw(seed, *shape)
    q, k, v, alpha, b, w = (cut(T, x) for x in (q, k, v, alpha, b, w))
    pb, ph = rng.permutation(B), rng.permutation(H)
    o, S = run(q, k, v, alpha, b, w, S0)
    perm = lambda x: x[pb][:, :, ph]
    op, Sp = run(*(perm(x) for x in (q, k, v, alpha, b, w)), S0[pb][:, ph])
    np.testing.assert_array_equal(op, perm(o))
    np.testing.assert_array_equal(Sp, S[pb][:, ph])


@SETTINGS
@given(shapes, st.integers(0, 2**32 - 1), st.floats(0.0, 1.0))
def test_cut_anywhere_and_resume(shape, seed, frac):
    B, T, H, K, V = shape
    _, (q, k, v, alpha, b, w, S0) = draw(seed, *shape)
    q, k, v, alpha, b, w = (cut(T, x) for x in (q, k, v, alpha, b, w))
    t = int(round(frac * T))
    o, S = run(q, k, v, alpha, b, w, S0)
    o1, S1 = run(*(x[:, :t] for x in (q, k, v, alpha, b, w)), S0)
    o2, S2 = run(*(x[:, t:] for x in (q, k, v, alpha, b, w)), S1)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=1), o, rtol=0, atol=1e-13 * (1 + np.abs(o).max(initial=0)))
    np.testing.assert_allclose(S2, S, rtol=0, atol=1e-13 * (1 + np.abs(S).max()))
