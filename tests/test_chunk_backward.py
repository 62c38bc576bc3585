"""The step-wise backward oracle against an independent chunkwise (WY-form) restatement of the same
gradient (tests/chunk_backward.py): every chunk size, ragged tails, with and without S0 and dS_T."""
import numpy as np
import pytest

from oracle import backward as ob
from tests.chunk_backward import chunked_grads
from tests.test_oracle_pins import rand_inputs

NAMES = ("dq", "dk", "dv", "dalpha", "db", "dw", "dS0")


@pytest.mark.parametrize("T,C", [(1, 8), (7, 8), (16, 8), (37, 8), (37, 16), (70, 64), (130, 64)])
@pytest.mark.parametrize("with_state", [True, False])
def test_chunkwise_gradient_matches_stepwise(rng, T, C, with_state):
    K, V = 6, 5
    *tok, S0 = rand_inputs(rng, 1, T, 1, K, V, unit_k=False)
    q, k, v, alpha, b, w = (a[0, :, 0] for a in tok)
    S0 = S0[0, 0]
    dO = rng.standard_normal((T, V))
    dST = rng.standard_normal((K, V)) if with_state else None
    if not with_state:
        S0 = None
    ref = ob.chain_backward(q, k, v, alpha, b, w, S0, dO, dST)
    got = chunked_grads(q, k, v, alpha, b, w, S0, dO, dST, C)
    for n, r, x in zip(NAMES, ref, got):
        np.testing.assert_allclose(x, r, rtol=1e-9, atol=1e-11 * max(1.0, np.max(np.abs(r))), err_msg=n)


@pytest.mark.parametrize("log_alpha_range", [(-3.0, -0.05), (-16.0, -10.0)])
def test_framed_chunkwise_gradient(rng, log_alpha_range):
    """The midpoint-framed chunkwise gradient equals the step-wise oracle; with strong decay
    (alpha down to e^-16, a 64-token span of ~830 nats) the unframed factors overflow fp64 while the
    framed ones stay in range."""
    from tests.chunk_backward import chunked_grads_framed
    T, K, V, C = 150, 8, 6, 64
    *tok, S0 = rand_inputs(rng, 1, T, 1, K, V, unit_k=False)
    q, k, v, _, b, w = (a[0, :, 0] for a in tok)
    alpha = np.exp(rng.uniform(*log_alpha_range, size=(T, K)))
    S0 = S0[0, 0]
    dO, dST = rng.standard_normal((T, V)), rng.standard_normal((K, V))
    ref = ob.chain_backward(q, k, v, alpha, b, w, S0, dO, dST)
    got = chunked_grads_framed(q, k, v, alpha, b, w, S0, dO, dST, C)
    for n, r, x in zip(NAMES, ref, got):
        # relative to the tensor's largest entry: the decay sums cancel terms of the gradients' size
        assert np.all(np.isfinite(x)), n
        assert np.max(np.abs(x - r)) <= 1e-8 * np.max(np.abs(r)), n
    if log_alpha_range[0] < -10:
        with np.errstate(over="ignore", invalid="ignore"):
            plain = chunked_grads(q, k, v, alpha, b, w, S0, dO, dST, C)
        assert not all(np.all(np.isfinite(x)) for x in plain)
