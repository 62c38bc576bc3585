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


@pytest.mark.parametrize("wl_name", ["prefill_1p3b", "prefill_slow_decay"])
def test_rounded_chunkwise_gradient_accuracy(wl_name):
    """What a tensor-core chunkwise backward can reach: the framed WY gradient with every product's
    operands rounded to tf32 or bf16 (fp32 accumulation and state), on the bench workloads' value
    distributions (d = 128, T = 512), against the fp64 step-wise oracle.  dq, dk, dv, db, dw, dS0 and
    the gradient of log alpha stay within 2e-2 (bf16 operands) and 2e-3 (tf32); neither reaches the
    1e-4 of the fp32 passes.  The gradient of alpha itself is d log alpha / alpha: at the bench
    workload's smallest decays (alpha ~ 3e-3) that division lifts the absolute error of d log alpha
    above 2e-2 of max |d alpha| with bf16 operands, so such a kernel would hand out d log alpha (what
    a decay produced from a logit needs) or form d alpha in fp32.  Unrounded fp32 operands check the
    emulation itself."""
    import synth
    from tests.chunk_backward import chunked_grads_rounded, tf32
    from tests.kernel_numerics import bf16
    wl0 = synth.WORKLOADS[wl_name]
    wl = synth.Workload(wl0.name, 1, 2, 512, wl0.K, wl0.V, wl0.dtype, wl0.alpha_mu, gates=wl0.gates,
                        seed=wl0.seed, alpha_scale=wl0.alpha_scale)
    x = synth.as_f64(synth.make_inputs(wl, chains=[(0, 1)]))
    dO, dST = synth.make_output_grads(wl, chains=[(0, 1)])
    args = [x[n][0] for n in ("q", "k", "v", "alpha", "b", "w")]
    alpha = args[3]
    dO, dST = dO[0].astype(np.float64), dST[0].astype(np.float64)
    ref = ob.chain_backward(*args, None, dO, dST)
    rel = lambda a, r: np.max(np.abs(a - r)) / np.max(np.abs(r))
    worst, dalpha = {}, {}
    for name, rnd in (("fp32", lambda a: np.asarray(a, dtype=np.float32).astype(np.float64)), ("tf32", tf32),
                      ("bf16", bf16)):
        got = chunked_grads_rounded(*args, None, dO, dST, 64, rnd)
        errs = [rel(g, r) for i, (g, r) in enumerate(zip(got, ref)) if i != 3]
        worst[name] = max(errs + [rel(got[3] * alpha, ref[3] * alpha)])
        dalpha[name] = rel(got[3], ref[3])
    assert worst["fp32"] <= 1e-5 and dalpha["fp32"] <= 1e-4, (worst, dalpha)
    assert worst["tf32"] <= 2e-3, worst
    assert worst["bf16"] <= 2e-2, worst
    if wl_name == "prefill_1p3b":
        assert dalpha["bf16"] > 2e-2, dalpha
