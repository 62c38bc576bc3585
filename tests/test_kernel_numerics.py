"""The precision of the tensor-core prefill's design, checked on the CPU: the emulation of its
number formats (tests/kernel_numerics.py) against the fp64 oracle on chains of the workloads,
within the 2e-2 bar of bf16 tokens.  (The GPU parity tests measure the kernel itself.)"""
import numpy as np
import pytest

import oracle
import synth
from tests.kernel_numerics import emulate_chain


def rel(x, y):
    return np.max(np.abs(x - y)) / np.max(np.abs(y))


@pytest.mark.parametrize("name,T", [("prefill_1p3b", 1024), ("prefill_slow_decay", 1024),
                                    ("prefill_kda", 512), ("prefill_gdn", 512), ("prefill_long", 2048)])
def test_emulated_kernel_precision(name, T):
    wl0 = synth.WORKLOADS[name]
    wl = synth.Workload(wl0.name, wl0.B, wl0.H, T, wl0.K, wl0.V, wl0.dtype, wl0.alpha_mu, gates=wl0.gates,
                        s0_std=wl0.s0_std, seed=wl0.seed, alpha_scale=wl0.alpha_scale)
    chain = [(0, 3)]
    x = synth.make_inputs(wl, chains=chain)
    S0 = synth.make_state(wl, chains=chain)
    c = {k: a[0].astype(np.float64) for k, a in x.items()}
    s0 = None if S0 is None else S0[0].astype(np.float64)
    o_ref, S_ref = oracle.chain_recurrence(*(x[k].astype(np.float64) for k in ("q", "k", "v", "alpha", "b", "w")),
                                           None if S0 is None else S0.astype(np.float64))
    o, S = emulate_chain(c["q"], c["k"], c["v"], c["alpha"], c["b"], c["w"], s0)
    assert rel(o, o_ref[0]) <= 2e-2 and rel(S, S_ref[0]) <= 2e-2, (rel(o, o_ref[0]), rel(S, S_ref[0]))


def test_wide_span_chunks(rng):
    """Decay spans past 120 nats per chunk take the wide-span branch: still within the bar."""
    T, K, V = 256, 128, 128
    wl = synth.Workload("ws", 1, 1, T, K, V, "bf16", 1.0, seed=31)
    x = synth.make_inputs(wl, chains=[(0, 0)])
    c = {k: a[0].astype(np.float64) for k, a in x.items()}
    c["alpha"] = np.asarray(np.exp(rng.uniform(-6.0, -1.0, size=(T, K))), dtype=np.float32).astype(np.float64)
    o_ref, S_ref = oracle.chain_recurrence(*(c[k][None] for k in ("q", "k", "v", "alpha", "b", "w")))
    o, S = emulate_chain(c["q"], c["k"], c["v"], c["alpha"], c["b"], c["w"], None)
    assert rel(o, o_ref[0]) <= 2e-2 and rel(S, S_ref[0]) <= 2e-2, (rel(o, o_ref[0]), rel(S, S_ref[0]))


def test_combined_frame_factors_fail_on_long_context():
    """Why the two frame factors between chunks are applied in turn: taken as one factor, 2 to the sum
    of their exponents flushes to zero on the channels whose chunk spans reach the long workload's
    typical ~150 log2, and the state those channels carry into the next chunk is lost (o errors of
    0.13-0.18 here against 0.006-0.01 for the kernel's order)."""
    wl0 = synth.WORKLOADS["prefill_long"]
    wl = synth.Workload(wl0.name, wl0.B, wl0.H, 2048, wl0.K, wl0.V, wl0.dtype, wl0.alpha_mu, s0_std=wl0.s0_std,
                        seed=wl0.seed)
    errs = []
    for h in range(4):
        x = synth.make_inputs(wl, chains=[(0, h)])
        S0 = synth.make_state(wl, chains=[(0, h)])
        c = {k: a[0].astype(np.float64) for k, a in x.items()}
        o_ref, _ = oracle.chain_recurrence(*(x[k].astype(np.float64) for k in ("q", "k", "v", "alpha", "b", "w")),
                                           S0.astype(np.float64))
        args = (c["q"], c["k"], c["v"], c["alpha"], c["b"], c["w"], S0[0].astype(np.float64))
        good, _ = emulate_chain(*args)
        bad, _ = emulate_chain(*args, combine_frame_factors=True)
        errs.append((rel(good, o_ref[0]), rel(bad, o_ref[0])))
    assert all(g <= 2e-2 for g, _ in errs), errs
    assert max(b for _, b in errs) > 2e-2, errs


def test_bf16_intermediates_of_a_split_prefill():
    """A prefill split into a parallel build/solve kernel and a state walk would pass W', Ũ, Q̂, K̃ and P
    through HBM; in bf16, Ũ is the one operand the fused kernel keeps wider (fp32 in TMEM).  Rounding
    it too keeps the bench workload's o within the bf16 bar."""
    wl0 = synth.WORKLOADS["prefill_1p3b"]
    wl = synth.Workload(wl0.name, 1, 4, 1024, wl0.K, wl0.V, wl0.dtype, wl0.alpha_mu, seed=wl0.seed)
    for h in range(2):
        x = synth.make_inputs(wl, chains=[(0, h)])
        c = {k: a[0].astype(np.float64) for k, a in x.items()}
        o_ref, S_ref = oracle.chain_recurrence(*(x[k].astype(np.float64) for k in ("q", "k", "v", "alpha", "b", "w")))
        args = (c["q"], c["k"], c["v"], c["alpha"], c["b"], c["w"], None)
        o, S = emulate_chain(*args, stored_u_bf16=True)
        assert rel(o, o_ref[0]) <= 2e-2 and rel(S, S_ref[0]) <= 2e-2, (rel(o, o_ref[0]), rel(S, S_ref[0]))
