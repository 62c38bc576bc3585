"""GPU parity of gdn2_decode_step against the fp64 oracle.

The full-size case runs the 1,000-step B=256, H=16, d=128 decode on every head of
the launch; heads are independent, so sampled heads receive the generator's exact
per-step tokens (and are checked against the oracle), the other heads cycle a pool
of generated steps.
"""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import TOL, assert_close, cuda_or_skip, f64, to_device

pytestmark = pytest.mark.gpu


def _step(g, torch, xd, S):
    B, H, K = xd["q"].shape
    o = torch.full((B, H, xd["v"].shape[-1]), float("nan"), dtype=xd["q"].dtype, device="cuda")
    g.gdn2_decode_step(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["b"], xd["w"], S, o)
    return o


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("K,V", [(64, 64), (64, 128), (128, 64), (128, 128)])
def test_decode_small(dtype, K, V):
    torch, g = cuda_or_skip()
    wl = synth.Workload("d", 3, 5, 1, K, V, dtype, 1.0, s0_std=0.05, seed=300 + K + V, decode=True, steps=20)
    S0 = synth.make_state(wl)
    S = torch.from_numpy(S0).cuda()
    S_ref = S0.astype(np.float64)
    for s in range(wl.steps):
        x = synth.make_inputs(wl, step=s)
        o = _step(g, torch, to_device(torch, x, dtype), S)
        ref = oracle.decode_step(*(x[k] for k in ("q", "k", "v", "alpha", "b", "w")), S_ref)
        torch.cuda.synchronize()
        assert_close(f"o step {s}", f64(o), ref, TOL[dtype])
    assert_close("S", f64(S), S_ref, TOL[dtype])


def test_decode_matches_T1_prefill():
    torch, g = cuda_or_skip()
    wl = synth.Workload("d1", 2, 3, 1, 128, 128, "bf16", 1.0, s0_std=0.05, seed=400)
    x = synth.make_inputs(wl)           # [B, 1, H, d]
    S0 = synth.make_state(wl)
    xd = to_device(torch, x, "bf16")
    S = torch.from_numpy(S0).cuda()
    o_pre = torch.empty((2, 1, 3, 128), dtype=torch.bfloat16, device="cuda")
    S_pre = torch.empty_like(S)
    ws = g.new_workspace(g.gdn2_chunk_fwd_workspace_bytes(2, 3, 1, 128, 128, 64, g.GDN2_BF16))
    g.gdn2_chunk_fwd(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["b"], xd["w"], S, o_pre, S_pre, workspace=ws)
    xdd = {k: v[:, 0].contiguous() for k, v in xd.items()}
    o_dec = _step(g, torch, xdd, S)
    torch.cuda.synchronize()
    ref_o, ref_S = oracle.recurrence(*(x[k] for k in ("q", "k", "v", "alpha", "b", "w")), S0)
    # both entry points against the oracle at the bf16 tolerance, and against each other
    assert_close("decode o", f64(o_dec), ref_o[:, 0], TOL["bf16"])
    assert_close("prefill o", f64(o_pre[:, 0]), ref_o[:, 0], TOL["bf16"])
    assert_close("decode S", f64(S), ref_S, TOL["bf16"])
    assert_close("prefill S", f64(S_pre), ref_S, TOL["bf16"])
    assert_close("decode vs prefill S", f64(S), f64(S_pre), TOL["bf16"])


def test_decode_b256_1000_steps_sampled_heads():
    torch, g = cuda_or_skip()
    wl = synth.WORKLOADS["decode_b256"]
    heads = [(0, 0), (17, 5), (255, 15), (128, 9)]
    S0 = synth.make_state(wl)
    S = torch.from_numpy(S0).cuda()
    S_ref = synth.make_state(wl, chains=heads).astype(np.float64)
    pool = [to_device(torch, synth.make_inputs(wl, step=s), "bf16") for s in range(4)]
    bi = torch.tensor([b for b, _ in heads], device="cuda")
    hi = torch.tensor([h for _, h in heads], device="cuda")
    for s in range(wl.steps):
        xs = synth.make_inputs(wl, chains=heads, step=s)        # exact tokens of the sampled heads
        xd = {k: v.clone() for k, v in pool[s % len(pool)].items()}
        exact = to_device(torch, xs, "bf16")
        for key in xd:
            xd[key][bi, hi] = exact[key]
        o = _step(g, torch, xd, S)
        ref = oracle.decode_step(*(xs[k][:, None] for k in ("q", "k", "v", "alpha", "b", "w")),
                                 S_ref.reshape(len(heads), 1, 128, 128), threads=4)
        if s % 100 == 99 or s == 0:
            torch.cuda.synchronize()
            assert_close(f"o step {s}", f64(o[bi, hi]), ref[:, 0], TOL["bf16"])
    torch.cuda.synchronize()
    assert_close("S after 1000 steps", f64(S[bi, hi]), S_ref, TOL["bf16"])
    assert torch.isfinite(S).all().item()
