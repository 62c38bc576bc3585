"""GPU parity of gdn2_chunk_bwd (the backward pass) against the fp64 backward oracle.

The CUDA backward computes every gradient in fp32 from the exact token values (bf16
tokens are widened, never re-rounded), so the bar is the fp32 one for both token
dtypes: max|gpu - oracle| / max|oracle| <= 1e-4 per gradient tensor, except dalpha.
dalpha is d(log alpha) / alpha; the kernels form d(log alpha) as a sum over at most 64
steps of per-step terms (plus an exact chunk-boundary term), so its absolute error is
that of fp32 sums of O(|q dq| + |k dk|) terms, divided by alpha.  Its bar is therefore
stated on alpha * dalpha (= d log alpha): 1e-4 relative to max|d log alpha|.

Small cases compare every element; the full-size workload runs the whole launch and
compares sampled (b, h) chains, which the oracle recomputes alone.
"""
import numpy as np
import pytest

import oracle
import synth
from oracle import backward as ob
from tests.gpu_util import assert_close, cuda_or_skip, f64, to_device, workload

pytestmark = pytest.mark.gpu

TOL = 1e-4
GRADS = ("dq", "dk", "dv", "dalpha", "db", "dw")


def output_grads(wl, chains=None):
    return synth.make_output_grads(wl, chains)


def run_bwd(torch, g, xd, S0, dO, dST, want_dS0=True):
    q = xd["q"]
    B, T, H, K = q.shape
    V = xd["v"].shape[-1]
    dev = q.device
    out = {n: torch.full((B, T, H, K if n in ("dq", "dk", "dalpha", "db") else V), float("nan"), device=dev)
           for n in GRADS}
    dS0 = torch.full((B, H, K, V), float("nan"), device=dev) if want_dS0 else None
    ws = torch.full((max(g.gdn2_chunk_bwd_workspace_bytes(B, H, T, K, V), 256),), 0xFF, dtype=torch.uint8,
                    device=dev)   # NaN pattern: a read of an unwritten word shows up
    g.gdn2_chunk_bwd(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["b"], xd["w"], S0, dO, dST, out["dq"], out["dk"],
                     out["dv"], out["dalpha"], out["db"], out["dw"], dS0, workspace=ws)
    torch.cuda.synchronize()
    res = {n: f64(t) for n, t in out.items()}
    res["dS0"] = None if dS0 is None else f64(dS0)
    return res


def check(name, got, ref, alpha, tol=TOL):
    if name.split()[0] == "dalpha":
        return assert_close("alpha*dalpha", got * alpha, ref * alpha, tol)
    return assert_close(name, got, ref, tol)


def full_case(wl, with_S0=True, with_dST=True):
    torch, g = cuda_or_skip()
    x = synth.make_inputs(wl)
    S0 = synth.make_state(wl) if (with_S0 and wl.s0_std) else None
    dO, dST = output_grads(wl)
    if not with_dST:
        dST = None
    xd = to_device(torch, x, wl.dtype)
    td = xd["q"].dtype
    got = run_bwd(torch, g, xd, None if S0 is None else torch.from_numpy(S0).cuda(),
                  torch.from_numpy(dO).cuda().to(td), None if dST is None else torch.from_numpy(dST).cuda())
    ref = ob.recurrence_backward(*(x[k] for k in ("q", "k", "v", "alpha", "b", "w")), S0, dO, dST)
    for name, r in zip(GRADS + ("dS0",), ref):
        check(name, got[name], r, x["alpha"].astype(np.float64))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("K,V", [(64, 64), (64, 128), (128, 64), (128, 128)])
@pytest.mark.parametrize("T", [1, 15, 64, 65, 200])
def test_small_shapes(dtype, K, V, T):
    wl = synth.Workload("bw", 2, 3, T, K, V, dtype, 1.0 if dtype == "bf16" else 0.0, s0_std=0.05,
                        seed=2000 + T + K + 3 * V)
    full_case(wl)


def test_zero_initial_state_and_no_state_gradient():
    wl = synth.Workload("bw0", 1, 4, 130, 128, 128, "bf16", 1.0, seed=2101)
    full_case(wl, with_S0=False, with_dST=False)


@pytest.mark.parametrize("gates", ["kda", "gdn"])
def test_collapsed_gates(gates):
    wl = synth.Workload("bwg", 1, 3, 150, 128, 128, "bf16", 1.0, gates=gates, s0_std=0.05, seed=2102)
    full_case(wl)


def test_slow_decay():
    wl = synth.Workload("bws", 1, 3, 300, 128, 128, "bf16", 1.0, alpha_scale=0.02, s0_std=0.05, seed=2103)
    full_case(wl)


def test_empty_sequence_copies_state_gradient():
    torch, g = cuda_or_skip()
    B, H, K, V = 2, 3, 128, 64
    dST = torch.randn(B, H, K, V, device="cuda")
    dS0 = torch.full_like(dST, float("nan"))
    e = torch.empty(B, 0, H, K, device="cuda")
    ev = torch.empty(B, 0, H, V, device="cuda")
    g.gdn2_chunk_bwd(e, e, ev, e, e, ev, None, ev, dST, e, e, ev, e, e, ev, dS0)
    torch.cuda.synchronize()
    assert torch.equal(dS0, dST)


def test_full_size_sampled_chains():
    """B8 H16 T4096 d=128 bf16 (the prefill workload): one launch, two chains checked."""
    torch, g = cuda_or_skip()
    wl = workload("prefill_1p3b")
    x = synth.make_inputs(wl)
    dO, dST = output_grads(wl)
    xd = to_device(torch, x, wl.dtype)
    got = run_bwd(torch, g, xd, None, torch.from_numpy(dO).cuda().to(torch.bfloat16), torch.from_numpy(dST).cuda())
    del xd
    for bb, h in ((0, 0), (7, 15)):
        c = {k: x[k][bb, :, h].astype(np.float64) for k in ("q", "k", "v", "alpha", "b", "w")}
        ref = ob.chain_backward(c["q"], c["k"], c["v"], c["alpha"], c["b"], c["w"], None, dO[bb, :, h],
                                dST[bb, h])
        for name, r in zip(GRADS, ref[:6]):
            check(f"{name} chain {bb},{h}", got[name][bb, :, h], r, c["alpha"])
        assert_close(f"dS0 chain {bb},{h}", got["dS0"][bb, h], ref[6], TOL)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_autograd_function(dtype):
    """gdn2_recurrence under torch.autograd: the gradients of L = sum(dO * o) + sum(dS_T * S_T) are the
    oracle's (inputs leaf tensors of the token dtype; the engine casts the fp32 gradients to it)."""
    torch, g = cuda_or_skip()
    wl = synth.Workload("bwa", 1, 2, 100, 64, 128, dtype, 1.0, s0_std=0.05, seed=2104)
    x = synth.make_inputs(wl)
    S0 = synth.make_state(wl)
    dO, dST = output_grads(wl)
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    names = ("q", "k", "v", "alpha", "b", "w")
    leaves = {n: torch.from_numpy(x[n]).cuda().to(torch.float32 if n == "alpha" else td).requires_grad_() for n in names}
    S0t = torch.from_numpy(S0).cuda().requires_grad_()
    o, ST = g.gdn2_recurrence(*(leaves[n] for n in names), S0t)
    L = (o.float() * torch.from_numpy(dO).cuda().to(td).float()).sum() + (ST * torch.from_numpy(dST).cuda()).sum()
    L.backward()
    ref = ob.recurrence_backward(*(x[n] for n in names), S0, dO, dST)
    a = x["alpha"].astype(np.float64)
    # bf16 leaves receive gradients rounded to bf16: the bar is the bf16 one there
    tol = TOL if dtype == "f32" else 2e-2
    for n, r in zip(names, ref[:6]):
        check("d" + n, f64(leaves[n].grad), r, a, tol if n != "alpha" else TOL)
    assert_close("dS0", f64(S0t.grad), ref[6], TOL)


def test_few_long_chains_column_split():
    """Two chains of 1,000 tokens (16 chunks): each chain's columns split over 4 blocks, so the row
    sums and the 16 chunk-boundary terms accumulate from every slice."""
    wl = synth.Workload("bwl", 1, 2, 1000, 128, 128, "bf16", 1.0, s0_std=0.05, seed=2105)
    full_case(wl)
