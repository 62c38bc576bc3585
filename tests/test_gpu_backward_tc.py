"""GPU parity of gdn2_chunk_bwd_tc (the tensor-core backward) against the fp64 backward oracle.

The tensor-core backward forms every product from bf16 operands with fp32 accumulation: the chunk
factors of the forward (rounded as in the forward's own tensor-core path), the saved state operand,
the state gradient's operand G̃ and dDelta, dR, dA and dP.  Each of those roundings is a relative
2^-9 on one operand; a gradient passes through at most four such products in a row (dDelta -> dR ->
dA -> dK̃), so its error is a few times the bf16 unit relative to the tensor's scale, the same order
as the forward's tensor-core path.  The bar is that path's: max|gpu - oracle| / max|oracle| <= 2e-2
per gradient tensor; dalpha is compared as alpha * dalpha (= d ln alpha), whose terms are sums of
products of the other gradients with the inputs.  The exact invariants of the chain rule are checked
without the oracle as well (test_gradient_invariants).

The reference is the step-by-step oracle (oracle/backward.py) on the same bf16-rounded inputs.
"""
import numpy as np
import pytest

import synth
from oracle import backward as ob
from tests.gpu_util import assert_close, cuda_or_skip, f64, to_device, workload

pytestmark = pytest.mark.gpu

TOL = 2e-2
GRADS = ("dq", "dk", "dv", "dalpha", "db", "dw")
NAMES = ("q", "k", "v", "alpha", "b", "w")


def run_bwd_tc(torch, g, xd, S0, dO, dST, want_dS0=True):
    q = xd["q"]
    B, T, H, K = q.shape
    V = xd["v"].shape[-1]
    dev = q.device
    out = {n: torch.full((B, T, H, K if n in ("dq", "dk", "dalpha", "db") else V), float("nan"), device=dev)
           for n in GRADS}
    dS0 = torch.full((B, H, K, V), float("nan"), device=dev) if want_dS0 else None
    nbytes = g.gdn2_chunk_bwd_tc_workspace_bytes(B, H, T, K, V)
    ws = g.new_workspace(nbytes, dev)
    if nbytes > g.STATUS_HEADER_BYTES:
        ws[g.STATUS_HEADER_BYTES:].fill_(0xFF)   # NaN pattern: a read of an unwritten word shows up
    g.gdn2_chunk_bwd_tc(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["b"], xd["w"], S0, dO, dST, out["dq"],
                        out["dk"], out["dv"], out["dalpha"], out["db"], out["dw"], dS0, workspace=ws)
    torch.cuda.synchronize()
    assert g.gdn2_workspace_status(ws) == 0
    res = {n: f64(t) for n, t in out.items()}
    res["dS0"] = None if dS0 is None else f64(dS0)
    return res


def check(name, got, ref, alpha, tol=TOL):
    if name.split()[0] == "dalpha":
        return assert_close(name.replace("dalpha", "alpha*dalpha"), got * alpha, ref * alpha, tol)
    return assert_close(name, got, ref, tol)


def full_case(wl, x=None, with_S0=True, with_dST=True):
    torch, g = cuda_or_skip()
    x = synth.make_inputs(wl) if x is None else x
    S0 = synth.make_state(wl) if (with_S0 and wl.s0_std) else None
    dO, dST = synth.make_output_grads(wl)
    if not with_dST:
        dST = None
    xd = to_device(torch, x, wl.dtype)
    dO_d = torch.from_numpy(dO).cuda().to(torch.bfloat16)
    got = run_bwd_tc(torch, g, xd, None if S0 is None else torch.from_numpy(S0).cuda(), dO_d,
                     None if dST is None else torch.from_numpy(dST).cuda())
    ref = ob.recurrence_backward(*(x[n] for n in NAMES), S0, dO_d.double().cpu().numpy(), dST)
    for name, r in zip(GRADS + ("dS0",), ref):
        check(name, got[name], r, x["alpha"].astype(np.float64))
    return got


@pytest.mark.parametrize("T", [1, 15, 64, 65, 200])
def test_small_shapes(T):
    wl = synth.Workload("bwtc", 2, 3, T, 128, 128, "bf16", 1.0, s0_std=0.05, seed=3000 + T)
    full_case(wl)


def test_zero_initial_state_and_no_state_gradient():
    wl = synth.Workload("bwtc0", 1, 4, 130, 128, 128, "bf16", 1.0, seed=3101)
    full_case(wl, with_S0=False, with_dST=False)


@pytest.mark.parametrize("gates", ["kda", "gdn"])
def test_collapsed_gates(gates):
    wl = synth.Workload("bwtcg", 1, 3, 150, 128, 128, "bf16", 1.0, gates=gates, s0_std=0.05, seed=3102)
    full_case(wl)


def test_slow_decay():
    wl = synth.Workload("bwtcs", 1, 3, 300, 128, 128, "bf16", 1.0, alpha_scale=0.02, s0_std=0.05, seed=3103)
    full_case(wl)


@pytest.mark.parametrize("span", [120.0, 176.0])
def test_wide_and_near_limit_chunk_spans(span):
    """Half of the key channels decay by about `span` (log2) per chunk: 120 keeps the tensor-core
    frame with factors up to 2^60, 176 sends every chunk down the wide-span branch (unscaled factors,
    K̃ = k 2^(g_C - g)); the other channels decay slowly so that the carried gradient matters."""
    wl = synth.Workload("bwtcw", 1, 3, 200, 128, 128, "bf16", 1.0, s0_std=0.05, seed=3104)
    x = synth.make_inputs(wl)
    a = x["alpha"].copy()
    a[..., ::2] = np.float32(2.0 ** (-span / 64.0))
    a[..., 1::2] = np.maximum(a[..., 1::2], np.float32(0.9))
    x["alpha"] = a
    full_case(wl, x=x)


def test_extreme_and_unit_decay():
    """alpha down to 1e-30 and rows of exact alpha = 1."""
    wl = synth.Workload("bwtcx", 1, 2, 130, 128, 128, "bf16", 1.0, s0_std=0.05, seed=3105)
    x = synth.make_inputs(wl)
    a = x["alpha"].copy()
    a[np.random.default_rng(7).random(a.shape) < 0.05] = np.float32(1e-30)
    a[:, 10:20] = 1.0
    x["alpha"] = a
    full_case(wl, x=x)


def test_few_long_chains_segmented_replay():
    """B1 H2 with 41 chunks (ragged): the forward replay walks each chain in segments (state maps per
    segment composed along the chain, then a walk from the true start states that saves every chunk's
    state operand); the reverse walk then runs over all 41 chunks."""
    wl = synth.Workload("bwtcl", 1, 2, 64 * 40 + 37, 128, 128, "bf16", 1.0, s0_std=0.05, seed=3106)
    full_case(wl)


def test_gradient_invariants():
    """Exact consequences of the chain rule, through the kernels alone.  The loss is linear in the
    output gradients, so scaling dO and dS_T by 2 doubles every gradient (bf16 dO stays exact);
    with alpha = 1, b = w = 0 the recurrence is S_t = S0, o_t = S0^T q_t, so dq_t = S0 dO_t, dS0 =
    dS_T + sum_t q_t dO_t^T, and dv = w ⊙ ddelta = 0 and dk = 0 (delta_t = u_t - Sbar_t^T e_t = 0)."""
    torch, g = cuda_or_skip()
    wl = synth.Workload("bwtci", 1, 2, 130, 128, 128, "bf16", 1.0, s0_std=0.05, seed=3107)
    x = synth.make_inputs(wl)
    S0 = synth.make_state(wl)
    dO, dST = synth.make_output_grads(wl)
    xd = to_device(torch, x, "bf16")
    dO_d = torch.from_numpy(dO).cuda().to(torch.bfloat16)
    S0_d, dST_d = torch.from_numpy(S0).cuda(), torch.from_numpy(dST).cuda()
    one = run_bwd_tc(torch, g, xd, S0_d, dO_d, dST_d)
    two = run_bwd_tc(torch, g, xd, S0_d, dO_d * 2, dST_d * 2)
    for n in GRADS + ("dS0",):
        np.testing.assert_array_equal(two[n], 2 * one[n], err_msg=n)

    fz = dict(x)
    fz["alpha"] = np.ones_like(x["alpha"])
    fz["b"] = np.zeros_like(x["b"])
    fz["w"] = np.zeros_like(x["w"])
    xd = to_device(torch, fz, "bf16")
    got = run_bwd_tc(torch, g, xd, S0_d, dO_d, dST_d)
    qd = xd["q"].double().cpu().numpy()
    dOd = dO_d.double().cpu().numpy()
    assert_close("dq = S0 dO", got["dq"], np.einsum("bhcv,bthv->bthc", S0.astype(np.float64), dOd), TOL)
    assert_close("dS0 = dS_T + sum q dO^T", got["dS0"], dST + np.einsum("bthc,bthv->bhcv", qd, dOd), TOL)
    for n in ("dv", "dk"):
        assert np.all(got[n] == 0.0), n


def test_empty_sequence_copies_state_gradient():
    torch, g = cuda_or_skip()
    B, H, K, V = 2, 3, 128, 128
    dST = torch.randn(B, H, K, V, device="cuda")
    dS0 = torch.full_like(dST, float("nan"))
    e = torch.empty(B, 0, H, K, device="cuda", dtype=torch.bfloat16)
    a = torch.empty(B, 0, H, K, device="cuda")
    f = torch.empty(B, 0, H, K, device="cuda")
    g.gdn2_chunk_bwd_tc(e, e, e, a, e, e, None, e, dST, f, f, f, f, f, f, dS0)
    torch.cuda.synchronize()
    assert torch.equal(dS0, dST)


def test_full_size_sampled_chains():
    """B8 H16 T4096 d=128 bf16 (the prefill workload): one launch, two chains checked."""
    torch, g = cuda_or_skip()
    wl = workload("prefill_1p3b")
    x = synth.make_inputs(wl)
    dO, dST = synth.make_output_grads(wl)
    xd = to_device(torch, x, wl.dtype)
    dO_d = torch.from_numpy(dO).cuda().to(torch.bfloat16)
    got = run_bwd_tc(torch, g, xd, None, dO_d, torch.from_numpy(dST).cuda())
    del xd
    dOr = dO_d.double().cpu().numpy()
    for bb, h in ((0, 0), (7, 15)):
        c = {n: x[n][bb, :, h].astype(np.float64) for n in NAMES}
        ref = ob.chain_backward(c["q"], c["k"], c["v"], c["alpha"], c["b"], c["w"], None, dOr[bb, :, h], dST[bb, h])
        for name, r in zip(GRADS, ref[:6]):
            check(f"{name} chain {bb},{h}", got[name][bb, :, h], r, c["alpha"])
        assert_close(f"dS0 chain {bb},{h}", got["dS0"][bb, h], ref[6], TOL)
