"""GPU parity of gdn2_chunk_fwd against the fp64 oracle (same seeded inputs).

Bar: max|gpu - oracle| / max|oracle| <= 1e-4 for fp32 tokens, <= 2e-2 for bf16 tokens
with fp32 state, on o and on S_T.  Small cases compare every element; the full-size
workloads run the whole launch and compare sampled (b, h) chains, which the oracle
recomputes alone from the same counter-based generator.
"""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import TOL, assert_close, cuda_or_skip, f64, prefill, to_device, workload

pytestmark = pytest.mark.gpu


def _full_check(wl, S0_np=None, C=64):
    torch, g = cuda_or_skip()
    x = synth.make_inputs(wl)
    xd = to_device(torch, x, wl.dtype)
    S0 = None if S0_np is None else torch.from_numpy(S0_np).cuda()
    o, ST = prefill(torch, g, xd, S0, C=C)
    ref_o, ref_S = oracle.recurrence(*(x[k] for k in ("q", "k", "v", "alpha", "b", "w")), S0_np)
    e1 = assert_close("o", f64(o), ref_o, TOL[wl.dtype])
    e2 = assert_close("S_T", f64(ST), ref_S, TOL[wl.dtype])
    return e1, e2


def test_tiny_f32_workload():
    _full_check(synth.WORKLOADS["tiny_f32"])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("K,V", [(64, 64), (64, 128), (128, 64), (128, 128)])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 200])
def test_small_shapes(dtype, K, V, T):
    wl = synth.Workload("s", 2, 3, T, K, V, dtype, 1.0 if dtype == "bf16" else 0.0, s0_std=0.05,
                        seed=1000 + T + K + 3 * V)
    _full_check(wl, synth.make_state(wl))


@pytest.mark.parametrize("gates", ["kda", "gdn"])
def test_collapsed_gates_small(gates):
    wl = synth.Workload("c", 2, 4, 192, 128, 128, "bf16", 1.0, gates=gates, seed=77)
    _full_check(wl)


def test_slow_decay_small():
    wl = synth.Workload("sd", 2, 4, 320, 128, 128, "bf16", 1.0, alpha_scale=0.02, s0_std=0.01, seed=78)
    _full_check(wl, synth.make_state(wl))


# (B, H): up to 64 chains run the fused kernel, more the two-stage path
PATHS = pytest.mark.parametrize("BH", [(1, 2), (2, 33)], ids=["fused", "two_stage"])


@PATHS
def test_extreme_decay_and_unit_decay(BH):
    """alpha spanning 1e-30 .. 1 (every factor stays finite), exact alpha = 1 rows."""
    torch, g = cuda_or_skip()
    wl = synth.Workload("x", BH[0], BH[1], 130, 128, 128, "bf16", 1.0, seed=79, s0_std=0.05)
    x = synth.make_inputs(wl)
    rng = np.random.default_rng(5)
    a = x["alpha"].copy()
    mask = rng.random(a.shape) < 0.05
    a[mask] = np.float32(1e-30)
    a[:, 10:20] = 1.0
    x["alpha"] = a
    S0 = synth.make_state(wl)
    xd = to_device(torch, x, wl.dtype)
    o, ST = prefill(torch, g, xd, torch.from_numpy(S0).cuda())
    ref_o, ref_S = oracle.recurrence(*(x[k] for k in ("q", "k", "v", "alpha", "b", "w")), S0)
    assert_close("o", f64(o), ref_o, TOL["bf16"])
    assert_close("S_T", f64(ST), ref_S, TOL["bf16"])


@PATHS
def test_tiny_first_decay_of_each_chunk(BH):
    """The first alpha of every chunk is 1e-30 in half of the key channels, whose other tokens decay
    by 1/2: each chunk's log-decay span (63 in log2) is far below the wide-span limit, but the
    midpoint of its prefix lies near -131, so a decay factor formed as exp(-m) before the chunk's
    first position would leave fp32's range.  Every factor the method needs, exp(g_r - m), is within
    exp(+-span/2)."""
    torch, g = cuda_or_skip()
    wl = synth.Workload("tf", BH[0], BH[1], 64 * 3 + 2, 128, 128, "bf16", 1.0, seed=88, s0_std=0.05)
    x = synth.make_inputs(wl)
    a = x["alpha"].copy()
    a[..., ::2] = np.float32(0.5)
    a[:, ::64, :, ::2] = np.float32(1e-30)
    x["alpha"] = a
    S0 = synth.make_state(wl)
    xd = to_device(torch, x, wl.dtype)
    o, ST = prefill(torch, g, xd, torch.from_numpy(S0).cuda())
    ref_o, ref_S = oracle.recurrence(*(x[k] for k in ("q", "k", "v", "alpha", "b", "w")), S0)
    assert_close("o", f64(o), ref_o, TOL["bf16"])
    assert_close("S_T", f64(ST), ref_S, TOL["bf16"])


@PATHS
@pytest.mark.parametrize("span", [120.0, 165.0, 172.0, 176.0])
def test_chunk_spans_near_the_tensor_core_limit(span, BH):
    """Every chunk decays by about `span` (log2) in half of the key channels, so the kernel's
    decay factors around the chunk midpoint reach 2^(span/2) and the frame factors of two
    consecutive chunks multiply to about 2^-span (below fp32's range for span > 149); 176 lies
    past the tensor-core limit (173) and takes the wide-span path.  The other channels decay
    slowly, so the carried state stays visible in o."""
    torch, g = cuda_or_skip()
    wl = synth.Workload("x", BH[0], BH[1], 320, 128, 128, "bf16", 1.0, seed=81, s0_std=0.05)
    x = synth.make_inputs(wl)
    a = x["alpha"].copy()
    a[..., ::2] = np.float32(2.0 ** (-span / 64.0))    # per-token decay of the fast channels
    a[..., 1::2] = np.maximum(a[..., 1::2], np.float32(0.9))
    x["alpha"] = a
    S0 = synth.make_state(wl)
    xd = to_device(torch, x, wl.dtype)
    o, ST = prefill(torch, g, xd, torch.from_numpy(S0).cuda())
    ref_o, ref_S = oracle.recurrence(*(x[k] for k in ("q", "k", "v", "alpha", "b", "w")), S0)
    assert_close("o", f64(o), ref_o, TOL["bf16"])
    assert_close("S_T", f64(ST), ref_S, TOL["bf16"])


@pytest.mark.parametrize("alpha_scale", [1.0, 0.02])
def test_segmented_prefill_few_long_chains(alpha_scale):
    """Few chains and a long, ragged sequence (B1 H2, 41 chunks): the prefill runs in parallel
    over five segments of each chain (state maps of every segment, composed along the chain,
    then a rerun from the true start states); with alpha near 1 the carried state dominates."""
    torch, g = cuda_or_skip()
    wl = synth.Workload("seg", 1, 2, 64 * 40 + 37, 128, 128, "bf16", 1.0, seed=83, s0_std=0.05,
                        alpha_scale=alpha_scale)
    x = synth.make_inputs(wl)
    S0 = synth.make_state(wl)
    xd = to_device(torch, x, wl.dtype)
    o, ST = prefill(torch, g, xd, torch.from_numpy(S0).cuda())
    ref_o, ref_S = oracle.recurrence(*(x[k] for k in ("q", "k", "v", "alpha", "b", "w")), S0)
    assert_close("o", f64(o), ref_o, TOL["bf16"])
    assert_close("S_T", f64(ST), ref_S, TOL["bf16"])


def test_T0_copies_state_and_empty_batch():
    torch, g = cuda_or_skip()
    B, H, K, V = 2, 3, 64, 128
    z = lambda d: torch.zeros((B, 0, H, d), device="cuda", dtype=torch.bfloat16)
    S0 = torch.randn(B, H, K, V, device="cuda")
    o = torch.empty((B, 0, H, V), device="cuda", dtype=torch.bfloat16)
    S_T = torch.full((B, H, K, V), float("nan"), device="cuda")
    ws = g.new_workspace(g.gdn2_chunk_fwd_workspace_bytes(B, H, 0, K, V, 64, g.GDN2_BF16))
    alpha = torch.zeros((B, 0, H, K), device="cuda")
    g.gdn2_chunk_fwd(z(K), z(K), z(V), alpha, z(K), z(V), S0, o, S_T, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(S_T, S0)
    g.gdn2_chunk_fwd(z(K), z(K), z(V), alpha, z(K), z(V), None, o, S_T, workspace=ws)
    torch.cuda.synchronize()
    assert torch.count_nonzero(S_T).item() == 0


def test_in_place_resume_and_split():
    """S_T aliasing S0; two calls joined by the state equal one call."""
    torch, g = cuda_or_skip()
    wl = synth.Workload("r", 2, 2, 200, 128, 128, "bf16", 1.0, seed=80, s0_std=0.02)
    x = synth.make_inputs(wl)
    S0 = synth.make_state(wl)
    xd = to_device(torch, x, wl.dtype)
    o_all, S_all = prefill(torch, g, xd, torch.from_numpy(S0).cuda())
    S = torch.from_numpy(S0).cuda()
    cut = 96
    part = lambda s: {k: v[:, s].contiguous() for k, v in xd.items()}
    B, T, H, K = xd["q"].shape
    for sl in (slice(0, cut), slice(cut, T)):
        p = part(sl)
        o = torch.empty((B, sl.stop - sl.start, H, 128), dtype=torch.bfloat16, device="cuda")
        ws = g.new_workspace(g.gdn2_chunk_fwd_workspace_bytes(B, H, sl.stop - sl.start, K, 128, 64, g.GDN2_BF16))
        g.gdn2_chunk_fwd(p["q"], p["k"], p["v"], p["alpha"], p["b"], p["w"], S, o, S, workspace=ws)
        torch.cuda.synchronize()
        if sl.start == 0:
            o1 = o
        else:
            o2 = o
    ref_o, ref_S = oracle.recurrence(*(x[k] for k in ("q", "k", "v", "alpha", "b", "w")), S0)
    assert_close("o split", f64(torch.cat([o1, o2], dim=1)), ref_o, TOL["bf16"])
    assert_close("S split", f64(S), ref_S, TOL["bf16"])
    assert_close("S one call", f64(S_all), ref_S, TOL["bf16"])


def _sampled_check(name, chains, threads=None):
    torch, g = cuda_or_skip()
    wl = synth.WORKLOADS[name]
    x = synth.make_inputs(wl)
    S0 = synth.make_state(wl)
    xd = to_device(torch, x, wl.dtype)
    del x
    S0d = None if S0 is None else torch.from_numpy(S0).cuda()
    o, ST = prefill(torch, g, xd, S0d, poison=True)
    del xd
    xs = synth.make_inputs(wl, chains=chains)
    S0s = synth.make_state(wl, chains=chains)
    ref_o, ref_S = oracle.chain_recurrence(*(xs[k] for k in ("q", "k", "v", "alpha", "b", "w")), S0s,
                                           threads=threads)
    for n, (b, h) in enumerate(chains):
        assert_close(f"o chain {b},{h}", f64(o[b, :, h]), ref_o[n], TOL[wl.dtype])
        assert_close(f"S_T chain {b},{h}", f64(ST[b, h]), ref_S[n], TOL[wl.dtype])
    assert torch.isfinite(o.float()).all().item()
    assert torch.isfinite(ST).all().item()


def test_prefill_1p3b_full_size_sampled():
    # two heads of every batch element: 16 of the 128 chains
    _sampled_check("prefill_1p3b", [(b, h) for b in range(8) for h in ((5 * b) % 16, (5 * b + 9) % 16)])


def test_prefill_kda_full_size_sampled():
    _sampled_check("prefill_kda", [(0, 1), (2, 14), (5, 6), (7, 9)])


def test_prefill_gdn_full_size_sampled():
    _sampled_check("prefill_gdn", [(1, 0), (3, 11), (4, 5), (7, 14)])


def test_prefill_long_all_chains():
    # every head: 1,024 chunks each, typical per-chunk log-decay spans of 100-170 (log2)
    _sampled_check("prefill_long", [(0, h) for h in range(16)])


def test_prefill_slow_decay_full_size_sampled():
    _sampled_check("prefill_slow_decay", [(0, 12), (2, 3), (6, 8)])


@pytest.mark.parametrize("case", ["segmented", "two_stage", "simt_f32", "simt_bf16_d64"])
def test_in_place_state_alias(case):
    """S_T passed as the same buffer as S0 (the ABI allows it): the segmented path (few long
    chains, B*H <= 64 and >= 32 chunks) and the CUDA-core path give the oracle's result."""
    torch, g = cuda_or_skip()
    if case == "segmented":
        wl = synth.Workload("ip", 1, 2, 64 * 40 + 5, 128, 128, "bf16", 1.0, seed=84, s0_std=0.05,
                            alpha_scale=0.02)
    elif case == "two_stage":
        wl = synth.Workload("ip", 2, 33, 200, 128, 128, "bf16", 1.0, seed=87, s0_std=0.05)
    elif case == "simt_f32":
        wl = synth.Workload("ip", 2, 3, 200, 64, 64, "f32", 0.0, seed=85, s0_std=0.05)
    else:
        wl = synth.Workload("ip", 2, 3, 130, 64, 128, "bf16", 1.0, seed=86, s0_std=0.05)
    x = synth.make_inputs(wl)
    S0 = synth.make_state(wl)
    xd = to_device(torch, x, wl.dtype)
    S = torch.from_numpy(S0).cuda()
    B, T, H, K = xd["q"].shape
    V = xd["v"].shape[-1]
    o = torch.full((B, T, H, V), float("nan"), dtype=xd["q"].dtype, device="cuda")
    dt = g.GDN2_BF16 if wl.dtype == "bf16" else g.GDN2_F32
    ws = g.new_workspace(g.gdn2_chunk_fwd_workspace_bytes(B, H, T, K, V, 64, dt))
    g.gdn2_chunk_fwd(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["b"], xd["w"], S, o, S, workspace=ws)
    torch.cuda.synchronize()
    assert g.gdn2_workspace_status(ws) == 0
    ref_o, ref_S = oracle.recurrence(*(x[k] for k in ("q", "k", "v", "alpha", "b", "w")), S0)
    assert_close("o", f64(o), ref_o, TOL[wl.dtype])
    assert_close("S_T (in place)", f64(S), ref_S, TOL[wl.dtype])


@pytest.mark.parametrize("T", [1, 63, 64, 65, 200])
def test_two_stage_small(T):
    """More than 64 chains: the intra-chunk stage runs over every chunk-head, then one block per
    chain walks the state; ragged and single-token sequences included."""
    torch, g = cuda_or_skip()
    wl = synth.Workload("ts", 2, 33, T, 128, 128, "bf16", 1.0, s0_std=0.05, seed=2000 + T)
    assert g.gdn2_chunk_fwd_path(2, 33, T, 128, 128, 64, g.GDN2_BF16) == 2
    _full_check(wl, synth.make_state(wl))


@pytest.mark.parametrize("gates", ["kda", "gdn"])
def test_two_stage_collapsed_gates(gates):
    wl = synth.Workload("tc", 2, 33, 192, 128, 128, "bf16", 1.0, gates=gates, seed=2010)
    _full_check(wl)


def test_two_stage_windows():
    """260 chunks of 65 chains: a window of the record buffer holds 252 chunks of every chain, so the
    sequence runs as two windows with the state carried between them; slow decay keeps the carried
    state visible.  Sampled chains against the oracle."""
    torch, g = cuda_or_skip()
    wl = synth.Workload("tw", 1, 65, 64 * 260 - 3, 128, 128, "bf16", 1.0, s0_std=0.05, seed=2100, alpha_scale=0.02)
    assert g.gdn2_chunk_fwd_path(1, 65, wl.T, 128, 128, 64, g.GDN2_BF16) == 2
    _sampled_wl_check(wl, [(0, 0), (0, 31), (0, 64)])


def test_two_stage_segmented_windows():
    """64 chains of 300 chunks: windows of 256 chunks, each chain's window cut into two segments
    walked in parallel and composed; the second window starts from the first one's state."""
    torch, g = cuda_or_skip()
    wl = synth.Workload("sw", 1, 64, 64 * 300 - 11, 128, 128, "bf16", 1.0, s0_std=0.05, seed=2101, alpha_scale=0.02)
    assert g.gdn2_chunk_fwd_path(1, 64, wl.T, 128, 128, 64, g.GDN2_BF16) == 2
    _sampled_wl_check(wl, [(0, 0), (0, 40), (0, 63)])


def _sampled_wl_check(wl, chains):
    torch, g = cuda_or_skip()
    x = synth.make_inputs(wl)
    S0 = synth.make_state(wl)
    xd = to_device(torch, x, wl.dtype)
    del x
    o, ST = prefill(torch, g, xd, torch.from_numpy(S0).cuda())
    del xd
    xs = synth.make_inputs(wl, chains=chains)
    S0s = synth.make_state(wl, chains=chains)
    ref_o, ref_S = oracle.chain_recurrence(*(xs[k] for k in ("q", "k", "v", "alpha", "b", "w")), S0s)
    for n, (b, h) in enumerate(chains):
        assert_close(f"o chain {b},{h}", f64(o[b, :, h]), ref_o[n], TOL[wl.dtype])
        assert_close(f"S_T chain {b},{h}", f64(ST[b, h]), ref_S[n], TOL[wl.dtype])
    assert torch.isfinite(o.float()).all().item()
