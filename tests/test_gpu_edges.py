"""GPU parity of gdn2_chunk_fwd_edges (the prefill with the layer edges fused) against the fp64
oracle: oracle.layer_edges on the stored raw inputs, the recurrence, oracle.rms_norm."""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import TOL, assert_close, cuda_or_skip, f64

pytestmark = pytest.mark.gpu


def raw_inputs(B, T, H, seed, chains=None):
    """Seeded raw layer inputs ([B,T,H,d], or [n,T,d] for a list of (b, h) chains), the recipe of
    synth.make_raw_inputs: unnormalised q, k (scale 3), v ~ N(0,1), decay logits ~ N(1,1) (fp32),
    gate logits ~ N(0,1)."""
    return synth.make_raw_inputs(synth.Workload("edges", B, H, T, 128, 128, "bf16", 1.0, seed=seed), chains)


def to_dev(torch, x):
    return {k: torch.from_numpy(np.ascontiguousarray(v)).cuda().to(torch.float32 if k == "a" else torch.bfloat16)
            for k, v in x.items()}


def assert_normed_close(name, got, ref_o, weight, tol):
    """RMSNorm output against the oracle: the norm turns each row's error relative to the largest
    row of o into an error relative to that row, so row i may deviate by tol * max_j |o_j| / |o_i|
    (relative to its own normalised size); this is the bf16 bound on o carried through the norm."""
    ref = oracle.rms_norm(ref_o, weight)
    rn_o = np.sqrt(np.mean(ref_o * ref_o, axis=-1))
    rn = np.sqrt(np.mean(ref * ref, axis=-1))
    err_row = np.sqrt(np.mean((got - ref) ** 2, axis=-1))
    allow = tol * rn * np.maximum(1.0, rn_o.max() / np.maximum(rn_o, 1e-30))
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    worst = np.max(err_row / allow)
    assert worst <= 1.0, f"{name}: row error {worst:.2f} x its allowance"


def reference(x, S0):
    q, k, alpha, b, w = oracle.layer_edges(x["q"], x["k"], x["a"], x["b"], x["w"])
    return oracle.recurrence(q, k, x["v"], alpha, b, w, S0)


def run(torch, g, xd, S0, weight):
    B, T, H, K = xd["q"].shape
    o = torch.full((B, T, H, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    ST = torch.full((B, H, K, 128), float("nan"), dtype=torch.float32, device="cuda")
    g.gdn2_chunk_fwd_edges(xd["q"], xd["k"], xd["v"], xd["a"], xd["b"], xd["w"], S0, weight, o, ST)
    torch.cuda.synchronize()
    return o, ST


@pytest.mark.parametrize("norm", [False, True])
@pytest.mark.parametrize("T", [1, 64, 200])
def test_edges_small(norm, T):
    torch, g = cuda_or_skip()
    x = raw_inputs(2, T, 3, seed=91)
    S0 = np.random.default_rng(7).normal(scale=0.05, size=(2, 3, 128, 128)).astype(np.float32)
    weight = np.random.default_rng(8).normal(size=128).astype(np.float32) if norm else None
    o, ST = run(torch, g, to_dev(torch, x), torch.from_numpy(S0).cuda(),
                None if weight is None else torch.from_numpy(weight).cuda())
    ref_o, ref_S = reference(x, S0)
    if weight is None:
        assert_close("o", f64(o), ref_o, TOL["bf16"])
    else:
        assert_normed_close("o", f64(o), ref_o, weight, TOL["bf16"])
    assert_close("S_T", f64(ST), ref_S, TOL["bf16"])


def test_edges_segmented_long_chain():
    """Few chains, 41 chunks: the segmented path runs with the edges fused as well."""
    torch, g = cuda_or_skip()
    x = raw_inputs(1, 64 * 40 + 37, 2, seed=92)
    S0 = np.random.default_rng(9).normal(scale=0.05, size=(1, 2, 128, 128)).astype(np.float32)
    weight = np.random.default_rng(10).normal(size=128).astype(np.float32)
    o, ST = run(torch, g, to_dev(torch, x), torch.from_numpy(S0).cuda(), torch.from_numpy(weight).cuda())
    ref_o, ref_S = reference(x, S0)
    assert_normed_close("o", f64(o), ref_o, weight, TOL["bf16"])
    assert_close("S_T", f64(ST), ref_S, TOL["bf16"])


def test_edges_full_size_sampled():
    """The 1.3B-layer prefill shape (B8 H16 T4096) from raw inputs, four chains checked."""
    torch, g = cuda_or_skip()
    B, T, H = 8, 4096, 16
    x = raw_inputs(B, T, H, seed=93)
    weight = np.random.default_rng(11).normal(size=128).astype(np.float32)
    o, ST = run(torch, g, to_dev(torch, x), None, torch.from_numpy(weight).cuda())
    del x
    chains = [(0, 0), (2, 9), (5, 4), (7, 15)]
    xs = raw_inputs(B, T, H, seed=93, chains=chains)
    q, k, alpha, b, w = oracle.layer_edges(xs["q"], xs["k"], xs["a"], xs["b"], xs["w"])
    ref_o, ref_S = oracle.chain_recurrence(q, k, xs["v"], alpha, b, w)
    for n, (bb, h) in enumerate(chains):
        assert_normed_close(f"o chain {bb},{h}", f64(o[bb, :, h]), ref_o[n], weight, TOL["bf16"])
        assert_close(f"S_T chain {bb},{h}", f64(ST[bb, h]), ref_S[n], TOL["bf16"])


def test_edges_rejects_unsupported_shapes():
    torch, g = cuda_or_skip()
    x = to_dev(torch, raw_inputs(1, 64, 1, seed=94))
    small = {k: v[..., :64].contiguous() for k, v in x.items()}
    o = torch.empty((1, 64, 1, 64), dtype=torch.bfloat16, device="cuda")
    ST = torch.empty((1, 1, 64, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(g.GDN2Error):
        g.gdn2_chunk_fwd_edges(small["q"], small["k"], small["v"], small["a"], small["b"], small["w"], None, None,
                               o, ST)


@pytest.mark.parametrize("norm", [False, True])
@pytest.mark.parametrize("T", [1, 65, 200])
def test_edges_two_stage_small(norm, T):
    """More than 64 chains: the maps fused into the two-stage path (prep: norms, sigmoids and the
    decay from its logit; walk: RMSNorm of the o rows)."""
    torch, g = cuda_or_skip()
    assert g.gdn2_chunk_fwd_path(2, 33, T, 128, 128, 64, g.GDN2_BF16) == 2
    x = raw_inputs(2, T, 33, seed=95)
    S0 = np.random.default_rng(12).normal(scale=0.05, size=(2, 33, 128, 128)).astype(np.float32)
    weight = np.random.default_rng(13).normal(size=128).astype(np.float32) if norm else None
    o, ST = run(torch, g, to_dev(torch, x), torch.from_numpy(S0).cuda(),
                None if weight is None else torch.from_numpy(weight).cuda())
    ref_o, ref_S = reference(x, S0)
    if weight is None:
        assert_close("o", f64(o), ref_o, TOL["bf16"])
    else:
        assert_normed_close("o", f64(o), ref_o, weight, TOL["bf16"])
    assert_close("S_T", f64(ST), ref_S, TOL["bf16"])


def test_layer_edge_maps_and_rms_norm():
    """The stand-alone map kernels against the oracle's maps: q, k, b, w are bf16 roundings of the
    fp64 maps (half an ulp, 2^-9 relative, plus the fp32 arithmetic), alpha fp32; RMSNorm likewise."""
    torch, g = cuda_or_skip()
    for B, T, H in ((2, 70, 3), (1, 5, 40)):
        x = raw_inputs(B, T, H, seed=96)
        xd = to_dev(torch, x)
        q, k, b = (torch.empty_like(xd["q"]) for _ in range(3))
        w = torch.empty_like(xd["w"])
        alpha = torch.empty_like(xd["a"])
        g.gdn2_layer_edge_maps(xd["q"], xd["k"], xd["a"], xd["b"], xd["w"], q, k, alpha, b, w)
        torch.cuda.synchronize()
        ref = oracle.layer_edges(*(xd[n].double().cpu().numpy() for n in ("q", "k", "a", "b", "w")))
        for name, got, r in zip(("q", "k", "alpha", "b", "w"), (q, k, alpha, b, w), ref):
            bar = 1e-5 if name == "alpha" else 2.0 ** -8
            err = np.max(np.abs(f64(got) - r) / np.maximum(np.abs(r), 1e-30))
            assert err <= bar, f"{name}: elementwise rel err {err:.2e} > {bar:.1e}"
        o = torch.randn((B, T, H, 128), device="cuda").to(torch.bfloat16)
        weight = torch.randn(128, device="cuda")
        ref_n = oracle.rms_norm(f64(o), weight.double().cpu().numpy())
        g.gdn2_rms_norm(o, weight)
        torch.cuda.synchronize()
        assert_close("rms_norm", f64(o), ref_n, 2.0 ** -7)


def test_edges_unfused_layer_matches():
    """The unfused layer -- the map kernel, the plain prefill, RMSNorm -- gives the oracle's result on
    the two-stage shapes, like the fused entry point."""
    torch, g = cuda_or_skip()
    x = raw_inputs(2, 130, 33, seed=97)
    xd = to_dev(torch, x)
    q, k, b = (torch.empty_like(xd["q"]) for _ in range(3))
    w = torch.empty_like(xd["w"])
    alpha = torch.empty_like(xd["a"])
    weight_np = np.random.default_rng(14).normal(size=128).astype(np.float32)
    weight = torch.from_numpy(weight_np).cuda()
    g.gdn2_layer_edge_maps(xd["q"], xd["k"], xd["a"], xd["b"], xd["w"], q, k, alpha, b, w)
    o, ST = g.chunk_fwd(q, k, xd["v"], alpha, b, w)
    g.gdn2_rms_norm(o, weight)
    torch.cuda.synchronize()
    ref_o, ref_S = reference(x, None)
    assert_normed_close("o", f64(o), ref_o, weight_np, TOL["bf16"])
    assert_close("S_T", f64(ST), ref_S, TOL["bf16"])
