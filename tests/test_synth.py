"""The seeded input generator: determinism, chain slices, distributions, rounding."""
import numpy as np
import pytest

import synth


def test_counter_based_offsets():
    a = synth.normal(7, 3, 1000)
    b = synth.normal(7, 3, 400, offset=600)
    np.testing.assert_array_equal(a[600:], b)
    c = synth.normal(7, 3, 1000, threads=1)
    np.testing.assert_array_equal(a, c)
    assert not np.array_equal(a, synth.normal(7, 4, 1000))
    assert not np.array_equal(a, synth.normal(8, 3, 1000))


def test_normal_moments():
    x = synth.normal(0x9D2, 0, 2_000_000)
    assert abs(x.mean()) < 5e-3
    assert abs(x.std() - 1.0) < 5e-3
    u = synth.uniform(1, 1, 200_000)
    assert u.min() > 0 and u.max() < 1 and abs(u.mean() - 0.5) < 5e-3


def test_bf16_rounding_is_representable_and_nearest():
    x = synth.normal(1, 2, 10000)
    r = synth.round_to(x, "bf16")
    r32 = r.astype(np.float32)
    assert np.all((r32.view(np.uint32) & 0xFFFF) == 0)
    # nearest: no other bf16 value is closer to fp32(x) than r
    x32 = x.astype(np.float32).astype(np.float64)
    spacing = 2.0 ** (np.floor(np.log2(np.abs(x32))) - 7)   # bf16 keeps 8 significant bits
    assert np.all(np.abs(r - x32) <= 0.5 * spacing)


def test_small_workload_shapes_and_ranges():
    wl = synth.WORKLOADS["tiny_f32"]
    x = synth.make_inputs(wl)
    assert x["q"].shape == (1, 256, 2, 64) and x["v"].shape == (1, 256, 2, 64)
    assert x["q"].dtype == np.float32
    np.testing.assert_allclose(np.linalg.norm(x["k"].astype(np.float64), axis=-1), 1.0, rtol=1e-6)
    assert np.all(x["alpha"] > 0) and np.all(x["alpha"] <= 1)
    assert np.all(x["b"] > 0) and np.all(x["b"] < 1)
    assert synth.make_state(wl) is None


@pytest.mark.parametrize("name", ["prefill_kda", "prefill_gdn", "prefill_long", "decode_b256"])
def test_chain_subset_matches_full_tensor(name):
    wl = synth.WORKLOADS[name]
    small = synth.Workload(name, min(wl.B, 3), min(wl.H, 4), 1 if wl.decode else 70, 16, 8, wl.dtype,
                           wl.alpha_mu, wl.gates, wl.s0_std, wl.seed, decode=wl.decode)
    full = synth.make_inputs(small, step=0 if small.decode else None)
    chains = [(0, 1), (small.B - 1, small.H - 1)]
    sub = synth.make_inputs(small, chains=chains, step=0 if small.decode else None)
    for key in ("q", "k", "v", "alpha", "b", "w"):
        for n, (b, h) in enumerate(chains):
            ref = full[key][b, h] if small.decode else full[key][b, :, h]
            np.testing.assert_array_equal(sub[key][n], ref)
    if small.s0_std is not None:
        S_full = synth.make_state(small)
        S_sub = synth.make_state(small, chains=chains)
        for n, (b, h) in enumerate(chains):
            np.testing.assert_array_equal(S_sub[n], S_full[b, h])


def test_collapsed_gates_are_broadcast():
    wl = synth.Workload("g", 2, 3, 20, 8, 6, "bf16", 1.0, gates="gdn", seed=5)
    x = synth.make_inputs(wl)
    assert np.all(x["b"] == x["b"][..., :1])
    assert np.all(x["w"][..., 0] == x["b"][..., 0])
    assert np.all(x["alpha"] == x["alpha"][..., :1])


def test_time_window_matches_full():
    wl = synth.Workload("t", 1, 2, 50, 8, 4, "f32", 0.0, seed=9)
    full = synth.make_inputs(wl)
    part = synth.make_inputs(wl, chains=[(0, 1)], t_range=(10, 30))
    np.testing.assert_array_equal(part["q"][0], full["q"][0, 10:30, 1])


def test_bf16_workload_values_are_bf16_representable():
    wl = synth.Workload("r", 2, 3, 10, 16, 8, "bf16", 1.0, seed=11)
    x = synth.make_inputs(wl)
    for key in ("q", "k", "v", "b", "w"):
        assert np.all((x[key].view(np.uint32) & 0xFFFF) == 0), key
    assert np.any((x["alpha"].view(np.uint32) & 0xFFFF) != 0)   # alpha stays fp32


def test_decay_distribution_matches_recipe():
    wl = synth.Workload("a", 4, 4, 512, 64, 8, "bf16", 1.0, seed=12)
    a = synth.make_inputs(wl)["alpha"].astype(np.float64)
    # alpha = exp(-softplus(x)), x ~ N(1, 1): the median is exp(-softplus(1)) ~ 0.2725
    assert abs(np.median(a) - np.exp(-np.logaddexp(0, 1.0))) < 0.01
    assert a.min() > 0 and a.max() <= 1
