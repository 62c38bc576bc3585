"""Host-side logic of bench.py: work accounting, the reference (oracle) arm's JSON line,
and the multi-rank plumbing (world size 2 over gloo on the CPU)."""
import json
import os
import socket

import pytest

import bench
from tests.test_binding_host import rec  # noqa: F401  (fixture)


def test_prefill_bytes_per_token_head():
    # q, k, b (3*128) and v, w (2*128) in bf16, alpha fp32, o bf16: 2,048 B per token-head
    B, T, H, K, V = 8, 4096, 16, 128, 128
    assert bench.prefill_bytes(B, T, H, K, V) == B * T * H * 2048 + 4 * B * H * K * V
    assert bench.prefill_bytes(1, 1, 1, K, V, s0=True) - bench.prefill_bytes(1, 1, 1, K, V) == 4 * K * V


def test_decode_bytes():
    # state read + write dominates: 2 x 256 MiB
    b = bench.decode_bytes(256, 16, 128, 128)
    assert b == 2 * 4 * 256 * 16 * 128 * 128 + 256 * 16 * (5 * 128 * 2 + 4 * 128 + 128 * 2)


def test_prefill_flops_positive_and_scaling():
    f1 = bench.prefill_flops(1, 64, 1, 128, 128)
    assert bench.prefill_flops(2, 128, 3, 128, 128) == 12 * f1


def test_peaks_loaded():
    p = bench.load_peaks()
    assert p["hbm_gbs"] > 1000 and p["bf16_tflops"] > 100


def test_reference_arm_json(capsys, monkeypatch):
    monkeypatch.setenv("RANK", "0")
    stub = {"measured_s": 0.5, "tokens": 1000.0, "full_step_s": 2.0, "desc": "stub", "cores": 3}
    monkeypatch.setattr(bench, "oracle_sample_time", lambda pw, dw, budget_s, max_chains: stub)
    assert bench.main(["--impl", "reference", "--steps", "2", "--warmup", "1"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["unit"] == "tokens/s" and line["metric"] == bench.METRIC
    # the sampled work per step is what ms_per_step reports; the rate is its tokens over its time
    assert line["ms_per_step"] == pytest.approx(500.0)
    assert line["value"] == pytest.approx(1000.0 / 0.5)
    assert line["full_step_ms_extrapolated"] == pytest.approx(2000.0)
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["cpu_baseline"]["cores"] == 3


def test_reference_arm_nonzero_rank_is_silent(capsys, monkeypatch):
    monkeypatch.setenv("RANK", "1")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "0"]) == 0
    assert capsys.readouterr().out == ""


def test_oracle_sample_time_small():
    import synth
    pw = synth.Workload("p", 1, 2, 128, 16, 16, "bf16", 1.0, seed=3)
    dw = synth.Workload("d", 4, 2, 1, 16, 16, "bf16", 1.0, s0_std=0.01, seed=4, decode=True)
    r = bench.oracle_sample_time(pw, dw, budget_s=0.5, max_chains=2)
    assert r["measured_s"] > 0 and r["cores"] >= 1 and "oracle" in r["desc"]
    # 2 of 2 chains (T = 128 over H = 2) and 8 decode heads over H = 2
    assert r["tokens"] == pytest.approx(2 * 128 / 2 + 8 / 2)
    assert r["full_step_s"] >= r["measured_s"] * 0.99


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import torch
    torch.cuda.is_available = lambda: False   # force the gloo branch on any box
    r, w, local, pg = bench.dist_setup(world)
    bench.barrier(pg)
    mx = bench.max_over_ranks(float(rank + 1) * 10.0, pg, "cpu")
    sm = bench.sum_over_ranks(float(rank + 1), pg, "cpu")
    seed = bench.rank_workload(bench.PREFILL, rank).seed
    pg.destroy_process_group()
    q.put((r, w, mx, sm, seed))


def test_two_rank_plumbing_gloo():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == [0, 1]
    assert all(r[2] == 20.0 and r[3] == 3.0 for r in res)     # max and sum over ranks
    assert res[0][4] != res[1][4]                              # distinct shards


def test_backward_accounting():
    import bench
    # 21 fp32 flops per state element per token-head across the three passes
    assert bench.backward_flops(8, 4096, 16, 128, 128) == 21 * 8 * 4096 * 16 * 128 * 128 == 180388626432
    # 148 SMs x 128 fp32 lanes x 2 flops x 1965 MHz
    assert abs(bench.fp32_alu_peak_tflops(148, 1965.0) - 74.44992) < 1e-9
    # tensor-core backward: q, k, v, b, w, dO bf16 and alpha fp32 read, six fp32 gradients written (5,120 B
    # per token-head), dS_T read and dS0 written per chain
    assert bench.backward_bytes(1, 1, 1, 128, 128) == 5120 + 2 * 4 * 128 * 128
    assert bench.backward_bytes(8, 4096, 16, 128, 128) == 8 * 4096 * 16 * 5120 + 2 * 4 * 128 * 128 * 128
    assert bench.backward_tc_mma_flops(8, 4096, 16, 128, 128) == 128 * 64 * bench.backward_tc_mma_flops(1, 64, 1, 128, 128)


def test_oracle_next_rows_sample_small():
    import bench
    import synth
    wl = synth.Workload("nr", 2, 3, 96, 64, 64, "bf16", 1.0, seed=5)
    out = bench.oracle_next_rows_sample(wl)
    for key in ("backward", "edges_prefill"):
        r = out[key]
        assert r["kind"] == "oracle" and r["cores"] == 1 and r["unit"] == "tokens/s" and r["value"] > 0


def test_next_rows_run_on_cpu_through_the_binding(rec, monkeypatch):
    """The bench's extra rows (backward, edge-fused prefill, segmented long prefill) driven on the CPU:
    the library's compute calls are recorded instead of launched and CUDA events return 1 ms per 5 timed calls, so the
    host code of each row (tensor shapes, binding arguments, accounting, the oracle baselines) runs
    end to end and every row comes back complete."""
    import types

    import torch

    import bench
    import gated_delta_rule_96_b200 as g
    import synth

    class Event:
        def __init__(self, enable_timing=False):
            pass

        def record(self, stream=None):
            pass

        def elapsed_time(self, other):
            return 1.0

    cuda = types.SimpleNamespace(Event=Event, synchronize=lambda dev=None: None,
                                 get_device_properties=lambda dev: types.SimpleNamespace(multi_processor_count=148))

    class FakeTorch:
        def __getattr__(self, name):
            return cuda if name == "cuda" else getattr(torch, name)

    monkeypatch.setitem(synth.WORKLOADS, "prefill_long",
                        synth.Workload("prefill_long", 1, 2, 200, 128, 128, "bf16", 1.0, s0_std=0.01, seed=7))
    monkeypatch.setattr(bench, "fp32_row_workloads", lambda: (
        ("tiny_f32", synth.WORKLOADS["tiny_f32"]),
        ("prefill_1p3b_f32", synth.Workload("f", 2, 3, 70, 128, 128, "f32", 1.0, seed=9))))
    wl = synth.Workload("nr", 1, 2, 96, 128, 128, "bf16", 1.0, seed=5)
    out = bench.run_next_rows(g, FakeTorch(), "cpu", None, wl, 0.5, {"sm_max_mhz": 1965.0})
    names = [c[0] for c in rec.calls]
    assert names.count("gdn2_chunk_bwd") == 7 and names.count("gdn2_chunk_fwd_edges") == 7
    assert names.count("gdn2_chunk_bwd_tc") == 7
    # segmented row 7; unfused edge layer 7; fp32 rows: tiny 3 + 20, the other 3 + 20 (small here)
    assert names.count("gdn2_chunk_fwd") == 7 + 7 + 23 + 23
    assert names.count("gdn2_layer_edge_maps") == 7 and names.count("gdn2_rms_norm") == 7
    f32 = out["fp32_prefill"]
    assert f32["tiny_f32"]["roofline"]["algorithmic_bytes_per_launch"] == bench.prefill_bytes(1, 256, 2, 64, 64, 4)
    assert f32["tiny_f32"]["cpu_baseline"]["value"] > 0
    bw, ed, sp = out["backward"], out["edges_prefill"], out["segmented_prefill"]
    ms = 1.0 / 5
    assert bw["ms"] == ms and bw["tokens_per_s"] == pytest.approx(96 / (ms * 1e-3))
    assert bw["roofline"]["bound"] == "alu" and bw["roofline"]["flops_per_launch"] == bench.backward_flops(
        1, 96, 2, 128, 128)
    bt = out["backward_tc"]
    assert bt["ms"] == ms and bt["roofline"]["bound"] == "hbm" and bt["launches"] == 4
    assert bt["roofline"]["algorithmic_bytes_per_launch"] == bench.backward_bytes(1, 96, 2, 128, 128)
    assert ed["ms"] == ms and ed["plain_prefill_ms"] == 0.5 and sp["ms"] == ms
    assert sp["roofline"]["algorithmic_bytes_per_launch"] == bench.prefill_bytes(1, 200, 2, 128, 128, s0=True)
    for row in (bw, ed, sp):
        c = row["cpu_baseline"]
        assert "unavailable" not in c and c["kind"] == "oracle" and c["value"] > 0, c


def test_clock_sampler_without_nvidia_smi(monkeypatch):
    """No nvidia-smi (or no GPU): the sampler reports 'unavailable' instead of failing the run."""
    monkeypatch.setenv("PATH", "/nonexistent")
    with bench.ClockSampler(0) as c:
        pass
    s = c.summary()
    assert s["reasons"] == ["unavailable"] and s["samples"] == 0


def test_clock_sampler_summary(tmp_path):
    """Median SM clock under load, the max clock, and the throttle reasons seen Active."""
    p = tmp_path / "clocks.csv"
    p.write_text("0, 1965, 1965, 700.5, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n"
                 "0, 1800, 1965, 1000.1, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n"
                 "0, 1900, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n"
                 "garbage line\n")
    c = bench.ClockSampler(0)
    c.path = str(p)
    s = c.summary()
    assert s["sm_mhz"] == 1900 and s["sm_max_mhz"] == 1965 and s["samples"] == 3
    assert s["reasons"] == ["sw_power_cap"] and s["power_w_max"] == 1000.1
    assert not p.exists()
