"""Benchmark of the GDN-2 recurrence hot path on B200: one step = one chunkwise prefill
over the 1.3B-scale layer workload (B=8, H=16, T=4096, d_k=d_v=128, bf16 tokens, fp32
alpha and state, C=64) plus one batched decode step (B=256, H=16, d=128, 256 MiB fp32
state updated in place).  Prints one JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torchrun, one rank per GPU; every rank runs the same per-GPU workload
on its own seeded shard (independent chains, no data-path collective: weak scaling).
The only collectives are the barrier and the max-over-ranks of the device time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "tokens/s GDN-2 chunk fwd (B8 H16 T4k d128) + decode; % tensor/HBM roofline"
PATH_NAMES = {0: "simt", 1: "tcgen05 fused", 2: "tcgen05 two-stage (prep_kernel + walk_kernel)"}
PREFILL = "prefill_1p3b"
DECODE = "decode_b256"


# ----------------------------------------------------------------------------- work accounting

def prefill_bytes(B, T, H, K, V, tok_bytes=2, s0=False):
    """Algorithmic HBM bytes of one prefill call: every input read once, every output
    written once (q, k, b: d_k; v, w: d_v in the token dtype; alpha fp32; o; S_T; S0)."""
    per_token_head = (3 * K + 2 * V) * tok_bytes + 4 * K + V * tok_bytes
    state = 4 * B * H * K * V
    return B * T * H * per_token_head + state * (2 if s0 else 1)


def prefill_flops(B, T, H, K, V, C=64):
    """Chunked-algorithm flops: intra-chunk Gram matrices and WY factors (2*C*(2K) + 2*C*(K+V)
    per token-head... counted as the tensor-core products), inter-chunk products and the
    C x C triangular inverse."""
    per_chunk = (2 * C * C * K * 2          # A and P
                 + 2 * C * C * (K + V)      # W = T E+, U~ = T U
                 + 2 * C * K * V * 3        # W S, Q+ S, K^T Delta
                 + 2 * C * C * V            # P Delta
                 + C ** 3 // 3)             # (I + A)^-1
    n_chunks = B * H * ((T + C - 1) // C)
    return n_chunks * per_chunk


def backward_flops(B, T, H, K, V):
    """fp32 arithmetic of the backward's three passes on the d_k x d_v carried matrix, per
    token-head and state element: pass 1 (decay 1, erase read 2, write 2, S dO 2), pass 2
    (q dO^T 2, G^T k 2, G delta 2, erase 2, decay 1), pass 3 (S ddelta 2, write 2, decay 1): 21."""
    return 21 * B * T * H * K * V


def backward_bytes(B, T, H, K, V, tok_bytes=2):
    """Algorithmic HBM bytes of one backward call: the forward's inputs and dO read once, the six
    fp32 token gradients written once, dS_T read and dS0 written (S0 = 0 in the workload)."""
    per_token_head = (3 * K + 2 * V) * tok_bytes + 4 * K + V * tok_bytes + 4 * (4 * K + 2 * V)
    return B * T * H * per_token_head + 2 * 4 * B * H * K * V


def backward_tc_mma_flops(B, T, H, K, V, C=64):
    """Flops of the tensor-core products the tensor-core backward issues per chunk-head (its M = 128
    tiles included): the forward replay (G1, G2, G3, G4, G5), the reverse walk (dDelta^T = dO^T P +
    G^T K^T, dY += [-W'; Q]^T [dDelta; dO]) and the gradient kernel (T^T dDelta, [dA; dP], [dE; dQ],
    dK)."""
    m = 128
    replay = 2 * m * C * K + 2 * 2 * m * V * C + 2 * m * V * K + 2 * 2 * m * V * C
    rwalk = 2 * m * C * C + 2 * m * C * K + 2 * m * V * 2 * C
    grad = 2 * m * V * C + 2 * m * C * V + 2 * m * K * V + 2 * m * K * C + 2 * m * K * V + 2 * 2 * m * K * C
    return B * H * ((T + C - 1) // C) * (replay + rwalk + grad)


def fp32_alu_peak_tflops(n_sm, sm_mhz):
    """Dense fp32 FMA peak from unit counts and clock: 128 fp32 lanes per SM, 2 flops per FMA."""
    return n_sm * 128 * 2 * sm_mhz * 1e6 / 1e12


def decode_bytes(B, H, K, V, tok_bytes=2):
    state = 4 * B * H * K * V
    return 2 * state + B * H * ((3 * K + 2 * V) * tok_bytes + 4 * K + V * tok_bytes)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]), "src": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "src": "fallback"}


def kernel_source_sha(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_key):
    """DRAM bytes per launch from a committed ncu capture, if the kernel is unchanged since."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[kernel_key]
        if kernel_source_sha(rec["sources"]) != rec["sources_sha"]:
            return None
        return float(rec["dram_bytes_per_launch"])
    except Exception:
        return None


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None
        self.out = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
                self.proc.wait(timeout=5)
        if self.out is not None:
            self.out.close()

    def summary(self):
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 9:
                        rows.append(parts)
        except Exception:
            pass
        finally:
            try:
                os.unlink(self.path)
            except Exception:
                pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        pw = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows), "power_w_max": max(pw) if pw else None}


# ----------------------------------------------------------------------------- distributed plumbing

def dist_setup(n_gpus):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}: launch N>1 with torchrun")
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        pg = dist
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local, pg


def barrier(pg):
    if pg is not None:
        pg.barrier()


def max_over_ranks(x, pg, device):
    """Max of a float over ranks (the only reduction: timing)."""
    if pg is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x, pg, device):
    if pg is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.SUM)
    return float(t.item())


def rank_workload(name, rank):
    """Per-rank shard: same shapes, its own seed (independent chains)."""
    import synth
    wl = synth.WORKLOADS[name]
    if rank == 0:
        return wl
    fields = {f: getattr(wl, f) for f in wl.__dataclass_fields__}
    fields["seed"] = wl.seed + 0x10000 * rank
    return synth.Workload(**fields)


# ----------------------------------------------------------------------------- oracle (CPU) timing

def oracle_sample_time(prefill_wl, decode_wl, budget_s=12.0, max_chains=None):
    """Time the fp64 oracle as it stands on a bounded sample of the step's work.

    Prefill: whole (b, h) chains of the prefill workload (full T), as many as fit the
    budget (at least 2*cores, capped by the workload); decode: one decode step of a
    slice of the heads.  Returns a dict: the seconds actually measured, the work share
    of one full step that the sample covers, the seconds of a FULL step extrapolated by
    that share, a description and the threads used."""
    import numpy as np

    import oracle
    import synth
    cores = os.cpu_count() or 1
    B, H, T = prefill_wl.B, prefill_wl.H, prefill_wl.T
    all_chains = [(b, h) for b in range(B) for h in range(H)]
    n = min(len(all_chains), max(2 * cores, 4)) if max_chains is None else min(max_chains, len(all_chains))
    chains = all_chains[:n]
    x = synth.as_f64(synth.make_inputs(prefill_wl, chains=chains))
    S0 = synth.make_state(prefill_wl, chains=chains)
    t0 = time.perf_counter()
    oracle.chain_recurrence(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], S0, threads=cores)
    t_pre = time.perf_counter() - t0
    # grow the sample while well under budget (more chains give a steadier rate)
    if max_chains is None and t_pre < budget_s / 4 and n < len(all_chains):
        n2 = min(len(all_chains), int(n * max(2.0, (budget_s / 2) / max(t_pre, 1e-3))))
        chains = all_chains[:n2]
        x = synth.as_f64(synth.make_inputs(prefill_wl, chains=chains))
        S0 = synth.make_state(prefill_wl, chains=chains)
        t0 = time.perf_counter()
        oracle.chain_recurrence(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], S0, threads=cores)
        t_pre = time.perf_counter() - t0
        n = n2
    full_pre = t_pre * len(all_chains) / n
    # decode: one step over a slice of the heads
    heads = [(b, h) for b in range(min(decode_wl.B, 64)) for h in range(decode_wl.H)]
    xd = synth.as_f64(synth.make_inputs(decode_wl, chains=heads, step=0))
    S = synth.make_state(decode_wl, chains=heads).astype(np.float64).reshape(len(heads), 1, decode_wl.K,
                                                                              decode_wl.V)
    t0 = time.perf_counter()
    oracle.decode_step(*(xd[k][:, None] for k in ("q", "k", "v", "alpha", "b", "w")), S, threads=cores)
    t_dec = time.perf_counter() - t0
    full_dec = t_dec * (decode_wl.B * decode_wl.H) / len(heads)
    desc = (f"fp64 oracle on {n} of {len(all_chains)} prefill chains (full T={T}) and one decode step of "
            f"{len(heads)} of {decode_wl.B * decode_wl.H} heads")
    # tokens of the metric covered by the sample: a chain is 1/H of a prefill token row, a decode
    # head 1/H of a decode token
    tokens = n * T / H + len(heads) / decode_wl.H
    return {"measured_s": t_pre + t_dec, "tokens": tokens, "full_step_s": full_pre + full_dec, "desc": desc,
            "cores": cores}


def bench_config(world):
    """The workload description both arms print (per GPU sizes are fixed: weak scaling)."""
    import synth
    pw, dw = synth.WORKLOADS[PREFILL], synth.WORKLOADS[DECODE]
    return {"workload": f"{PREFILL} (B8 H16 T4096 d_k=d_v=128, C=64, bf16 tokens, fp32 alpha/state) + "
                        f"{DECODE} (B256 H16 d128 decode step, 256 MiB fp32 state in place)",
            "per_gpu": {"prefill": [pw.B, pw.T, pw.H, pw.K, pw.V], "decode": [dw.B, dw.H, dw.K, dw.V]},
            "global_batch": {"prefill": pw.B * world, "decode": dw.B * world},
            "l2": "inputs larger than L2 (1.09 GB prefill inputs, 256 MiB decode state); no flush",
            "parallelism": f"replicas x{world} (independent chains, no collective)"}


# ----------------------------------------------------------------------------- reference arm

def run_reference(args):
    """The oracle arm: each step times the fp64 oracle on a bounded sample of the step's work
    (whole prefill chains and a slice of the decode heads).  `ms_per_step` is the time of the
    sampled work actually run; `value` is the tokens that sample covers per second; the time a
    full step would take at that rate is reported on its own under `full_step_ms_extrapolated`."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import synth
    pw, dw = synth.WORKLOADS[PREFILL], synth.WORKLOADS[DECODE]
    cores = os.cpu_count() or 1
    meas, toks, full, desc = [], [], [], ""
    for i in range(args.warmup + args.steps):
        r = oracle_sample_time(pw, dw, budget_s=4.0, max_chains=max(2, cores))
        desc, cores = r["desc"], r["cores"]
        if i >= args.warmup:
            meas.append(r["measured_s"])
            toks.append(r["tokens"])
            full.append(r["full_step_s"])
    sec = statistics.mean(meas)
    value = sum(toks) / sum(meas)
    out = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(args.gpus),
        "full_step_ms_extrapolated": statistics.mean(full) * 1e3,
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": desc + " per step; ms_per_step is that sample's time"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(out), flush=True)
    return 0


# ----------------------------------------------------------------------------- tensor-core phases

def tensor_phase_probe(g, torch, dev, stream, peak_tflops, reps=(4000, 1500)):
    """The prefill's tensor-core products of one chunk (G1, G2, G3, G4/G5 with the kernels' shapes and
    shared-memory operand layouts), run alone on every SM: mode 0 back to back (the tensor pipe's rate
    on these GEMM phases), mode 1 each group waiting for the one before (the prefill's dependency
    order).  Event-timed; fractions of the measured bf16 peak."""
    nsm = torch.cuda.get_device_properties(dev).multi_processor_count
    ws = g.new_workspace(256, dev)
    out = {"kernel": "phase_kernel", "ctas": nsm, "flops_per_chunk": g.PHASE_PROBE_FLOPS_PER_CHUNK,
           "peak": peak_tflops, "unit": "TFLOP/s"}
    for mode, r in zip((0, 1), reps):
        g.gdn2_gemm_phase_probe(mode, 50, nsm, ws, stream=stream)
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        g.gdn2_gemm_phase_probe(mode, r, nsm, ws, stream=stream)
        b.record(stream)
        torch.cuda.synchronize(dev)
        ms = a.elapsed_time(b)
        tf = r * nsm * g.PHASE_PROBE_FLOPS_PER_CHUNK / (ms * 1e-3) / 1e12
        key = "back_to_back" if mode == 0 else "dependent"
        out[key] = {"chunks_per_cta": r, "ms": ms, "achieved": tf, "frac": tf / peak_tflops}
    if g.gdn2_workspace_status(ws) != 0:
        raise RuntimeError("phase probe reported an expired wait")
    return out


# ----------------------------------------------------------------------------- our arm

def run_ours(args):
    import torch

    import gated_delta_rule_96_b200 as g
    import synth

    rank, world, local, pg = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    g.load_library()
    pw, dw = rank_workload(PREFILL, rank), rank_workload(DECODE, rank)
    if args.prefill_shape:   # profiling aid: another prefill size (not a bench line)
        Bp, Hp, Tp = (int(x) for x in args.prefill_shape.split(","))
        fields = {f: getattr(pw, f) for f in pw.__dataclass_fields__}
        fields.update(B=Bp, H=Hp, T=Tp)
        pw = synth.Workload(**fields)

    def dev_tokens(x, dtype):
        out = {}
        for k, a in x.items():
            t = torch.from_numpy(a).to(dev)
            out[k] = t if k == "alpha" else t.to(dtype)
        return out

    # ---- inputs resident in HBM
    xp = synth.make_inputs(pw)
    P = dev_tokens(xp, torch.bfloat16)
    B, T, H, K = P["q"].shape
    V = P["v"].shape[-1]
    o_p = torch.empty((B, T, H, V), dtype=torch.bfloat16, device=dev)
    S_T = torch.empty((B, H, K, V), dtype=torch.float32, device=dev)
    ws_bytes = g.gdn2_chunk_fwd_workspace_bytes(B, H, T, K, V, 64, g.GDN2_BF16)
    ws = g.new_workspace(ws_bytes, dev)
    path = g.gdn2_chunk_fwd_path(B, H, T, K, V, 64, g.GDN2_BF16)
    xd = synth.make_inputs(dw, step=0)
    D = dev_tokens(xd, torch.bfloat16)
    S_dec = torch.from_numpy(synth.make_state(dw)).to(dev)
    o_d = torch.empty((dw.B, dw.H, dw.V), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    parts = set(args.parts.split(","))
    if "backward_tc" in parts:   # profiling aid: the tensor-core backward on the prefill workload
        dO_np, dST_np = synth.make_output_grads(pw)
        BW = {"dO": torch.from_numpy(dO_np).to(dev).to(torch.bfloat16), "dST": torch.from_numpy(dST_np).to(dev),
              "dS0": torch.empty((B, H, K, V), dtype=torch.float32, device=dev),
              "ws": g.new_workspace(g.gdn2_chunk_bwd_tc_workspace_bytes(B, H, T, K, V), dev)}
        for n in ("dq", "dk", "dv", "dalpha", "db", "dw"):
            BW[n] = torch.empty((B, T, H, K), dtype=torch.float32, device=dev)
        del dO_np, dST_np

    def backward_tc():
        if "backward_tc" not in parts:
            return
        g.gdn2_chunk_bwd_tc(P["q"], P["k"], P["v"], P["alpha"], P["b"], P["w"], None, BW["dO"], BW["dST"], BW["dq"],
                            BW["dk"], BW["dv"], BW["dalpha"], BW["db"], BW["dw"], BW["dS0"], workspace=BW["ws"],
                            stream=stream)

    def prefill():
        if "prefill" not in parts:
            return
        g.gdn2_chunk_fwd(P["q"], P["k"], P["v"], P["alpha"], P["b"], P["w"], None, o_p, S_T, workspace=ws,
                         stream=stream)

    def decode():
        if "decode" not in parts:
            return
        g.gdn2_decode_step(D["q"], D["k"], D["v"], D["alpha"], D["b"], D["w"], S_dec, o_d, stream=stream)

    for _ in range(args.warmup):
        prefill()
        decode()
        backward_tc()
    torch.cuda.synchronize(dev)
    if "backward_tc" in parts and g.gdn2_workspace_status(BW["ws"]) != 0:
        raise SystemExit("backward kernels reported an internal error during warm-up")
    if g.gdn2_workspace_status(ws) != 0:
        raise SystemExit("prefill kernel reported an internal error during warm-up")

    ev = lambda: torch.cuda.Event(enable_timing=True)
    marks = [(ev(), ev(), ev()) for _ in range(args.steps)]
    start, stop = ev(), ev()
    barrier(pg)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        start.record(stream)
        for (a, b_, c) in marks:
            a.record(stream)
            prefill()
            b_.record(stream)
            decode()
            c.record(stream)
            backward_tc()
        stop.record(stream)
        torch.cuda.synchronize(dev)
    barrier(pg)
    clocks = clk.summary()
    if g.gdn2_workspace_status(ws) != 0:
        raise SystemExit("prefill kernel reported an internal error in the timed region")
    total_ms = start.elapsed_time(stop)
    pre_ms = statistics.mean(a.elapsed_time(b_) for a, b_, _ in marks)
    dec_ms = statistics.mean(b_.elapsed_time(c) for _, b_, c in marks)
    total_ms = max_over_ranks(total_ms, pg, dev)
    pre_ms_max = max_over_ranks(pre_ms, pg, dev)
    dec_ms_max = max_over_ranks(dec_ms, pg, dev)

    tokens_rank = B * T + dw.B
    tokens_all = sum_over_ranks(tokens_rank, pg, dev)
    ms_per_step = total_ms / args.steps
    value = tokens_all / (ms_per_step * 1e-3)

    # ---- steady state: the same step back to back for >= 1.5 s, clocks sampled throughout
    steady = None
    if args.steady_s > 0:
        n_steady = max(args.steps, int(args.steady_s * 1e3 / max(ms_per_step, 1e-3)) + 1)
        s0_, s1_ = ev(), ev()
        barrier(pg)
        torch.cuda.synchronize(dev)
        with ClockSampler(local) as clk2:
            s0_.record(stream)
            for _ in range(n_steady):
                prefill()
                decode()
            s1_.record(stream)
            torch.cuda.synchronize(dev)
        barrier(pg)
        st_ms = max_over_ranks(s0_.elapsed_time(s1_), pg, dev) / n_steady
        steady = {"steps": n_steady, "ms_per_step": st_ms, "value": tokens_all / (st_ms * 1e-3),
                  "timed_s": st_ms * n_steady * 1e-3, "clocks": clk2.summary()}
        if g.gdn2_workspace_status(ws) != 0:
            raise SystemExit("prefill kernel reported an internal error in the steady-state region")

    peaks = load_peaks()
    pb = prefill_bytes(B, T, H, K, V)
    db = decode_bytes(dw.B, dw.H, dw.K, dw.V)
    pre_gbs = pb / (pre_ms * 1e-3) / 1e9
    dec_gbs = db / (dec_ms * 1e-3) / 1e9
    pflops = prefill_flops(B, T, H, K, V)
    pre_kernel_key = {2: "prefill_two_stage", 1: "prefill_tc"}.get(path, "prefill_simt")
    tr_pre = recorded_traffic(pre_kernel_key)
    tr_dec = recorded_traffic("decode")
    roof_pre = {"bound": "hbm", "achieved": pre_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": pre_gbs / peaks["hbm_gbs"], "traffic": tr_pre, "peak_src": peaks["src"],
                "kernel": pre_kernel_key, "algorithmic_bytes_per_launch": pb,
                "tensor_tflops": pflops / (pre_ms * 1e-3) / 1e12}
    roof_dec = {"bound": "hbm", "achieved": dec_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": dec_gbs / peaks["hbm_gbs"], "traffic": tr_dec, "peak_src": peaks["src"],
                "kernel": "decode", "algorithmic_bytes_per_launch": db}

    # ---- the tensor pipe on the prefill's GEMM phases (outside the timed region)
    try:
        tp = tensor_phase_probe(g, torch, dev, stream, peaks["bf16_tflops"])
        roof_pre["tensor_phase_frac"] = tp["back_to_back"]["frac"]
        roof_pre["tensor_phase_dependent_frac"] = tp["dependent"]["frac"]
        roof_pre["tensor_phase"] = tp
    except Exception as e:   # a measurement aid: never lose the step's line over it
        roof_pre["tensor_phase"] = {"unavailable": repr(e)[:200]}

    # ---- end to end through the public API: pinned host inputs -> device -> results -> host.
    # Every step copies its inputs in from pinned host memory and its results (o, S_T, the decode o)
    # out to pinned host memory.  Measured twice: serially on one stream, and pipelined over three
    # streams with two device buffer sets, so that step i+1's inputs cross PCIe while step i computes
    # and step i-1's results cross the other way (the link is full duplex).
    host = {k: v.to("cpu").pin_memory() for k, v in P.items()}
    host_d = {k: v.to("cpu").pin_memory() for k, v in D.items()}
    o_h = torch.empty(o_p.shape, dtype=o_p.dtype).pin_memory()
    S_h = torch.empty(S_T.shape, dtype=S_T.dtype).pin_memory()
    od_h = torch.empty(o_d.shape, dtype=o_d.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values()) + \
        sum(t.numel() * t.element_size() for t in host_d.values())
    d2h = o_h.numel() * o_h.element_size() + S_h.numel() * S_h.element_size() + od_h.numel() * od_h.element_size()
    e2e_steps = max(2, min(args.steps, 8))
    do_pre, do_dec = "prefill" in parts, "decode" in parts
    sets = [{"P": P, "D": D, "o": o_p, "S": S_T, "od": o_d},
            {"P": {k: torch.empty_like(v) for k, v in P.items()}, "D": {k: torch.empty_like(v) for k, v in D.items()},
             "o": torch.empty_like(o_p), "S": torch.empty_like(S_T), "od": torch.empty_like(o_d)}]

    def copy_in(bs):
        for k2 in P:
            bs["P"][k2].copy_(host[k2], non_blocking=True)
        for k2 in D:
            bs["D"][k2].copy_(host_d[k2], non_blocking=True)

    def compute(bs):
        if do_pre:
            g.gdn2_chunk_fwd(bs["P"]["q"], bs["P"]["k"], bs["P"]["v"], bs["P"]["alpha"], bs["P"]["b"], bs["P"]["w"],
                             None, bs["o"], bs["S"], workspace=ws, stream=stream)
        if do_dec:
            g.gdn2_decode_step(bs["D"]["q"], bs["D"]["k"], bs["D"]["v"], bs["D"]["alpha"], bs["D"]["b"], bs["D"]["w"],
                               S_dec, bs["od"], stream=stream)

    def copy_out(bs):
        o_h.copy_(bs["o"], non_blocking=True)
        S_h.copy_(bs["S"], non_blocking=True)
        od_h.copy_(bs["od"], non_blocking=True)

    def serial_steps(n):
        for _ in range(n):
            copy_in(sets[0])
            compute(sets[0])
            copy_out(sets[0])

    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def pipelined_steps(n, start_ev):
        s_in.wait_event(start_ev)
        for i in range(n):
            j, bs = i % 2, sets[i % 2]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_done[j])   # step i-2 has finished reading this set's inputs
                copy_in(bs)
                ev_in[j].record(s_in)
            stream.wait_event(ev_in[j])
            if i >= 2:
                stream.wait_event(ev_out[j])      # step i-2's results in this set are copied out
            compute(bs)
            ev_done[j].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[j])
                copy_out(bs)
                ev_out[j].record(s_out)
        stream.wait_event(ev_out[(n - 1) % 2])    # the last results are on the host

    def timed(fn):
        torch.cuda.synchronize(dev)
        barrier(pg)
        e0, e1 = ev(), ev()
        e0.record(stream)
        fn(e0)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return max_over_ranks(e0.elapsed_time(e1) / e2e_steps, pg, dev)

    serial_steps(1)
    warm = torch.cuda.Event()
    warm.record(stream)
    pipelined_steps(2, warm)
    torch.cuda.synchronize(dev)
    e2e_serial_ms = timed(lambda e0: serial_steps(e2e_steps))
    e2e_ms = timed(lambda e0: pipelined_steps(e2e_steps, e0))
    e2e_value = tokens_all / (e2e_ms * 1e-3)
    del sets[1]

    extras = None
    if not (args.no_extras or world > 1):
        try:   # timed after the step's region: a failure here must not cost the step's line
            extras = run_next_rows(g, torch, dev, stream, pw, pre_ms, clocks, with_cpu=not args.no_cpu_baseline)
        except Exception as e:
            extras = {"unavailable": repr(e)[:200]}

    launches_per_step = (1 if path == 1 else 2 * max(1, -(-((T + 63) // 64) // 64)) if path == 2 else 2) + 1
    out = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": bench_config(world),
        "roofline": roof_pre,
        "parts": {"prefill": {"ms": pre_ms_max, "tokens_per_s": B * T * world / (pre_ms_max * 1e-3),
                              "path": PATH_NAMES.get(path, "simt"), "roofline": roof_pre},
                  "decode": {"ms": dec_ms_max, "tokens_per_s": dw.B * world / (dec_ms_max * 1e-3),
                             "roofline": roof_dec}},
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps, "pipelined": True, "ms_per_step": e2e_ms,
                "serial": {"value": tokens_all / (e2e_serial_ms * 1e-3), "ms_per_step": e2e_serial_ms}},
        "clocks": clocks,
        "gpu_launches": launches_per_step * args.steps,
    }
    if steady is not None:
        out["steady"] = steady
    if extras is not None:
        out["next_rows"] = extras
    if parts != {"prefill", "decode"}:
        out["config"]["parts_only"] = sorted(parts)   # profiling run: not a bench line
    if args.prefill_shape:
        out["config"]["prefill_shape"] = args.prefill_shape   # profiling run: not a bench line
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        r = oracle_sample_time(pw, dw)
        out["cpu_baseline"] = {"value": r["tokens"] / r["measured_s"], "unit": "tokens/s", "cores": r["cores"],
                               "kind": "oracle", "sample": r["desc"] + f" ({r['measured_s']:.1f} s)"}
    if rank == 0:
        print(json.dumps(out), flush=True)
    if pg is not None:
        pg.destroy_process_group()
    return 0


def oracle_next_rows_sample(wl):
    """The fp64 oracles of the rows beyond the step, timed on one (b, h) chain of the workload with
    one thread: the backward (the C oracle's gdn2_oracle_backward) and the edge maps plus the
    recurrence.  Returns
    {"backward": ..., "edges_prefill": ...} in tokens/s of the whole workload (B*T tokens over its
    B*H chains run one after another)."""
    import numpy as np
    import threadpoolctl

    import oracle
    import synth
    chain = [(0, 0)]
    scale = lambda sec: wl.B * wl.T / (sec * wl.B * wl.H)
    x = {k: v[0].astype("float64") for k, v in synth.make_inputs(wl, chains=chain).items()}
    dO, dST = synth.make_output_grads(wl, chains=chain)
    r4 = lambda a: a.reshape(1, a.shape[0], 1, a.shape[-1])   # one chain as [B=1, T, H=1, d]
    with threadpoolctl.threadpool_limits(1):
        t0 = time.perf_counter()
        oracle.recurrence_backward_c(*(r4(x[n]) for n in ("q", "k", "v", "alpha", "b", "w")), None,
                                     r4(dO[0].astype("float64")), dST[0].astype("float64")[None, None], threads=1)
        t_bwd = time.perf_counter() - t0
        r = {k: v[0].astype("float64") for k, v in synth.make_raw_inputs(wl, chains=chain).items()}
        t0 = time.perf_counter()
        q, k, alpha, b, w = oracle.layer_edges(r["q"], r["k"], r["a"], r["b"], r["w"])
        o, _ = oracle.chain_recurrence(q[None], k[None], r["v"][None], alpha[None], b[None], w[None], threads=1)
        oracle.rms_norm(o, np.ones(wl.V))
        t_edges = time.perf_counter() - t0
    desc = f"one chain (b=0, h=0, T={wl.T}) of the {wl.B * wl.H}, one thread, scaled by the chain count"
    return {"backward": {"value": scale(t_bwd), "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": desc},
            "edges_prefill": {"value": scale(t_edges), "unit": "tokens/s", "cores": 1, "kind": "oracle",
                              "sample": desc}}


def long_prefill_row(g, torch, dev, stream, timed, with_cpu):
    """The prefill of few long chains (B1 H16 T65536, S0 given): segments in time, their state maps
    composed along each chain (the transition scan), then every segment rerun from its start state."""
    import numpy as np
    import threadpoolctl

    import oracle
    import synth
    lw = synth.WORKLOADS["prefill_long"]
    x = synth.make_inputs(lw)
    S0_np = synth.make_state(lw)
    X = {k: torch.from_numpy(a).to(dev).to(torch.float32 if k == "alpha" else torch.bfloat16) for k, a in x.items()}
    del x
    S0 = torch.from_numpy(S0_np).to(dev)
    B, T, H, K = X["q"].shape
    V = X["v"].shape[-1]
    o = torch.empty((B, T, H, V), dtype=torch.bfloat16, device=dev)
    S_T = torch.empty((B, H, K, V), device=dev)
    ws = g.new_workspace(g.gdn2_chunk_fwd_workspace_bytes(B, H, T, K, V, 64, g.GDN2_BF16), dev)
    ms = timed(lambda: g.gdn2_chunk_fwd(X["q"], X["k"], X["v"], X["alpha"], X["b"], X["w"], S0, o, S_T,
                                        workspace=ws, stream=stream))
    if g.gdn2_workspace_status(ws) != 0:
        raise RuntimeError("segmented prefill reported an internal error")
    peaks = load_peaks()
    nbytes = prefill_bytes(B, T, H, K, V, s0=True)
    gbs = nbytes / (ms * 1e-3) / 1e9
    row = {"workload": f"{lw.name} (B{B} H{H} T{T} d_k=d_v={K}, bf16 tokens, S0 given)", "ms": ms,
           "tokens_per_s": B * T / (ms * 1e-3), "launches": 5,
           "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": gbs / peaks["hbm_gbs"], "algorithmic_bytes_per_launch": nbytes,
                        "traffic": recorded_traffic("prefill_segmented"), "peak_src": peaks["src"],
                        "note": "prep over every chunk-head, three walks over the segments' records, the "
                                "fp32 scan: the records are read three times"}}
    del X, o, S_T, ws, S0
    if with_cpu:
        try:
            xs = synth.as_f64(synth.make_inputs(lw, chains=[(0, 0)]))
            with threadpoolctl.threadpool_limits(1):
                t0 = time.perf_counter()
                oracle.chain_recurrence(*(xs[k] for k in ("q", "k", "v", "alpha", "b", "w")),
                                        np.asarray(S0_np[0, :1], dtype=np.float64), threads=1)
                sec = time.perf_counter() - t0
            row["cpu_baseline"] = {"value": B * T / (sec * B * H), "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                   "sample": f"one chain (b=0, h=0, T={T}) of the {B * H}, one thread, "
                                             "scaled by the chain count"}
        except Exception as e:
            row["cpu_baseline"] = {"unavailable": repr(e)[:200]}
    return row


def fp32_row_workloads():
    import synth
    return (("tiny_f32", synth.WORKLOADS["tiny_f32"]),
            ("prefill_1p3b_f32", synth.Workload("prefill_1p3b_f32", 8, 16, 4096, 128, 128, "f32", 1.0, seed=0x9D2 + 1)))


def fp32_prefill_rows(g, torch, dev, stream, timed, with_cpu):
    """The CUDA-core prefill (fp32 tokens, or d = 64): the tiny fp32 workload the 1e-4 bar applies to
    (B1 H2 T256 d64) and the 1.3B-scale layer with fp32 tokens (B8 H16 T4096 d128), each against the
    HBM roofline of its algorithmic bytes (fp32 q, k, v, b, w, alpha read once, o and S_T written once)."""
    import numpy as np
    import threadpoolctl

    import oracle
    import synth
    peaks = load_peaks()
    rows = {}
    for name, wl in fp32_row_workloads():
        x = synth.make_inputs(wl)
        X = {k: torch.from_numpy(a).to(dev) for k, a in x.items()}
        B, T, H, K = X["q"].shape
        V = X["v"].shape[-1]
        o = torch.empty((B, T, H, V), device=dev)
        S_T = torch.empty((B, H, K, V), device=dev)
        ws = g.new_workspace(g.gdn2_chunk_fwd_workspace_bytes(B, H, T, K, V, 64, g.GDN2_F32), dev)
        ms = timed(lambda: g.gdn2_chunk_fwd(X["q"], X["k"], X["v"], X["alpha"], X["b"], X["w"], None, o, S_T,
                                            workspace=ws, stream=stream), warm=3, reps=20 if T * B * H < 1e5 else 5)
        nbytes = prefill_bytes(B, T, H, K, V, tok_bytes=4)
        gbs = nbytes / (ms * 1e-3) / 1e9
        row = {"workload": f"{name} (B{B} H{H} T{T} d_k=d_v={K}, fp32 tokens)", "ms": ms,
               "tokens_per_s": B * T / (ms * 1e-3), "launches": 2, "path": "simt",
               "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                            "frac": gbs / peaks["hbm_gbs"], "algorithmic_bytes_per_launch": nbytes,
                            "traffic": None, "peak_src": peaks["src"]}}
        del X, o, S_T, ws
        if with_cpu:
            xs = synth.as_f64(synth.make_inputs(wl, chains=[(0, 0)]))
            with threadpoolctl.threadpool_limits(1):
                t0 = time.perf_counter()
                oracle.chain_recurrence(*(xs[k] for k in ("q", "k", "v", "alpha", "b", "w")), None, threads=1)
                sec = time.perf_counter() - t0
            row["cpu_baseline"] = {"value": B * T / (sec * B * H), "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                   "sample": f"one chain (b=0, h=0, T={T}) of the {B * H}, one thread, scaled by the "
                                             "chain count"}
        rows[name] = row
    return rows


def run_next_rows(g, torch, dev, stream, wl, plain_prefill_ms, clocks, with_cpu=True):
    """Timings of the rows beyond the step (not part of `value`): the backward pass of the
    prefill workload and the prefill with the layer edges fused, both on that workload's sizes."""
    import synth

    def timed(fn, warm=2, reps=5):
        for _ in range(warm):
            fn()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / reps

    x = synth.make_inputs(wl)
    B, T, H, K, V = wl.B, wl.T, wl.H, wl.K, wl.V
    to = lambda a, dt: torch.from_numpy(a).to(dev).to(dt)
    X = {k: to(a, torch.float32 if k == "alpha" else torch.bfloat16) for k, a in x.items()}
    dO_np, dST_np = synth.make_output_grads(wl)
    dO, dST = to(dO_np, torch.bfloat16), to(dST_np, torch.float32)
    del x, dO_np, dST_np
    grads = {n: torch.empty((B, T, H, K if n in ("dq", "dk", "dalpha", "db") else V), device=dev)
             for n in ("dq", "dk", "dv", "dalpha", "db", "dw")}
    dS0 = torch.empty((B, H, K, V), device=dev)
    wsb = g.new_workspace(g.gdn2_chunk_bwd_workspace_bytes(B, H, T, K, V), dev)
    bwd_ms = timed(lambda: g.gdn2_chunk_bwd(X["q"], X["k"], X["v"], X["alpha"], X["b"], X["w"], None, dO, dST,
                                            grads["dq"], grads["dk"], grads["dv"], grads["dalpha"], grads["db"],
                                            grads["dw"], dS0, workspace=wsb, stream=stream))
    wst = g.new_workspace(g.gdn2_chunk_bwd_tc_workspace_bytes(B, H, T, K, V), dev)
    bwd_tc_ms = timed(lambda: g.gdn2_chunk_bwd_tc(X["q"], X["k"], X["v"], X["alpha"], X["b"], X["w"], None, dO,
                                                  dST, grads["dq"], grads["dk"], grads["dv"], grads["dalpha"],
                                                  grads["db"], grads["dw"], dS0, workspace=wst, stream=stream))
    if g.gdn2_workspace_status(wst) != 0:
        raise RuntimeError("tensor-core backward reported an internal error")
    del grads, dS0, wsb, wst, X, dO, dST
    peaks = load_peaks()
    hbm = peaks["hbm_gbs"]
    tc_bytes = backward_bytes(B, T, H, K, V)
    tc_gbs = tc_bytes / (bwd_tc_ms * 1e-3) / 1e9
    backward_tc = {"ms": bwd_tc_ms, "tokens_per_s": B * T / (bwd_tc_ms * 1e-3), "launches": 4,
                   "kernels": "prep_kernel + walk_kernel (forward replay), rwalk_kernel, grad_kernel",
                   "roofline": {"bound": "hbm", "achieved": tc_gbs, "peak": hbm, "unit": "GB/s",
                                "frac": tc_gbs / hbm, "algorithmic_bytes_per_launch": tc_bytes,
                                "traffic": recorded_traffic("backward_tc"),
                                "peak_src": peaks["src"],
                                "tensor_tflops": backward_tc_mma_flops(B, T, H, K, V) / (bwd_tc_ms * 1e-3) / 1e12}}
    n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
    sm_mhz = (clocks or {}).get("sm_max_mhz") or 1965.0
    peak = fp32_alu_peak_tflops(n_sm, sm_mhz)
    flops = backward_flops(B, T, H, K, V)
    achieved = flops / (bwd_ms * 1e-3) / 1e12
    backward = {"ms": bwd_ms, "tokens_per_s": B * T / (bwd_ms * 1e-3), "launches": 3,
                "roofline": {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                             "frac": achieved / peak, "flops_per_launch": flops,
                             "traffic": recorded_traffic("backward"),
                             "peak_src": f"derived: {n_sm} SMs x 128 fp32 lanes x 2 flops x {sm_mhz:.0f} MHz"}}

    r = synth.make_raw_inputs(wl)
    R = {k: to(a, torch.float32 if k == "a" else torch.bfloat16) for k, a in r.items()}
    del r
    o = torch.empty((B, T, H, V), dtype=torch.bfloat16, device=dev)
    S_T = torch.empty((B, H, K, V), device=dev)
    weight = torch.ones(V, device=dev)
    ws = g.new_workspace(g.gdn2_chunk_fwd_edges_workspace_bytes(B, H, T, K, V), dev)
    edge_ms = timed(lambda: g.gdn2_chunk_fwd_edges(R["q"], R["k"], R["v"], R["a"], R["b"], R["w"], None, weight, o,
                                                   S_T, workspace=ws, stream=stream))
    if g.gdn2_workspace_status(ws) != 0:
        raise RuntimeError("edge prefill kernel reported an internal error")
    # the unfused layer on the same inputs: the map kernel, the plain prefill, RMSNorm
    M = {"q": torch.empty_like(R["q"]), "k": torch.empty_like(R["k"]), "b": torch.empty_like(R["b"]),
         "w": torch.empty_like(R["w"]), "alpha": torch.empty_like(R["a"])}
    ws2 = g.new_workspace(g.gdn2_chunk_fwd_workspace_bytes(B, H, T, K, V, 64, g.GDN2_BF16), dev)

    def unfused():
        g.gdn2_layer_edge_maps(R["q"], R["k"], R["a"], R["b"], R["w"], M["q"], M["k"], M["alpha"], M["b"], M["w"],
                               stream=stream)
        g.gdn2_chunk_fwd(M["q"], M["k"], R["v"], M["alpha"], M["b"], M["w"], None, o, S_T, workspace=ws2,
                         stream=stream)
        g.gdn2_rms_norm(o, weight, stream=stream)

    unfused_ms = timed(unfused)
    del M, ws2
    edges = {"ms": edge_ms, "tokens_per_s": B * T / (edge_ms * 1e-3), "launches": 2, "rmsnorm": True,
             "unfused_ms": unfused_ms,
             "unfused": "gdn2_layer_edge_maps + gdn2_chunk_fwd + gdn2_rms_norm on the same inputs",
             "plain_prefill_ms": plain_prefill_ms,
             "inputs": "raw q, k ~ N(0, 9), decay logit ~ N(1, 1) (alpha = exp(-softplus(a)): the plain "
                       "workload's alpha distribution), gate logits ~ N(0, 1)"}
    out = {"workload": f"{wl.name} (B{B} H{H} T{T} d_k=d_v={K}, bf16 tokens)", "backward": backward,
           "backward_tc": backward_tc, "edges_prefill": edges}
    if with_cpu:
        try:
            cpu = oracle_next_rows_sample(wl)
            backward["cpu_baseline"], edges["cpu_baseline"] = cpu["backward"], cpu["edges_prefill"]
            backward_tc["cpu_baseline"] = cpu["backward"]
        except Exception as e:   # the CPU figures are context: never lose the GPU line over them
            backward["cpu_baseline"] = edges["cpu_baseline"] = {"unavailable": repr(e)[:200]}
    try:
        out["segmented_prefill"] = long_prefill_row(g, torch, dev, stream, timed, with_cpu)
    except Exception as e:   # likewise: this row must not cost the step's line
        out["segmented_prefill"] = {"unavailable": repr(e)[:200]}
    try:
        out["fp32_prefill"] = fp32_prefill_rows(g, torch, dev, stream, timed, with_cpu)
    except Exception as e:
        out["fp32_prefill"] = {"unavailable": repr(e)[:200]}
    return out


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing leg")
    ap.add_argument("--no-extras", action="store_true", help="skip the backward / fused-edge timings")
    ap.add_argument("--steady-s", type=float, default=1.5,
                    help="length of the extra back-to-back region reported under 'steady' (0: skip)")
    ap.add_argument("--prefill-shape", default="",
                    help="profiling aid: B,H,T of the prefill instead of the bench workload (not a bench line)")
    ap.add_argument("--parts", default="prefill,decode",
                    help="profiling aid: run only some parts of the step (the default runs the whole step); "
                         "'backward_tc' adds the tensor-core backward on the prefill workload")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
