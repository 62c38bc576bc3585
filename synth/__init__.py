"""Seeded synthetic inputs for the gated delta-rule recurrence.

This module is shared by the oracle tests, the GPU parity tests and the
benchmark.  It draws numbers and shapes them into the workloads' value
distributions; it contains none of the recurrence's arithmetic.

Recipe (one place, used everywhere):

* every tensor is a counter-based stream of ``synth_gen.c`` keyed by
  ``(seed, stream)``; the flat row-major index of an element in its full
  tensor is its counter, so one (batch, head) chain can be regenerated alone;
* q, k: N(0,1) per element, then L2-normalised over the head dimension per
  (token, head), in fp64;
* v: N(0,1);
* alpha = exp(-softplus(x)), x ~ N(mu, 1) (mu = 0 for the small fp32 case,
  1 for the bf16 workloads), one value per key channel;
* b, w = sigmoid(N(0,1)) per key / value channel ("channel" gates), or one
  beta = sigmoid(N(0,1)) per (token, head) broadcast over the channels
  ("kda"); "gdn" additionally draws alpha once per (token, head);
* S0: N(0, s0_std^2) or absent (zero state);
* values are drawn and shaped in fp64 (in synth_gen.c) and rounded to the
  storage dtype (fp64 -> fp32 -> bf16, each round-to-nearest-even); arrays are
  returned as float32 holding exactly the stored values, and the oracle is fed
  those values widened to fp64.

Token tensors are [B, T, H, d] (d fastest); states are [B, H, d_k, d_v].
Decode tokens are [B, H, d]; decode step s uses streams 16*(s+1) + id.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth_gen.c")
_LIB_PATH = os.path.join(_HERE, "libsynth_gen.so")
_lib = None

STREAM = {"q": 0, "k": 1, "v": 2, "alpha": 3, "b": 4, "w": 5, "S0": 6, "beta": 7, "alpha_s": 8}


def build(force: bool = False) -> str:
    """Compile the generator with gcc (host only)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        u64, sz, dp = ctypes.c_uint64, ctypes.c_size_t, ctypes.POINTER(ctypes.c_double)
        lib.synth_normal.argtypes = [u64, u64, u64, sz, dp]
        lib.synth_uniform.argtypes = [u64, u64, u64, sz, dp]
        lib.synth_normal_mt.argtypes = [u64, u64, u64, sz, dp, ctypes.c_int]
        lib.synth_normal_rows.argtypes = [u64, u64, ctypes.POINTER(ctypes.c_uint64), sz, sz, dp]
        lib.synth_rows.argtypes = [u64, u64, ctypes.c_int, ctypes.c_double, ctypes.c_double,
                                   ctypes.POINTER(ctypes.c_uint64), u64, sz, sz, ctypes.c_int, ctypes.c_int,
                                   ctypes.POINTER(ctypes.c_float), ctypes.c_int]
        lib.synth_rows.restype = ctypes.c_int
        _lib = lib
    return _lib


def _dp(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def normal(seed: int, stream: int, n: int, offset: int = 0, threads: int | None = None) -> np.ndarray:
    lib = _load()
    out = np.empty(n, dtype=np.float64)
    if n:
        nt = threads if threads is not None else min(os.cpu_count() or 1, 32)
        lib.synth_normal_mt(seed, stream, offset, n, _dp(out), nt)
    return out


def uniform(seed: int, stream: int, n: int, offset: int = 0) -> np.ndarray:
    lib = _load()
    out = np.empty(n, dtype=np.float64)
    if n:
        lib.synth_uniform(seed, stream, offset, n, _dp(out))
    return out


def normal_rows(seed: int, stream: int, offsets: np.ndarray, rowlen: int) -> np.ndarray:
    lib = _load()
    offs = np.ascontiguousarray(offsets, dtype=np.uint64)
    out = np.empty((offs.size, rowlen), dtype=np.float64)
    if offs.size:
        lib.synth_normal_rows(seed, stream, offs.ctypes.data_as(ctypes.POINTER(ctypes.c_uint64)),
                              offs.size, rowlen, _dp(out))
    return out


# ----------------------------------------------------------------------------- shaping

KIND_NORMAL, KIND_L2, KIND_SIGMOID, KIND_DECAY = 0, 1, 2, 3


def rows(seed: int, stream: int, kind: int, d: int, row_index=None, nrows: int | None = None, row0: int = 0,
         mu: float = 0.0, scale: float = 1.0, per_token: bool = False, bf16: bool = False,
         threads: int | None = None) -> np.ndarray:
    """Shaped rows ([nrows, d] float32); see synth_rows in synth_gen.c."""
    lib = _load()
    if row_index is not None:
        idx = np.ascontiguousarray(row_index, dtype=np.uint64)
        n = idx.size
        iptr = idx.ctypes.data_as(ctypes.POINTER(ctypes.c_uint64))
    else:
        idx, n, iptr = None, int(nrows), None
    out = np.empty((n, d), dtype=np.float32)
    if n:
        nt = threads if threads is not None else min(os.cpu_count() or 1, 32)
        rc = lib.synth_rows(seed, stream, kind, mu, scale, iptr, row0, n, d, 1 if per_token else 0,
                            1 if bf16 else 0, out.ctypes.data_as(ctypes.POINTER(ctypes.c_float)), nt)
        if rc != 0:
            raise ValueError("synth_rows rejected its arguments")
    return out


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round values to the storage dtype; returned as fp64 (exactly representable)."""
    if dtype == "f64":
        return np.asarray(x, dtype=np.float64)
    x32 = np.asarray(x, dtype=np.float32)
    if dtype == "f32":
        return x32.astype(np.float64)
    if dtype == "bf16":
        u = x32.view(np.uint32).astype(np.uint64)
        lsb = (u >> 16) & 1
        u = (u + 0x7FFF + lsb) & 0xFFFF0000
        return u.astype(np.uint32).view(np.float32).astype(np.float64)
    raise ValueError(dtype)


# ----------------------------------------------------------------------------- workloads

@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    K: int
    V: int
    dtype: str            # storage dtype of q, k, v, b, w and o ("f32" or "bf16")
    alpha_mu: float       # mean of the normal inside the softplus
    gates: str = "channel"   # "channel" | "kda" | "gdn"
    s0_std: float | None = None
    seed: int = 0x9D2
    steps: int = 0        # decode steps (decode workloads only)
    decode: bool = False
    alpha_scale: float = 1.0  # multiplies softplus (slow-decay stress variant uses 0.02)


WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", 1, 2, 256, 64, 64, "f32", 0.0, seed=0x9D2 + 0),
    "prefill_1p3b": Workload("prefill_1p3b", 8, 16, 4096, 128, 128, "bf16", 1.0, seed=0x9D2 + 1),
    "prefill_long": Workload("prefill_long", 1, 16, 65536, 128, 128, "bf16", 1.0, s0_std=0.01,
                             seed=0x9D2 + 2),
    "prefill_kda": Workload("prefill_kda", 8, 16, 4096, 128, 128, "bf16", 1.0, gates="kda",
                            seed=0x9D2 + 3),
    "prefill_gdn": Workload("prefill_gdn", 8, 16, 4096, 128, 128, "bf16", 1.0, gates="gdn",
                            seed=0x9D2 + 3 + 0x100),
    "decode_b256": Workload("decode_b256", 256, 16, 1, 128, 128, "bf16", 1.0, s0_std=0.01,
                            seed=0x9D2 + 4, steps=1000, decode=True),
    "prefill_slow_decay": Workload("prefill_slow_decay", 8, 16, 4096, 128, 128, "bf16", 1.0,
                                   seed=0x9D2 + 5, alpha_scale=0.02),
}


def _row_index(wl: Workload, T_full: int, chains, t0: int, t1: int):
    """Flat (b, t, h) row indices of the requested rows, or None for the full tensor."""
    if chains is None and (t0, t1) == (0, T_full):
        return None
    if chains is None:
        chains = [(b, h) for b in range(wl.B) for h in range(wl.H)]
    t = np.arange(t0, t1, dtype=np.uint64)
    parts = [(np.uint64(b) * np.uint64(T_full) + t) * np.uint64(wl.H) + np.uint64(h) for (b, h) in chains]
    return np.concatenate(parts) if parts else np.zeros(0, dtype=np.uint64)


def make_inputs(wl: Workload, chains=None, t_range=None, step: int | None = None):
    """Inputs of a workload as float32 arrays holding exactly the stored values.

    chains=None gives full tensors ([B,T,H,d] tokens); a list of (b, h) gives the
    same values for just those chains ([n, T, d]).  For decode workloads `step`
    selects the token of that step and tokens drop the T axis ([B,H,d] / [n,d]).
    """
    T_full = 1 if wl.decode else wl.T
    t0, t1 = (0, T_full) if t_range is None else t_range
    base = 0 if step is None else 16 * (step + 1)
    idx = _row_index(wl, T_full, chains, t0, t1)
    nrows = wl.B * T_full * wl.H if idx is None else idx.size
    bf = wl.dtype == "bf16"
    K, V = wl.K, wl.V

    def tok(name, kind, d, bf16=bf, mu=0.0, scale=1.0, per_token=False, stream_name=None):
        st = base + STREAM[stream_name or name]
        return rows(wl.seed, st, kind, d, row_index=idx, nrows=nrows, mu=mu, scale=scale,
                    per_token=per_token, bf16=bf16)

    out = {
        "q": tok("q", KIND_L2, K),
        "k": tok("k", KIND_L2, K),
        "v": tok("v", KIND_NORMAL, V),
    }
    if wl.gates == "gdn":
        out["alpha"] = tok("alpha", KIND_DECAY, K, bf16=False, mu=wl.alpha_mu, scale=wl.alpha_scale,
                           per_token=True, stream_name="alpha_s")
    else:
        out["alpha"] = tok("alpha", KIND_DECAY, K, bf16=False, mu=wl.alpha_mu, scale=wl.alpha_scale)
    if wl.gates in ("kda", "gdn"):
        out["b"] = tok("b", KIND_SIGMOID, K, per_token=True, stream_name="beta")
        out["w"] = tok("w", KIND_SIGMOID, V, per_token=True, stream_name="beta")
    else:
        out["b"] = tok("b", KIND_SIGMOID, K)
        out["w"] = tok("w", KIND_SIGMOID, V)
    n_ch = None if chains is None else len(chains)
    for key, a in out.items():
        d = a.shape[1]
        if wl.decode:
            out[key] = a.reshape(wl.B, wl.H, d) if n_ch is None else a.reshape(n_ch, d)
        else:
            out[key] = a.reshape(wl.B, t1 - t0, wl.H, d) if n_ch is None else a.reshape(n_ch, t1 - t0, d)
    return out


def make_state(wl: Workload, chains=None):
    """Initial state S0 ([B,H,K,V] or [n,K,V]) as float32, or None for a zero state."""
    if wl.s0_std is None:
        return None
    K, V = wl.K, wl.V
    if chains is None:
        x = rows(wl.seed, STREAM["S0"], KIND_NORMAL, K * V, nrows=wl.B * wl.H, scale=wl.s0_std)
        return x.reshape(wl.B, wl.H, K, V)
    idx = np.array([b * wl.H + h for (b, h) in chains], dtype=np.uint64)
    x = rows(wl.seed, STREAM["S0"], KIND_NORMAL, K * V, row_index=idx, scale=wl.s0_std)
    return x.reshape(len(chains), K, V)


RAW_QK_SCALE = 3.0   # raw (unnormalised) q, k rows of the layer-edge workloads: N(0, 3^2)


def make_raw_inputs(wl: Workload, chains=None):
    """The layer's raw inputs for the fused-edge prefill, same shapes as make_inputs: q, k ~ N(0, 9)
    (not normalised), v ~ N(0, 1), the decay logit a ~ N(alpha_mu, 1) in fp32 (the recurrence's
    alpha is exp(-softplus(a)), so its distribution matches make_inputs' alpha), the gate logits
    b, w ~ N(0, 1).  Streams 10..15 of the workload's seed."""
    T_full = wl.T
    idx = _row_index(wl, T_full, chains, 0, T_full)
    nrows = wl.B * T_full * wl.H if idx is None else idx.size
    bf = wl.dtype == "bf16"

    def tok(st, d, mu=0.0, scale=1.0, bf16=bf):
        return rows(wl.seed, st, KIND_NORMAL, d, row_index=idx, nrows=nrows, mu=mu, scale=scale, bf16=bf16)

    out = {"q": tok(10, wl.K, scale=RAW_QK_SCALE), "k": tok(11, wl.K, scale=RAW_QK_SCALE), "v": tok(12, wl.V),
           "a": tok(13, wl.K, mu=wl.alpha_mu, bf16=False), "b": tok(14, wl.K), "w": tok(15, wl.V)}
    shape = (wl.B, T_full, wl.H) if chains is None else (len(chains), T_full)
    return {key: a.reshape(*shape, a.shape[-1]) for key, a in out.items()}


def make_output_grads(wl: Workload, chains=None, dst_std: float = 0.05):
    """Gradients at the recurrence's outputs for the backward workloads: dO ~ N(0, 1) in the token
    dtype ([B,T,H,V] or [n,T,V]) and dS_T ~ N(0, dst_std^2) fp32 ([B,H,K,V] or [n,K,V]).
    Streams 9 (dO) and 10 + 256 (dS_T) of the workload's seed."""
    T_full = wl.T
    idx = _row_index(wl, T_full, chains, 0, T_full)
    nrows = wl.B * T_full * wl.H if idx is None else idx.size
    dO = rows(wl.seed, 9, KIND_NORMAL, wl.V, row_index=idx, nrows=nrows, bf16=wl.dtype == "bf16")
    if chains is None:
        dST = rows(wl.seed, 266, KIND_NORMAL, wl.K * wl.V, nrows=wl.B * wl.H, scale=dst_std)
        return dO.reshape(wl.B, T_full, wl.H, wl.V), dST.reshape(wl.B, wl.H, wl.K, wl.V)
    sidx = np.array([b * wl.H + h for (b, h) in chains], dtype=np.uint64)
    dST = rows(wl.seed, 266, KIND_NORMAL, wl.K * wl.V, row_index=sidx, scale=dst_std)
    return dO.reshape(len(chains), T_full, wl.V), dST.reshape(len(chains), wl.K, wl.V)


def as_f64(d: dict) -> dict:
    """fp64 copies (for the oracle) of a dict of float32 input arrays."""
    return {k: (None if v is None else np.asarray(v, dtype=np.float64)) for k, v in d.items()}
