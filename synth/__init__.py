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
* values are drawn in fp64 and rounded to the storage dtype (fp64 -> fp32
  -> bf16, each round-to-nearest-even); the oracle is fed the rounded values.

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

def softplus(x):
    return np.logaddexp(0.0, x)


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def l2_normalise(x):
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
    return x / np.maximum(n, 1e-300)


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round fp64 values to the storage dtype; returned as fp64 (exactly representable)."""
    if dtype == "f64":
        return np.asarray(x, dtype=np.float64)
    x32 = np.asarray(x, dtype=np.float32)
    if dtype == "f32":
        return x32.astype(np.float64)
    if dtype == "bf16":
        u = x32.view(np.uint32).astype(np.uint64)
        # round-to-nearest-even on the top 16 bits (inputs here are finite)
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
    alpha_scale: float = 1.0  # multiplies softplus (stress variant uses 0.02)
    extra: dict = field(default_factory=dict, compare=False)


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


def _token_offsets(B, T, H, d, chains, t0, t1):
    """Counter offsets of rows (b, t, h, :) for t in [t0, t1) of each chain (b, h)."""
    rows = []
    for (b, h) in chains:
        t = np.arange(t0, t1, dtype=np.uint64)
        rows.append(((np.uint64(b) * np.uint64(T) + t) * np.uint64(H) + np.uint64(h)) * np.uint64(d))
    return np.concatenate(rows) if rows else np.zeros(0, dtype=np.uint64)


def _draw_tokens(wl: Workload, name: str, d: int, chains, t0, t1, stream_base, T_full):
    """Normals for token tensor `name` as [n_chains, t1-t0, d] (chain subset) or [B,T,H,d]."""
    seed, st = wl.seed, stream_base + STREAM[name]
    if chains is None:
        x = normal(seed, st, wl.B * T_full * wl.H * d)
        return x.reshape(wl.B, T_full, wl.H, d)
    offs = _token_offsets(wl.B, T_full, wl.H, d, chains, t0, t1)
    return normal_rows(seed, st, offs, d).reshape(len(chains), t1 - t0, d)


def _draw_per_token(wl: Workload, name: str, chains, t0, t1, stream_base, T_full):
    """One normal per (b, t, h): returned as [..., 1] to broadcast over channels."""
    seed, st = wl.seed, stream_base + STREAM[name]
    if chains is None:
        x = normal(seed, st, wl.B * T_full * wl.H)
        return x.reshape(wl.B, T_full, wl.H, 1)
    offs = _token_offsets(wl.B, T_full, wl.H, 1, chains, t0, t1)
    return normal_rows(seed, st, offs, 1).reshape(len(chains), t1 - t0, 1)


def make_inputs(wl: Workload, chains=None, t_range=None, step: int | None = None):
    """Inputs of a workload, rounded to their storage dtypes, as fp64 numpy arrays.

    chains=None gives full tensors ([B,T,H,d] tokens, [B,H,K,V] state); a list of
    (b, h) gives the same values for just those chains ([n, T, d] tokens,
    [n, K, V] state).  For decode workloads, `step` selects the token of that
    step (T = 1) and S0 is the state before step 0.
    """
    T_full = 1 if wl.decode else wl.T
    t0, t1 = (0, T_full) if t_range is None else t_range
    stream_base = 0 if step is None else 16 * (step + 1)
    tok = wl.dtype
    K, V = wl.K, wl.V
    out = {}
    q = _draw_tokens(wl, "q", K, chains, t0, t1, stream_base, T_full)
    out["q"] = round_to(l2_normalise(q), tok)
    k = _draw_tokens(wl, "k", K, chains, t0, t1, stream_base, T_full)
    out["k"] = round_to(l2_normalise(k), tok)
    out["v"] = round_to(_draw_tokens(wl, "v", V, chains, t0, t1, stream_base, T_full), tok)
    if wl.gates == "gdn":
        a = _draw_per_token(wl, "alpha_s", chains, t0, t1, stream_base, T_full) + wl.alpha_mu
        a = np.broadcast_to(np.exp(-wl.alpha_scale * softplus(a)), q.shape[:-1] + (K,))
    else:
        a = _draw_tokens(wl, "alpha", K, chains, t0, t1, stream_base, T_full) + wl.alpha_mu
        a = np.exp(-wl.alpha_scale * softplus(a))
    out["alpha"] = round_to(np.ascontiguousarray(a), "f32")
    if wl.gates in ("kda", "gdn"):
        beta = sigmoid(_draw_per_token(wl, "beta", chains, t0, t1, stream_base, T_full))
        out["b"] = round_to(np.ascontiguousarray(np.broadcast_to(beta, q.shape[:-1] + (K,))), tok)
        out["w"] = round_to(np.ascontiguousarray(np.broadcast_to(beta, q.shape[:-1] + (V,))), tok)
    else:
        out["b"] = round_to(sigmoid(_draw_tokens(wl, "b", K, chains, t0, t1, stream_base, T_full)), tok)
        out["w"] = round_to(sigmoid(_draw_tokens(wl, "w", V, chains, t0, t1, stream_base, T_full)), tok)
    if wl.decode:
        # decode tokens drop the T axis: [B, H, d] (or [n, d] for a chain subset)
        for key in ("q", "k", "v", "alpha", "b", "w"):
            out[key] = out[key][:, 0] if chains is None else out[key][:, 0]
    return out


def make_state(wl: Workload, chains=None):
    """Initial state S0 ([B,H,K,V] or [n,K,V]) rounded to fp32, or None for a zero state."""
    if wl.s0_std is None:
        return None
    K, V = wl.K, wl.V
    st = STREAM["S0"]
    if chains is None:
        x = normal(wl.seed, st, wl.B * wl.H * K * V).reshape(wl.B, wl.H, K, V)
    else:
        offs = np.array([((b * wl.H + h) * K * V) for (b, h) in chains], dtype=np.uint64)
        x = normal_rows(wl.seed, st, offs, K * V).reshape(len(chains), K, V)
    return round_to(wl.s0_std * x, "f32")
