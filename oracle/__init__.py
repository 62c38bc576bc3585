"""fp64 CPU oracle of the Gated DeltaNet-2 recurrence -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference leg may import this package.  The library path (the CUDA kernels
behind the C ABI) never calls it, and the two share no code.

Definition followed (page "NVIDIA представила Gated DeltaNet-2 ...", section
"Техническая схема", the state-update equation):

    S_t = (I - k_t (b_t ⊙ k_t)^T) Diag(alpha_t) S_{t-1} + k_t (w_t ⊙ v_t)^T,
    o_t = S_t^T q_t.

The C source (``gdn2_oracle.c``) evaluates it token by token in fp64.  Every
function here is pinned by ``tests/test_oracle_pins.py``; none is
"parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn2_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libgdn2_oracle.so")
_lib = None


def build(force: bool = False, src: str | None = None, out: str | None = None) -> str:
    """Compile the oracle with gcc.  `src`/`out` let tests build a modified copy."""
    src = src or _SRC
    out = out or _LIB_PATH
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        # -ffp-contract=off: plain fp64 multiplies and adds, no fused multiply-add
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fPIC", "-shared", "-o", tmp, src,
                               "-lpthread"])
        os.replace(tmp, out)
    return out


def _bind(lib):
    dp = ctypes.POINTER(ctypes.c_double)
    i = ctypes.c_int
    lib.gdn2_oracle_recurrence.argtypes = [dp] * 9 + [i] * 6
    lib.gdn2_oracle_recurrence.restype = i
    lib.gdn2_oracle_decode_step.argtypes = [dp] * 8 + [i] * 5
    lib.gdn2_oracle_decode_step.restype = i
    lib.gdn2_oracle_backward.argtypes = [dp] * 16 + [i] * 6
    lib.gdn2_oracle_backward.restype = i
    return lib


def load(path: str | None = None):
    """Load the compiled oracle (or another build of it, for tests)."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def _threads(n):
    return n if n is not None else (os.cpu_count() or 1)


def recurrence(q, k, v, alpha, b, w, S0=None, threads=None, lib=None):
    """Sequential fp64 recurrence.

    q, k, alpha, b: [B, T, H, K]; v, w: [B, T, H, V]; S0: [B, H, K, V] or None.
    Returns (o [B, T, H, V], S_T [B, H, K, V]) as fp64 arrays.
    """
    lib = lib or load()
    q, k, v, alpha, b, w, S0 = map(_f64, (q, k, v, alpha, b, w, S0))
    B, T, H, K = q.shape
    V = v.shape[-1]
    for name, a, d in (("k", k, K), ("alpha", alpha, K), ("b", b, K), ("v", v, V), ("w", w, V)):
        if a.shape != (B, T, H, d):
            raise ValueError(f"{name} has shape {a.shape}, expected {(B, T, H, d)}")
    if S0 is not None and S0.shape != (B, H, K, V):
        raise ValueError(f"S0 has shape {S0.shape}, expected {(B, H, K, V)}")
    o = np.empty((B, T, H, V), dtype=np.float64)
    ST = np.empty((B, H, K, V), dtype=np.float64)
    rc = lib.gdn2_oracle_recurrence(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(b), _ptr(w), _ptr(S0),
                                    _ptr(o), _ptr(ST), B, H, T, K, V, _threads(threads))
    if rc != 0:
        raise RuntimeError(f"oracle returned {rc}")
    return o, ST


def decode_step(q, k, v, alpha, b, w, S, threads=None, lib=None):
    """One decode token per chain.  Tokens [B, H, d]; S [B, H, K, V] is updated IN PLACE.

    Returns o [B, H, V].
    """
    lib = lib or load()
    q, k, v, alpha, b, w = map(_f64, (q, k, v, alpha, b, w))
    if not (isinstance(S, np.ndarray) and S.dtype == np.float64 and S.flags.c_contiguous):
        raise ValueError("S must be a C-contiguous float64 array (updated in place)")
    B, H, K = q.shape
    V = v.shape[-1]
    if S.shape != (B, H, K, V):
        raise ValueError(f"S has shape {S.shape}, expected {(B, H, K, V)}")
    o = np.empty((B, H, V), dtype=np.float64)
    rc = lib.gdn2_oracle_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(b), _ptr(w), _ptr(S),
                                     _ptr(o), B, H, K, V, _threads(threads))
    if rc != 0:
        raise RuntimeError(f"oracle returned {rc}")
    return o


def recurrence_backward_c(q, k, v, alpha, b, w, S0, dO, dST, threads=None, mem_budget=8 << 30, lib=None):
    """The gradient of oracle/backward.py computed by the C oracle (gdn2_oracle_backward), chains in
    parallel.  Same arguments and results ([B, T, H, d] tokens, [B, H, K, V] states, S0 / dST may be
    None).  Each thread keeps its chain's T+1 states: threads are capped so that they fit mem_budget."""
    lib = lib or load()
    q, k, v, alpha, b, w, S0, dO, dST = map(_f64, (q, k, v, alpha, b, w, S0, dO, dST))
    B, T, H, K = q.shape
    V = v.shape[-1]
    per_chain = 8 * (T + 1) * K * V
    nt = max(1, min(_threads(threads), int(mem_budget // max(per_chain, 1))))
    outs = [np.empty((B, T, H, K)), np.empty((B, T, H, K)), np.empty((B, T, H, V)), np.empty((B, T, H, K)),
            np.empty((B, T, H, K)), np.empty((B, T, H, V)), np.empty((B, H, K, V))]
    rc = lib.gdn2_oracle_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(b), _ptr(w), _ptr(S0), _ptr(dO),
                                  _ptr(dST), *(_ptr(o) for o in outs), B, H, T, K, V, nt)
    if rc != 0:
        raise RuntimeError(f"oracle backward returned {rc}")
    return tuple(outs)


def chain_recurrence(q, k, v, alpha, b, w, S0=None, threads=None):
    """Recurrence for independent chains given as [n, T, d] token arrays and [n, K, V] states."""
    n, T, K = q.shape
    V = v.shape[-1]
    r = lambda a: None if a is None else np.ascontiguousarray(a).reshape(n, T, 1, a.shape[-1])
    S0r = None if S0 is None else np.ascontiguousarray(S0).reshape(n, 1, K, V)
    o, ST = recurrence(r(q), r(k), r(v), r(alpha), r(b), r(w), S0r, threads=threads)
    return o.reshape(n, T, V), ST.reshape(n, K, V)


def rel_err(x, y):
    """max|x - y| / max|y| (the parity metric)."""
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    den = float(np.max(np.abs(y))) if y.size else 0.0
    num = float(np.max(np.abs(x - y))) if y.size else 0.0
    if den == 0.0:
        return num
    return num / den


# ----------------------------------------------------------------------------- layer edges
# The layer around the recurrence (page "NVIDIA представила Gated DeltaNet-2 ...", the paragraph on
# the layer: q and k pass an L2 norm, the gates b and w are sigmoid projections, the output goes
# through RMSNorm).  The pages fix neither the norms' epsilons nor how the decay is produced from
# its projection; the readings taken: eps = 1e-6 in both norms, alpha = exp(-softplus(a)).  All fp64.

NORM_EPS = 1e-6
RMS_EPS = 1e-6


def sigmoid(x):
    x = _f64(x)
    return 0.5 * (1.0 + np.tanh(0.5 * x))


def softplus(x):
    x = _f64(x)
    return np.logaddexp(0.0, x)


def l2_normalize(x, eps=NORM_EPS):
    """x / max(|x|_2, eps) over the last axis."""
    x = _f64(x)
    return x / np.maximum(np.linalg.norm(x, axis=-1, keepdims=True), eps)


def layer_edges(q_raw, k_raw, a_logit, b_logit, w_logit):
    """Recurrence inputs (q, k, alpha, b, w) from the layer's raw inputs."""
    return (l2_normalize(q_raw), l2_normalize(k_raw), np.exp(-softplus(a_logit)), sigmoid(b_logit),
            sigmoid(w_logit))


def rms_norm(o, weight, eps=RMS_EPS):
    """o / sqrt(mean(o^2) + eps) * weight over the last axis."""
    o = _f64(o)
    return o / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + eps) * _f64(weight)
