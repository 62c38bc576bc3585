"""Python binding of libgdn2 (Gated DeltaNet-2 recurrence on B200, sm_100a).

Argument marshalling only: every step of the computation runs in the CUDA kernels
behind the C ABI declared in ``include/gdn2.h``.  PyTorch supplies device memory and
streams.  There is no CPU fallback: if ``libgdn2.so`` is missing or no CUDA device
is present the calls raise.

The operation (page "NVIDIA представила Gated DeltaNet-2 ...", section
"Техническая схема"):  S_t = (I - k_t (b_t ⊙ k_t)^T) Diag(alpha_t) S_{t-1}
+ k_t (w_t ⊙ v_t)^T,  o_t = S_t^T q_t.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "GDN2Error", "load_library", "library_path", "gdn2_chunk_fwd", "gdn2_chunk_fwd_edges", "gdn2_decode_step",
    "gdn2_chunk_fwd_workspace_bytes", "gdn2_chunk_fwd_path", "gdn2_workspace_status", "gdn2_status_str",
    "gdn2_chunk_fwd_noalloc", "NOALLOC_SCRATCH_BYTES",
    "chunk_fwd", "decode_step", "new_workspace", "gdn2_chunk_bwd", "gdn2_chunk_bwd_workspace_bytes",
    "gdn2_chunk_bwd_tc", "gdn2_chunk_bwd_tc_workspace_bytes",
    "gdn2_chunk_fwd_edges_workspace_bytes", "gdn2_recurrence", "gdn2_gemm_phase_probe",
    "PHASE_PROBE_FLOPS_PER_CHUNK", "gdn2_layer_edge_maps", "gdn2_rms_norm",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libgdn2.so"
_lib = None

GDN2_F32, GDN2_BF16 = 0, 1
STATUS_HEADER_BYTES = 256
NOALLOC_SCRATCH_BYTES = 32 << 20   # GDN2_NOALLOC_SCRATCH_BYTES in include/gdn2.h
PHASE_PROBE_FLOPS_PER_CHUNK = 14680064   # GDN2_PHASE_PROBE_FLOPS_PER_CHUNK in include/gdn2.h


class GDN2Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: status {status} ({gdn2_status_str(status)})")


def library_path() -> str:
    return os.path.join(_HERE, _LIB_NAME)


def load_library():
    """Load the in-tree libgdn2.so (built by __graft_entry__.build() / build.py)."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is not built; run `python -c 'import __graft_entry__ as g; g.build()'` "
                           "(the CUDA library is required: there is no CPU fallback)")
    lib = ctypes.CDLL(path)
    vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.gdn2_chunk_fwd_workspace_bytes.argtypes = [i] * 7
    lib.gdn2_chunk_fwd_workspace_bytes.restype = sz
    lib.gdn2_chunk_fwd_path.argtypes = [i] * 7
    lib.gdn2_chunk_fwd_path.restype = i
    lib.gdn2_chunk_fwd.argtypes = [vp] * 9 + [i] * 7 + [vp, sz, vp]
    lib.gdn2_chunk_fwd.restype = i
    lib.gdn2_decode_step.argtypes = [vp] * 8 + [i] * 5 + [vp]
    lib.gdn2_decode_step.restype = i
    lib.gdn2_workspace_status.argtypes = [vp, i, ctypes.POINTER(i), vp]
    lib.gdn2_workspace_status.restype = i
    lib.gdn2_chunk_fwd_noalloc.argtypes = [vp] * 9 + [i] * 7 + [vp]
    lib.gdn2_chunk_fwd_noalloc.restype = i
    lib.gdn2_chunk_fwd_edges.argtypes = [vp] * 10 + [i] * 7 + [vp, sz, vp]
    lib.gdn2_chunk_fwd_edges.restype = i
    lib.gdn2_chunk_fwd_edges_workspace_bytes.argtypes = [i] * 6
    lib.gdn2_chunk_fwd_edges_workspace_bytes.restype = sz
    lib.gdn2_chunk_bwd_workspace_bytes.argtypes = [i] * 5
    lib.gdn2_chunk_bwd_workspace_bytes.restype = sz
    lib.gdn2_chunk_bwd.argtypes = [vp] * 16 + [i] * 6 + [vp, sz, vp]
    lib.gdn2_chunk_bwd.restype = i
    lib.gdn2_chunk_bwd_tc_workspace_bytes.argtypes = [i] * 5
    lib.gdn2_chunk_bwd_tc_workspace_bytes.restype = sz
    lib.gdn2_chunk_bwd_tc.argtypes = [vp] * 16 + [i] * 6 + [vp, sz, vp]
    lib.gdn2_chunk_bwd_tc.restype = i
    lib.gdn2_layer_edge_maps.argtypes = [vp] * 10 + [i] * 5 + [vp]
    lib.gdn2_layer_edge_maps.restype = i
    lib.gdn2_rms_norm.argtypes = [vp, vp, ctypes.c_longlong, i, vp]
    lib.gdn2_rms_norm.restype = i
    lib.gdn2_gemm_phase_probe.argtypes = [i, i, i, vp, sz, vp]
    lib.gdn2_gemm_phase_probe.restype = i
    lib.gdn2_status_str.argtypes = [i]
    lib.gdn2_status_str.restype = ctypes.c_char_p
    _lib = lib
    return lib


def gdn2_status_str(status: int) -> str:
    return load_library().gdn2_status_str(int(status)).decode()


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return GDN2_BF16
    if t.dtype == torch.float32:
        return GDN2_F32
    raise TypeError(f"token tensors must be bfloat16 or float32, got {t.dtype}")


def gdn2_chunk_fwd_workspace_bytes(B, H, T, d_k, d_v, C=64, dtype=GDN2_BF16) -> int:
    return int(load_library().gdn2_chunk_fwd_workspace_bytes(B, H, T, d_k, d_v, C, int(dtype)))


def gdn2_chunk_fwd_path(B, H, T, d_k, d_v, C=64, dtype=GDN2_BF16) -> int:
    return int(load_library().gdn2_chunk_fwd_path(B, H, T, d_k, d_v, C, int(dtype)))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check_cuda(*ts):
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors (no CPU path)")
        if not t.is_contiguous():
            raise ValueError("all tensors must be contiguous")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"all tensors must be on one device ({dev} and {t.device} given)")


def _check_dtypes(ref, named):
    """Every (name, tensor) in `named` (None skipped) has the dtype of `ref`: the library reads all
    token tensors of a call in one dtype, so a mismatch would read the wrong number of bytes."""
    for name, t in named:
        if t is not None and t.dtype != ref.dtype:
            raise TypeError(f"{name} must have the token dtype {ref.dtype}, got {t.dtype}")


def _check_shapes(named):
    for name, t, shp in named:
        if t is not None and tuple(t.shape) != tuple(shp):
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shp)}")


def _on_device(t):
    """Make t's device current for the call: the library launches on the current device and on the
    given (or that device's current) stream."""
    import contextlib

    import torch
    return torch.cuda.device(t.device) if getattr(t, "is_cuda", False) else contextlib.nullcontext()


def new_workspace(nbytes: int, device=None):
    """Workspace tensor with its status header zeroed."""
    import torch
    ws = torch.empty(max(int(nbytes), STATUS_HEADER_BYTES), dtype=torch.uint8, device=device or "cuda")
    ws[:STATUS_HEADER_BYTES].zero_()
    return ws


def gdn2_chunk_fwd(q, k, v, alpha, b, w, S0, o, S_T, C=64, workspace=None, stream=None) -> None:
    """Prefill through the C ABI.  Shapes: q,k,b,alpha [B,T,H,d_k]; v,w,o [B,T,H,d_v];
    S0 (or None), S_T [B,H,d_k,d_v] fp32.  Raises GDN2Error on a nonzero status."""
    import torch
    _check_cuda(q, k, v, alpha, b, w, S0, o, S_T, workspace)
    B, T, H, K = q.shape
    V = v.shape[-1]
    dt = _dtype_code(q)
    if alpha.dtype != torch.float32 or S_T.dtype != torch.float32 or (S0 is not None and S0.dtype != torch.float32):
        raise TypeError("alpha and the states must be float32")
    _check_dtypes(q, (("k", k), ("b", b), ("v", v), ("w", w), ("o", o)))
    _check_shapes((("k", k, (B, T, H, K)), ("b", b, (B, T, H, K)), ("alpha", alpha, (B, T, H, K)),
                   ("w", w, (B, T, H, V)), ("o", o, (B, T, H, V)), ("S_T", S_T, (B, H, K, V)),
                   ("S0", S0, (B, H, K, V))))
    need = gdn2_chunk_fwd_workspace_bytes(B, H, T, K, V, C, dt)
    if workspace is None:
        workspace = new_workspace(need, q.device)
    with _on_device(q):
        rc = load_library().gdn2_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(b), _ptr(w), _ptr(S0),
                                           _ptr(o), _ptr(S_T), B, H, T, K, V, C, dt, _ptr(workspace),
                                           workspace.numel() * workspace.element_size(), _stream(stream))
    if rc != 0:
        raise GDN2Error(rc, "gdn2_chunk_fwd")


def gdn2_chunk_fwd_edges_workspace_bytes(B, H, T, d_k, d_v, C=64) -> int:
    return int(load_library().gdn2_chunk_fwd_edges_workspace_bytes(B, H, T, d_k, d_v, C))


def gdn2_chunk_fwd_edges(q_raw, k_raw, v, a_logit, b_logit, w_logit, S0, o_weight, o, S_T, C=64, workspace=None,
                         stream=None) -> None:
    """Prefill with the layer edges fused (include/gdn2.h, gdn2_chunk_fwd_edges): q, k L2-normalised,
    b = sigmoid(b_logit), w = sigmoid(w_logit), alpha = exp(-softplus(a_logit)), optional RMSNorm of o
    with weight o_weight [d_v] (None: no norm).  bf16 tokens, d_k = d_v = 128."""
    import torch
    _check_cuda(q_raw, k_raw, v, a_logit, b_logit, w_logit, S0, o_weight, o, S_T, workspace)
    B, T, H, K = q_raw.shape
    V = v.shape[-1]
    dt = _dtype_code(q_raw)
    for name, t in (("a_logit", a_logit), ("S_T", S_T), ("S0", S0), ("o_weight", o_weight)):
        if t is not None and t.dtype != torch.float32:
            raise TypeError(f"{name} must be float32")
    _check_dtypes(q_raw, (("k_raw", k_raw), ("v", v), ("b_logit", b_logit), ("w_logit", w_logit), ("o", o)))
    _check_shapes((("k_raw", k_raw, (B, T, H, K)), ("b_logit", b_logit, (B, T, H, K)),
                   ("a_logit", a_logit, (B, T, H, K)), ("v", v, (B, T, H, V)), ("w_logit", w_logit, (B, T, H, V)),
                   ("o", o, (B, T, H, V)), ("S_T", S_T, (B, H, K, V)), ("S0", S0, (B, H, K, V)),
                   ("o_weight", o_weight, (V,))))
    need = gdn2_chunk_fwd_edges_workspace_bytes(B, H, T, K, V, C)
    if workspace is None:
        workspace = new_workspace(need, q_raw.device)
    with _on_device(q_raw):
        rc = load_library().gdn2_chunk_fwd_edges(_ptr(q_raw), _ptr(k_raw), _ptr(v), _ptr(a_logit), _ptr(b_logit),
                                                 _ptr(w_logit), _ptr(S0), _ptr(o_weight), _ptr(o), _ptr(S_T), B, H,
                                                 T, K, V, C, dt, _ptr(workspace),
                                                 workspace.numel() * workspace.element_size(), _stream(stream))
    if rc != 0:
        raise GDN2Error(rc, "gdn2_chunk_fwd_edges")


def gdn2_chunk_bwd_workspace_bytes(B, H, T, d_k, d_v) -> int:
    return int(load_library().gdn2_chunk_bwd_workspace_bytes(B, H, T, d_k, d_v))


def gdn2_chunk_bwd(q, k, v, alpha, b, w, S0, dO, dS_T, dq, dk, dv, dalpha, db, dw, dS0, workspace=None,
                   stream=None) -> None:
    """Backward of the recurrence (include/gdn2.h, gdn2_chunk_bwd): fp32 gradients of every forward
    input from dO (token dtype) and dS_T (fp32 or None); dS0 may be None."""
    import torch
    _check_cuda(q, k, v, alpha, b, w, S0, dO, dS_T, dq, dk, dv, dalpha, db, dw, dS0, workspace)
    B, T, H, K = q.shape
    V = v.shape[-1]
    dt = _dtype_code(q)
    for name, t in (("alpha", alpha), ("S0", S0), ("dS_T", dS_T), ("dq", dq), ("dk", dk), ("dv", dv),
                    ("dalpha", dalpha), ("db", db), ("dw", dw), ("dS0", dS0)):
        if t is not None and t.dtype != torch.float32:
            raise TypeError(f"{name} must be float32")
    _check_dtypes(q, (("k", k), ("v", v), ("b", b), ("w", w), ("dO", dO)))
    tk, tv, st = (B, T, H, K), (B, T, H, V), (B, H, K, V)
    _check_shapes((("k", k, tk), ("b", b, tk), ("alpha", alpha, tk), ("v", v, tv), ("w", w, tv),
                   ("dO", dO, tv), ("S0", S0, st), ("dS_T", dS_T, st), ("dq", dq, tk), ("dk", dk, tk),
                   ("dalpha", dalpha, tk), ("db", db, tk), ("dv", dv, tv), ("dw", dw, tv), ("dS0", dS0, st)))
    if workspace is None:
        workspace = new_workspace(max(gdn2_chunk_bwd_workspace_bytes(B, H, T, K, V), 256), q.device)
    with _on_device(q):
        rc = load_library().gdn2_chunk_bwd(*(_ptr(t) for t in (q, k, v, alpha, b, w, S0, dO, dS_T, dq, dk, dv,
                                                               dalpha, db, dw, dS0)), B, H, T, K, V, dt,
                                           _ptr(workspace), workspace.numel() * workspace.element_size(),
                                           _stream(stream))
    if rc != 0:
        raise GDN2Error(rc, "gdn2_chunk_bwd")


def gdn2_chunk_bwd_tc_workspace_bytes(B, H, T, d_k, d_v) -> int:
    return int(load_library().gdn2_chunk_bwd_tc_workspace_bytes(B, H, T, d_k, d_v))


def gdn2_chunk_bwd_tc(q, k, v, alpha, b, w, S0, dO, dS_T, dq, dk, dv, dalpha, db, dw, dS0, workspace=None,
                      stream=None) -> None:
    """Tensor-core backward (include/gdn2.h, gdn2_chunk_bwd_tc): the gradients of gdn2_chunk_bwd for bf16
    tokens with d_k = d_v = 128, from bf16 tensor-core products.  A workspace passed in must start with a
    zeroed status header (new_workspace gives one)."""
    import torch
    _check_cuda(q, k, v, alpha, b, w, S0, dO, dS_T, dq, dk, dv, dalpha, db, dw, dS0, workspace)
    B, T, H, K = q.shape
    V = v.shape[-1]
    dt = _dtype_code(q)
    for name, t in (("alpha", alpha), ("S0", S0), ("dS_T", dS_T), ("dq", dq), ("dk", dk), ("dv", dv),
                    ("dalpha", dalpha), ("db", db), ("dw", dw), ("dS0", dS0)):
        if t is not None and t.dtype != torch.float32:
            raise TypeError(f"{name} must be float32")
    _check_dtypes(q, (("k", k), ("v", v), ("b", b), ("w", w), ("dO", dO)))
    tk, tv, st = (B, T, H, K), (B, T, H, V), (B, H, K, V)
    _check_shapes((("k", k, tk), ("b", b, tk), ("alpha", alpha, tk), ("v", v, tv), ("w", w, tv),
                   ("dO", dO, tv), ("S0", S0, st), ("dS_T", dS_T, st), ("dq", dq, tk), ("dk", dk, tk),
                   ("dalpha", dalpha, tk), ("db", db, tk), ("dv", dv, tv), ("dw", dw, tv), ("dS0", dS0, st)))
    if workspace is None:
        workspace = new_workspace(max(gdn2_chunk_bwd_tc_workspace_bytes(B, H, T, K, V), 256), q.device)
    with _on_device(q):
        rc = load_library().gdn2_chunk_bwd_tc(*(_ptr(t) for t in (q, k, v, alpha, b, w, S0, dO, dS_T, dq, dk, dv,
                                                                  dalpha, db, dw, dS0)), B, H, T, K, V, dt,
                                              _ptr(workspace), workspace.numel() * workspace.element_size(),
                                              _stream(stream))
    if rc != 0:
        raise GDN2Error(rc, "gdn2_chunk_bwd_tc")


def gdn2_chunk_fwd_noalloc(q, k, v, alpha, b, w, S0, o, S_T, C=64, stream=None) -> None:
    """Prefill for callers that cannot allocate device memory: no workspace argument; the
    library's fixed scratch array is used instead (see include/gdn2.h for the size limit
    and for the rule that overlapping calls race on the shared array)."""
    import torch
    _check_cuda(q, k, v, alpha, b, w, S0, o, S_T)
    B, T, H, K = q.shape
    V = v.shape[-1]
    dt = _dtype_code(q)
    if alpha.dtype != torch.float32 or S_T.dtype != torch.float32 or (S0 is not None and S0.dtype != torch.float32):
        raise TypeError("alpha and the states must be float32")
    _check_dtypes(q, (("k", k), ("b", b), ("v", v), ("w", w), ("o", o)))
    _check_shapes((("k", k, (B, T, H, K)), ("b", b, (B, T, H, K)), ("alpha", alpha, (B, T, H, K)),
                   ("w", w, (B, T, H, V)), ("o", o, (B, T, H, V)), ("S_T", S_T, (B, H, K, V)),
                   ("S0", S0, (B, H, K, V))))
    with _on_device(q):
        rc = load_library().gdn2_chunk_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(b), _ptr(w),
                                                   _ptr(S0), _ptr(o), _ptr(S_T), B, H, T, K, V, C, dt,
                                                   _stream(stream))
    if rc != 0:
        raise GDN2Error(rc, "gdn2_chunk_fwd_noalloc")


def gdn2_decode_step(q, k, v, alpha, b, w, S, o, stream=None) -> None:
    """One decode token: q,k,b,alpha [B,H,d_k]; v,w,o [B,H,d_v]; S [B,H,d_k,d_v] fp32 in place."""
    import torch
    _check_cuda(q, k, v, alpha, b, w, S, o)
    B, H, K = q.shape
    V = v.shape[-1]
    dt = _dtype_code(q)
    if alpha.dtype != torch.float32 or S.dtype != torch.float32:
        raise TypeError("alpha and S must be float32")
    _check_dtypes(q, (("k", k), ("b", b), ("v", v), ("w", w), ("o", o)))
    _check_shapes((("k", k, (B, H, K)), ("b", b, (B, H, K)), ("alpha", alpha, (B, H, K)), ("v", v, (B, H, V)),
                   ("w", w, (B, H, V)), ("o", o, (B, H, V)), ("S", S, (B, H, K, V))))
    with _on_device(q):
        rc = load_library().gdn2_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(b), _ptr(w), _ptr(S),
                                             _ptr(o), B, H, K, V, dt, _stream(stream))
    if rc != 0:
        raise GDN2Error(rc, "gdn2_decode_step")


def gdn2_layer_edge_maps(q_raw, k_raw, a_logit, b_logit, w_logit, q, k, alpha, b, w, stream=None) -> None:
    """The layer's edge maps as one kernel (include/gdn2.h): raw q, k, decay and gate logits -> the
    normalised q, k, alpha = exp(-softplus(a)), b = sigmoid, w = sigmoid.  bf16 tokens, fp32 logits of alpha."""
    import torch
    _check_cuda(q_raw, k_raw, a_logit, b_logit, w_logit, q, k, alpha, b, w)
    B, T, H, K = q_raw.shape
    V = w_logit.shape[-1]
    for name, t in (("a_logit", a_logit), ("alpha", alpha)):
        if t.dtype != torch.float32:
            raise TypeError(f"{name} must be float32")
    for name, t in (("q_raw", q_raw), ("k_raw", k_raw), ("b_logit", b_logit), ("w_logit", w_logit), ("q", q),
                    ("k", k), ("b", b), ("w", w)):
        if t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be bfloat16")
    tk, tv = (B, T, H, K), (B, T, H, V)
    _check_shapes((("k_raw", k_raw, tk), ("a_logit", a_logit, tk), ("b_logit", b_logit, tk), ("w_logit", w_logit, tv),
                   ("q", q, tk), ("k", k, tk), ("alpha", alpha, tk), ("b", b, tk), ("w", w, tv)))
    with _on_device(q_raw):
        rc = load_library().gdn2_layer_edge_maps(*(_ptr(t) for t in (q_raw, k_raw, a_logit, b_logit, w_logit, q, k,
                                                                     alpha, b, w)), B, T, H, K, V, _stream(stream))
    if rc != 0:
        raise GDN2Error(rc, "gdn2_layer_edge_maps")


def gdn2_rms_norm(o, weight, stream=None) -> None:
    """RMSNorm of o in place over its last axis (include/gdn2.h): bf16 o, fp32 weight [d_v]."""
    import torch
    _check_cuda(o, weight)
    V = o.shape[-1]
    if o.dtype != torch.bfloat16 or weight.dtype != torch.float32 or tuple(weight.shape) != (V,):
        raise TypeError("o must be bfloat16 and weight float32 of shape [d_v]")
    with _on_device(o):
        rc = load_library().gdn2_rms_norm(_ptr(o), _ptr(weight), o.numel() // V, V, _stream(stream))
    if rc != 0:
        raise GDN2Error(rc, "gdn2_rms_norm")


def gdn2_gemm_phase_probe(mode, reps, nctas, workspace, stream=None) -> None:
    """Measurement aid (include/gdn2.h): one chunk's tensor-core products, `reps` chunks per CTA on
    `nctas` CTAs; mode 0 back to back, mode 1 each group waiting for the one before."""
    _check_cuda(workspace)
    with _on_device(workspace):
        rc = load_library().gdn2_gemm_phase_probe(int(mode), int(reps), int(nctas), _ptr(workspace),
                                                  workspace.numel() * workspace.element_size(), _stream(stream))
    if rc != 0:
        raise GDN2Error(rc, "gdn2_gemm_phase_probe")


def gdn2_workspace_status(workspace, clear=False, stream=None) -> int:
    out = ctypes.c_int(0)
    with _on_device(workspace):
        rc = load_library().gdn2_workspace_status(_ptr(workspace), 1 if clear else 0, ctypes.byref(out),
                                                  _stream(stream))
    if rc != 0:
        raise GDN2Error(rc, "gdn2_workspace_status")
    return out.value


def chunk_fwd(q, k, v, alpha, b, w, S0=None, C=64, workspace=None, stream=None):
    """Allocating convenience wrapper: returns (o, S_T)."""
    import torch
    B, T, H, K = q.shape
    V = v.shape[-1]
    o = torch.empty((B, T, H, V), dtype=q.dtype, device=q.device)
    S_T = torch.empty((B, H, K, V), dtype=torch.float32, device=q.device)
    gdn2_chunk_fwd(q, k, v, alpha, b, w, S0, o, S_T, C=C, workspace=workspace, stream=stream)
    return o, S_T


def decode_step(q, k, v, alpha, b, w, S, stream=None):
    """Allocating convenience wrapper: updates S in place, returns o."""
    import torch
    B, H, K = q.shape
    o = torch.empty((B, H, v.shape[-1]), dtype=q.dtype, device=q.device)
    gdn2_decode_step(q, k, v, alpha, b, w, S, o, stream=stream)
    return o


def _recurrence_function():
    """torch.autograd.Function over the C ABI: forward gdn2_chunk_fwd, backward gdn2_chunk_bwd."""
    import torch

    class GDN2Recurrence(torch.autograd.Function):
        @staticmethod
        def forward(ctx, q, k, v, alpha, b, w, S0):
            o, S_T = chunk_fwd(q, k, v, alpha, b, w, S0)
            ctx.save_for_backward(q, k, v, alpha, b, w, S0)
            ctx.has_s0 = S0 is not None
            return o, S_T

        @staticmethod
        def backward(ctx, dO, dS_T):
            q, k, v, alpha, b, w, S0 = ctx.saved_tensors
            if not ctx.has_s0:
                S0 = None
            B, T, H, K = q.shape
            V = v.shape[-1]
            dO = torch.zeros_like(v) if dO is None else dO.to(q.dtype).contiguous()
            dS_T = None if dS_T is None else dS_T.to(torch.float32).contiguous()
            dev = q.device
            gk = [torch.empty((B, T, H, K), dtype=torch.float32, device=dev) for _ in range(4)]   # dq dk dalpha db
            gv = [torch.empty((B, T, H, V), dtype=torch.float32, device=dev) for _ in range(2)]   # dv dw
            dS0 = torch.empty((B, H, K, V), dtype=torch.float32, device=dev) if ctx.has_s0 else None
            gdn2_chunk_bwd(q, k, v, alpha, b, w, S0, dO, dS_T, gk[0], gk[1], gv[0], gk[2], gk[3], gv[1], dS0)
            # the autograd engine casts each gradient to its input's dtype
            return gk[0], gk[1], gv[0], gk[2], gk[3], gv[1], dS0

    return GDN2Recurrence


_GDN2_FN = None


def gdn2_recurrence(q, k, v, alpha, b, w, S0=None):
    """Differentiable prefill: (o, S_T) = recurrence(q, k, v, alpha, b, w, S0) with gradients of every
    input through gdn2_chunk_bwd.  Same shapes and dtypes as gdn2_chunk_fwd (CUDA tensors only)."""
    global _GDN2_FN
    if _GDN2_FN is None:
        _GDN2_FN = _recurrence_function()
    return _GDN2_FN.apply(q, k, v, alpha, b, w, S0)
