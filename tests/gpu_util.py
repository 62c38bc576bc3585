"""Helpers of the GPU parity tests: move seeded inputs to the device, call the C ABI
through the binding, bring results back as fp64 numpy arrays."""
import numpy as np
import pytest

import oracle
import synth

TOL = {"f32": 1e-4, "bf16": 2e-2}   # max|gpu - ref| / max|ref| per tensor


def cuda_or_skip():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gated_delta_rule_96_b200 as g
    g.load_library()   # must exist on a GPU machine: missing library is a failure, not a skip
    return torch, g


def tok_dtype(torch, dtype):
    return torch.bfloat16 if dtype == "bf16" else torch.float32


def to_device(torch, x: dict, dtype: str):
    td = tok_dtype(torch, dtype)
    out = {}
    for key, a in x.items():
        t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
        out[key] = t if key == "alpha" else t.to(td)
    return out


def prefill(torch, g, xd, S0=None, C=64, workspace=None, poison=True):
    q = xd["q"]
    B, T, H, K = q.shape
    V = xd["v"].shape[-1]
    o = torch.empty((B, T, H, V), dtype=q.dtype, device=q.device)
    S_T = torch.empty((B, H, K, V), dtype=torch.float32, device=q.device)
    if poison:
        o.fill_(float("nan"))
        S_T.fill_(float("nan"))
    if workspace is None:
        dt = g.GDN2_BF16 if q.dtype == torch.bfloat16 else g.GDN2_F32
        nbytes = g.gdn2_chunk_fwd_workspace_bytes(B, H, T, K, V, C, dt)
        workspace = g.new_workspace(nbytes, q.device)
        if poison and nbytes > g.STATUS_HEADER_BYTES:
            workspace[g.STATUS_HEADER_BYTES:].fill_(0xFF)   # NaN pattern: unwritten reads show up
    g.gdn2_chunk_fwd(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["b"], xd["w"], S0, o, S_T, C=C,
                     workspace=workspace)
    torch.cuda.synchronize()
    assert g.gdn2_workspace_status(workspace) == 0
    return o, S_T


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def elementwise_rel_err(got, ref):
    """Elementwise relative error, floored at 1e-3 of the tensor's largest magnitude so that
    entries near zero do not dominate: max_i |x_i - y_i| / (|y_i| + 1e-3 max|y|).  Reported
    beside the bar's metric as information; the bar itself is the max-normalised error."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    scale = np.max(np.abs(ref)) if ref.size else 0.0
    if ref.size == 0 or scale == 0.0:
        return float(np.max(np.abs(got - ref))) if ref.size else 0.0
    return float(np.max(np.abs(got - ref) / (np.abs(ref) + 1e-3 * scale)))


def assert_close(name, got, ref, tol):
    err = oracle.rel_err(got, ref)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    elem = elementwise_rel_err(got, ref)
    print(f"{name}: max-normalised err {err:.3e} (bar {tol:.1e}); elementwise err {elem:.3e}")
    assert err <= tol, f"{name}: rel err {err:.3e} > {tol:.1e} (elementwise {elem:.3e})"
    return err


def workload(name, **kw):
    wl = synth.WORKLOADS[name]
    if kw:
        fields = {f: getattr(wl, f) for f in wl.__dataclass_fields__}
        fields.update(kw)
        wl = synth.Workload(**fields)
    return wl
