"""Host-side checks of the Python binding's argument marshalling, on the CPU: the compute entry
points of the library are replaced by a recorder (the workspace-size queries stay the real
library's), the device checks by no-ops, and the recorded C arguments are compared with the
tensors passed in: order of the pointers, sizes, dtype code, workspace size; shape and dtype
errors are raised before any call."""
import ctypes

import pytest
import torch

import gated_delta_rule_96_b200 as g


class Recorder:
    def __init__(self, real):
        self.real = real
        self.calls = []

    def __getattr__(self, name):
        if name.endswith("_workspace_bytes") or name in ("gdn2_status_str", "gdn2_chunk_fwd_path"):
            return getattr(self.real, name)

        def record(*args):
            self.calls.append((name, args))
            return 0
        return record


@pytest.fixture
def rec(monkeypatch):
    r = Recorder(g.load_library())
    monkeypatch.setattr(g, "load_library", lambda: r)
    monkeypatch.setattr(g, "_check_cuda", lambda *ts: None)
    monkeypatch.setattr(g, "_stream", lambda s: ctypes.c_void_p(0))
    monkeypatch.setattr(g, "new_workspace", lambda n, device=None: torch.zeros(max(int(n), 256), dtype=torch.uint8))
    return r


def addr(p):
    return None if p is None else p.value


def test_bwd_marshalling(rec):
    B, T, H, K, V = 2, 70, 3, 64, 128
    tk = lambda dt=torch.bfloat16: torch.zeros(B, T, H, K, dtype=dt)
    tv = lambda dt=torch.bfloat16: torch.zeros(B, T, H, V, dtype=dt)
    st = lambda: torch.zeros(B, H, K, V)
    ins = [tk(), tk(), tv(), tk(torch.float32), tk(), tv(), st(), tv(), st()]
    outs = [tk(torch.float32), tk(torch.float32), tv(torch.float32), tk(torch.float32), tk(torch.float32),
            tv(torch.float32), st()]
    g.gdn2_chunk_bwd(*ins, *outs)
    name, args = rec.calls[-1]
    assert name == "gdn2_chunk_bwd"
    assert [addr(a) for a in args[:16]] == [t.data_ptr() for t in ins + outs]
    assert args[16:22] == (B, H, T, K, V, g.GDN2_BF16)
    assert args[23] >= g.gdn2_chunk_bwd_workspace_bytes(B, H, T, K, V)
    # optional S0, dS_T and dS0 travel as NULL
    g.gdn2_chunk_bwd(*ins[:6], None, ins[7], None, *outs[:6], None)
    _, args = rec.calls[-1]
    assert args[6] is None and args[8] is None and args[15] is None


def test_bwd_rejects_bad_arguments(rec):
    B, T, H, K, V = 1, 8, 2, 64, 64
    z = lambda *s, dt=torch.float32: torch.zeros(*s, dtype=dt)
    tk, tv, st = (B, T, H, K), (B, T, H, V), (B, H, K, V)
    good = [z(*tk), z(*tk), z(*tv), z(*tk), z(*tk), z(*tv), None, z(*tv), None,
            z(*tk), z(*tk), z(*tv), z(*tk), z(*tk), z(*tv), None]
    bad_shape = list(good)
    bad_shape[9] = z(B, T, H, K + 1)
    with pytest.raises(ValueError):
        g.gdn2_chunk_bwd(*bad_shape)
    bad_dtype = list(good)
    bad_dtype[7] = z(*tv, dt=torch.bfloat16)      # dO must have the token dtype
    with pytest.raises(TypeError):
        g.gdn2_chunk_bwd(*bad_dtype)
    bad_grad = list(good)
    bad_grad[12] = z(*tk, dt=torch.bfloat16)      # gradients are fp32
    with pytest.raises(TypeError):
        g.gdn2_chunk_bwd(*bad_grad)
    assert rec.calls == []


def test_edges_marshalling(rec):
    B, T, H, K, V = 1, 100, 2, 128, 128
    bf = lambda *s: torch.zeros(*s, dtype=torch.bfloat16)
    q, k, b = bf(B, T, H, K), bf(B, T, H, K), bf(B, T, H, K)
    v, w, o = bf(B, T, H, V), bf(B, T, H, V), bf(B, T, H, V)
    a = torch.zeros(B, T, H, K)
    weight, ST = torch.ones(V), torch.zeros(B, H, K, V)
    g.gdn2_chunk_fwd_edges(q, k, v, a, b, w, None, weight, o, ST)
    name, args = rec.calls[-1]
    assert name == "gdn2_chunk_fwd_edges"
    assert [addr(x) for x in args[:10]] == [q.data_ptr(), k.data_ptr(), v.data_ptr(), a.data_ptr(), b.data_ptr(),
                                           w.data_ptr(), None, weight.data_ptr(), o.data_ptr(), ST.data_ptr()]
    assert args[10:17] == (B, H, T, K, V, 64, g.GDN2_BF16)
    assert args[18] >= g.gdn2_chunk_fwd_edges_workspace_bytes(B, H, T, K, V)
    with pytest.raises(ValueError):
        g.gdn2_chunk_fwd_edges(q, k, v, a, b, w, None, torch.ones(V + 1), o, ST)
    with pytest.raises(TypeError):
        g.gdn2_chunk_fwd_edges(q, k, v, a.bfloat16(), b, w, None, weight, o, ST)


def test_fwd_and_decode_marshalling(rec):
    B, T, H, K, V = 2, 65, 3, 128, 64
    f = lambda *s, dt=torch.float32: torch.zeros(*s, dtype=dt)
    q, k, b, a = f(B, T, H, K), f(B, T, H, K), f(B, T, H, K), f(B, T, H, K)
    v, w, o = f(B, T, H, V), f(B, T, H, V), f(B, T, H, V)
    S0, ST = f(B, H, K, V), f(B, H, K, V)
    g.gdn2_chunk_fwd(q, k, v, a, b, w, S0, o, ST)
    name, args = rec.calls[-1]
    assert name == "gdn2_chunk_fwd"
    assert [addr(x) for x in args[:9]] == [t.data_ptr() for t in (q, k, v, a, b, w, S0, o, ST)]
    assert args[9:16] == (B, H, T, K, V, 64, g.GDN2_F32)
    assert args[17] >= g.gdn2_chunk_fwd_workspace_bytes(B, H, T, K, V, 64, g.GDN2_F32)
    qd, kd, bd, ad = f(B, H, K), f(B, H, K), f(B, H, K), f(B, H, K)
    vd, wd, od = f(B, H, V), f(B, H, V), f(B, H, V)
    g.gdn2_decode_step(qd, kd, vd, ad, bd, wd, S0, od)
    name, args = rec.calls[-1]
    assert name == "gdn2_decode_step"
    assert [addr(x) for x in args[:8]] == [t.data_ptr() for t in (qd, kd, vd, ad, bd, wd, S0, od)]
    assert args[8:13] == (B, H, K, V, g.GDN2_F32)


def test_autograd_op_calls_backward_with_token_dtype_gradients(rec):
    """gdn2_recurrence: the forward calls gdn2_chunk_fwd once; backward hands gdn2_chunk_bwd dO in the
    token dtype and dS_T in fp32, fp32 gradient buffers, and the saved inputs."""
    B, T, H, K, V = 1, 10, 2, 64, 64
    leaf = lambda *s, dt=torch.bfloat16: torch.zeros(*s, dtype=dt).requires_grad_()
    q, k, b, v, w = leaf(B, T, H, K), leaf(B, T, H, K), leaf(B, T, H, K), leaf(B, T, H, V), leaf(B, T, H, V)
    a, S0 = leaf(B, T, H, K, dt=torch.float32), leaf(B, H, K, V, dt=torch.float32)
    o, ST = g.gdn2_recurrence(q, k, v, a, b, w, S0)
    assert [c[0] for c in rec.calls] == ["gdn2_chunk_fwd"]
    (o.float().sum() + ST.sum()).backward()
    name, args = rec.calls[-1]
    assert name == "gdn2_chunk_bwd"
    assert [addr(x) for x in args[:7]] == [t.data_ptr() for t in (q, k, v, a, b, w, S0)]
    assert args[7] is not None and args[8] is not None and args[15] is not None
    assert args[16:22] == (B, H, T, K, V, g.GDN2_BF16)
    for t in (q, k, v, b, w):
        assert t.grad is not None and t.grad.dtype == torch.bfloat16 and t.grad.shape == t.shape
    assert a.grad.dtype == torch.float32 and S0.grad.shape == S0.shape


def test_token_dtype_mismatch_refused_before_any_call(rec):
    """The library reads every token tensor of a call in q's dtype: a tensor of another dtype would be
    read with the wrong element size, so the binding refuses it for every entry point."""
    B, T, H, K, V = 1, 8, 2, 64, 64
    bf = lambda *s: torch.zeros(*s, dtype=torch.bfloat16)
    f = lambda *s: torch.zeros(*s)
    tk, tv, st = (B, T, H, K), (B, T, H, V), (B, H, K, V)
    with pytest.raises(TypeError):     # v fp32 with bf16 q
        g.gdn2_chunk_fwd(bf(*tk), bf(*tk), f(*tv), f(*tk), bf(*tk), bf(*tv), None, bf(*tv), f(*st))
    with pytest.raises(TypeError):
        g.gdn2_chunk_fwd_noalloc(bf(*tk), f(*tk), bf(*tv), f(*tk), bf(*tk), bf(*tv), None, bf(*tv), f(*st))
    with pytest.raises(TypeError):     # w_logit fp32 with bf16 q_raw
        g.gdn2_chunk_fwd_edges(bf(*tk), bf(*tk), bf(*tv), f(*tk), bf(*tk), f(*tv), None, None, bf(*tv), f(*st))
    with pytest.raises(TypeError):     # k bf16 with fp32 q
        g.gdn2_chunk_bwd(f(*tk), bf(*tk), f(*tv), f(*tk), f(*tk), f(*tv), None, f(*tv), None,
                         f(*tk), f(*tk), f(*tv), f(*tk), f(*tk), f(*tv), None)
    with pytest.raises(TypeError):     # decode: b fp32 with bf16 q
        g.gdn2_decode_step(bf(B, H, K), bf(B, H, K), bf(B, H, V), f(B, H, K), f(B, H, K), bf(B, H, V), f(*st),
                           bf(B, H, V))
    assert rec.calls == []


def test_shape_mismatch_refused_before_any_call(rec):
    B, T, H, K, V = 1, 8, 2, 64, 64
    f = lambda *s: torch.zeros(*s)
    tk, tv, st = (B, T, H, K), (B, T, H, V), (B, H, K, V)
    with pytest.raises(ValueError):    # decode: k of another head count
        g.gdn2_decode_step(f(B, H, K), f(B, H + 1, K), f(B, H, V), f(B, H, K), f(B, H, K), f(B, H, V), f(*st),
                           f(B, H, V))
    with pytest.raises(ValueError):    # no-alloc prefill: alpha one token short
        g.gdn2_chunk_fwd_noalloc(f(*tk), f(*tk), f(*tv), f(B, T - 1, H, K), f(*tk), f(*tv), None, f(*tv), f(*st))
    with pytest.raises(ValueError):    # edges: v with another time length
        g.gdn2_chunk_fwd_edges(f(*tk).bfloat16(), f(*tk).bfloat16(), f(B, T + 1, H, V).bfloat16(), f(*tk),
                               f(*tk).bfloat16(), f(*tv).bfloat16(), None, None, f(*tv).bfloat16(), f(*st))
    assert rec.calls == []


class FakeTensor:
    def __init__(self, device, is_cuda=True, contiguous=True):
        self.device, self.is_cuda, self._c = device, is_cuda, contiguous

    def is_contiguous(self):
        return self._c


def test_check_cuda_rules():
    """CUDA tensors only, contiguous, all on one device (a kernel launched on one device must not be
    handed another device's pointers)."""
    d0, d1 = torch.device("cuda", 0), torch.device("cuda", 1)
    g._check_cuda(FakeTensor(d0), None, FakeTensor(d0))
    with pytest.raises(ValueError, match="one device"):
        g._check_cuda(FakeTensor(d0), FakeTensor(d1))
    with pytest.raises(ValueError, match="CUDA"):
        g._check_cuda(FakeTensor(torch.device("cpu"), is_cuda=False))
    with pytest.raises(ValueError, match="contiguous"):
        g._check_cuda(FakeTensor(d0, contiguous=False))
