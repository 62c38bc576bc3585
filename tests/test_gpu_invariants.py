"""Exact invariants of the update equation, run through the CUDA kernels (prefill on both of
its paths, and decode).  They follow from the equation alone (page "NVIDIA представила
Gated DeltaNet-2 ...", section "Техническая схема"), so they check the kernels against
the mathematics without going through the oracle:

- frozen state: alpha = 1, b = w = 0 make every factor of the update the identity, so
  S_T = S0 (to fp32 rounding) and every output is o_t = S0^T q_t;
- erase-then-write: with b = 1 and a unit-norm key, k^T (I - k k^T) = 0 removes what the
  decayed state held along k and the write puts w ⊙ v there, so k_t^T S_t = (w_t ⊙ v_t)^T
  for any alpha.  fp32 tokens use L2-normalised keys; bf16 tokens use one-hot keys, whose
  norm is exactly 1 in bf16.
"""
import numpy as np
import pytest

import synth
from tests.gpu_util import TOL, assert_close, cuda_or_skip, f64, prefill, to_device

pytestmark = pytest.mark.gpu

ARGS = ("q", "k", "v", "alpha", "b", "w")
FP32_ROUNDING = 1e-6   # a few fp32 ulps, relative to max|S0|


def _inputs(B, H, T, K, V, dtype, seed):
    wl = synth.Workload("inv", B, H, T, K, V, dtype, 1.0, s0_std=0.05, seed=seed)
    return synth.make_inputs(wl), synth.make_state(wl)


def _frozen(x):
    x = dict(x)
    x["alpha"] = np.ones_like(x["alpha"])
    x["b"] = np.zeros_like(x["b"])
    x["w"] = np.zeros_like(x["w"])
    return x


def _one_hot_keys(x, rng):
    x = dict(x)
    K = x["k"].shape[-1]
    idx = rng.integers(0, K, size=x["k"].shape[:-1])
    x["k"] = (np.arange(K) == idx[..., None]).astype(np.float32)
    x["b"] = np.ones_like(x["b"])
    return x, idx


@pytest.mark.parametrize("dtype,K,V,T", [("bf16", 128, 128, 200), ("bf16", 64, 128, 130), ("f32", 128, 128, 130),
                                         ("f32", 64, 64, 65)])
def test_frozen_state_prefill(dtype, K, V, T):
    torch, g = cuda_or_skip()
    x, S0 = _inputs(2, 3, T, K, V, dtype, 0x51)
    x = _frozen(x)
    xd = to_device(torch, x, dtype)
    o, S_T = prefill(torch, g, xd, torch.from_numpy(S0).cuda())
    assert_close("S_T = S0", f64(S_T), S0.astype(np.float64), FP32_ROUNDING)
    q = xd["q"].double().cpu().numpy()      # the token values the kernel read
    ref_o = np.einsum("bthc,bhcv->bthv", q, S0.astype(np.float64))
    assert_close("o = S0^T q", f64(o), ref_o, TOL[dtype])


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_frozen_state_decode(dtype):
    torch, g = cuda_or_skip()
    x, S0 = _inputs(4, 5, 1, 128, 128, dtype, 0x52)
    x = {n: a[:, 0] for n, a in _frozen(x).items()}
    xd = to_device(torch, x, dtype)
    S = torch.from_numpy(S0).cuda()
    o = torch.full((4, 5, 128), float("nan"), dtype=xd["q"].dtype, device="cuda")
    g.gdn2_decode_step(*(xd[n] for n in ARGS), S, o)
    torch.cuda.synchronize()
    assert_close("S = S0", f64(S), S0.astype(np.float64), FP32_ROUNDING)
    ref_o = np.einsum("bhc,bhcv->bhv", xd["q"].double().cpu().numpy(), S0.astype(np.float64))
    assert_close("o = S0^T q", f64(o), ref_o, TOL[dtype])


@pytest.mark.parametrize("dtype,K,V,T", [("f32", 128, 128, 130), ("f32", 64, 64, 200), ("bf16", 128, 128, 200),
                                         ("bf16", 128, 64, 65)])
def test_erase_then_write_prefill(dtype, K, V, T):
    torch, g = cuda_or_skip()
    x, S0 = _inputs(2, 3, T, K, V, dtype, 0x53)
    x = dict(x)
    x["b"] = np.ones_like(x["b"])
    if dtype == "bf16":   # exactly unit-norm keys in bf16
        x, _ = _one_hot_keys(x, np.random.default_rng(9))
    xd = to_device(torch, x, dtype)
    o, S_T = prefill(torch, g, xd, torch.from_numpy(S0).cuda())
    k_last = xd["k"][:, -1].double().cpu().numpy()                       # [B, H, K]
    u_last = (xd["w"][:, -1].double() * xd["v"][:, -1].double()).cpu().numpy()   # [B, H, V]
    read = np.einsum("bhc,bhcv->bhv", k_last, f64(S_T))
    assert_close("k_T^T S_T = w_T * v_T", read, u_last, TOL[dtype])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_erase_then_write_decode(dtype):
    torch, g = cuda_or_skip()
    x, S0 = _inputs(4, 5, 1, 128, 128, dtype, 0x54)
    x = {n: a[:, 0] for n, a in x.items()}
    x["b"] = np.ones_like(x["b"])
    if dtype == "bf16":
        x, _ = _one_hot_keys(x, np.random.default_rng(10))
    xd = to_device(torch, x, dtype)
    S = torch.from_numpy(S0).cuda()
    o = torch.full((4, 5, 128), float("nan"), dtype=xd["q"].dtype, device="cuda")
    g.gdn2_decode_step(*(xd[n] for n in ARGS), S, o)
    torch.cuda.synchronize()
    read = np.einsum("bhc,bhcv->bhv", xd["k"].double().cpu().numpy(), f64(S))
    u = (xd["w"].double() * xd["v"].double()).cpu().numpy()
    assert_close("k^T S = w * v", read, u, TOL[dtype])
