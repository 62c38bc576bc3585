"""gdn2_chunk_fwd_noalloc: the prefill for callers that cannot allocate device memory
(hosts whose allocator owns all device memory, or paths that forbid cudaMalloc because
it can synchronise the device).  Its scratch is a fixed array inside the library that
every call shares and that keeps the previous call's contents.

The GPU test calls it through the C ABI twice in a row, the second call smaller than the
first and with a ragged last chunk, so that a result depending on the first call's
leftovers in the array would show.  Each result is checked against the fp64 oracle
within the parity bars of the other tests and, where gdn2_chunk_fwd runs the same
CUDA-core path, against gdn2_chunk_fwd bit for bit.  A third call resumes in place
(S_T aliasing S0).  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest

import gated_delta_rule_96_b200 as g
import oracle
import synth
from tests.gpu_util import TOL, assert_close, cuda_or_skip, f64, prefill, to_device

ARGS = ("q", "k", "v", "alpha", "b", "w")


def test_noalloc_rejects_problems_beyond_its_scratch():
    lib = g.load_library()
    fake = ctypes.c_void_p(0x10000)    # never dereferenced: the size check comes first
    # B*H*ceil(T/64) = 1*16*64 = 1024 chunk-heads at d = 128 needs ~151 MB > 32 MiB
    rc = lib.gdn2_chunk_fwd_noalloc(*(fake,) * 6, None, fake, fake, 1, 16, 4096, 128, 128, 64, 1, None)
    assert rc == -9
    assert "scratch" in g.gdn2_status_str(rc)
    assert lib.gdn2_chunk_fwd_noalloc(*(fake,) * 6, None, fake, fake, 1, 1, 64, 96, 128, 64, 1, None) == -4


def _case(call, B, T, H, K, V, dtype, seed):
    wl = synth.Workload(f"na{call}", B, H, T, K, V, dtype, 1.0 if dtype == "bf16" else 0.0, s0_std=0.02,
                        seed=seed)
    return wl, synth.make_inputs(wl), synth.make_state(wl)


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,K,V", [("bf16", 128, 128), ("f32", 64, 64)])
def test_noalloc_two_calls_against_oracle(dtype, K, V):
    torch, _ = cuda_or_skip()
    H = 4
    # the second call is smaller than the first, with a different, ragged T
    for call, (B, T, seed) in enumerate(((2, 300, 0xA11), (1, 70, 0xA12))):
        wl, x, S0_np = _case(call, B, T, H, K, V, dtype, seed)
        xd = to_device(torch, x, dtype)
        S0 = torch.from_numpy(S0_np).cuda()
        o = torch.full((B, T, H, V), float("nan"), dtype=xd["q"].dtype, device="cuda")
        S_T = torch.full((B, H, K, V), float("nan"), device="cuda")
        g.gdn2_chunk_fwd_noalloc(*(xd[n] for n in ARGS), S0, o, S_T)
        torch.cuda.synchronize()
        ref_o, ref_S = oracle.recurrence(*(x[n] for n in ARGS), S0_np)
        assert_close(f"o (call {call + 1})", f64(o), ref_o, TOL[dtype])
        assert_close(f"S_T (call {call + 1})", f64(S_T), ref_S, TOL[dtype])
        if g.gdn2_chunk_fwd_path(B, H, T, K, V, 64, g.GDN2_BF16 if dtype == "bf16" else g.GDN2_F32) == 0:
            # the workspace entry point runs the same kernels: identical bits
            o_ws, S_ws = prefill(torch, g, xd, S0)
            assert torch.equal(o.view(torch.int16 if dtype == "bf16" else torch.int32),
                               o_ws.view(torch.int16 if dtype == "bf16" else torch.int32))
            assert torch.equal(S_T.view(torch.int32), S_ws.view(torch.int32))


@pytest.mark.gpu
def test_noalloc_in_place_resume():
    """S_T aliasing S0: two calls joined through the one state buffer equal the oracle's
    single pass over the whole sequence."""
    torch, _ = cuda_or_skip()
    B, H, T, K, V, cut = 1, 3, 150, 128, 128, 64
    wl, x, S0_np = _case(2, B, T, H, K, V, "bf16", 0xA13)
    xd = to_device(torch, x, "bf16")
    S = torch.from_numpy(S0_np).cuda()
    outs = []
    for sl in (slice(0, cut), slice(cut, T)):
        p = {n: xd[n][:, sl].contiguous() for n in ARGS}
        o = torch.full((B, sl.stop - sl.start, H, V), float("nan"), dtype=torch.bfloat16, device="cuda")
        g.gdn2_chunk_fwd_noalloc(*(p[n] for n in ARGS), S, o, S)
        outs.append(o)
    torch.cuda.synchronize()
    ref_o, ref_S = oracle.recurrence(*(x[n] for n in ARGS), S0_np)
    assert_close("o (resumed in place)", f64(torch.cat(outs, dim=1)), ref_o, TOL["bf16"])
    assert_close("S_T (resumed in place)", f64(S), ref_S, TOL["bf16"])
    assert np.isfinite(f64(S)).all()
