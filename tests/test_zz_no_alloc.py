"""gdn2_chunk_fwd_noalloc: the prefill for callers that cannot allocate device memory
(hosts whose allocator owns all device memory, or paths that forbid cudaMalloc because
it can synchronise the device).  Its scratch is a fixed array inside the library.

The GPU test calls it through the C ABI twice in a row, on two different input sets,
and compares each result with gdn2_chunk_fwd on the same inputs, within the parity
tolerances of the other tests.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest

import gated_delta_rule_96_b200 as g
import synth
from tests.gpu_util import TOL, assert_close, cuda_or_skip, f64, prefill, to_device


def test_noalloc_rejects_problems_beyond_its_scratch():
    lib = g.load_library()
    fake = ctypes.c_void_p(0x10000)    # never dereferenced: the size check comes first
    # B*H*ceil(T/64) = 1*16*64 = 1024 chunk-heads at d = 128 needs ~151 MB > 32 MiB
    rc = lib.gdn2_chunk_fwd_noalloc(*(fake,) * 6, None, fake, fake, 1, 16, 4096, 128, 128, 64, 1, None)
    assert rc == -9
    assert "scratch" in g.gdn2_status_str(rc)
    assert lib.gdn2_chunk_fwd_noalloc(*(fake,) * 6, None, fake, fake, 1, 1, 64, 96, 128, 64, 1, None) == -4


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,K,V,T", [("bf16", 128, 128, 300), ("f32", 64, 64, 130)])
def test_noalloc_matches_workspace_entry_point_two_calls(dtype, K, V, T):
    torch, _ = cuda_or_skip()
    B, H = 2, 4
    for call, seed in enumerate((0xA11, 0xA12)):
        wl = synth.Workload(f"na{call}", B, H, T, K, V, dtype, 1.0 if dtype == "bf16" else 0.0, s0_std=0.02,
                            seed=seed)
        xd = to_device(torch, synth.make_inputs(wl), dtype)
        S0 = torch.from_numpy(synth.make_state(wl)).cuda()
        o_ref, S_ref = prefill(torch, g, xd, S0)
        o = torch.full_like(o_ref, float("nan"))
        S_T = torch.full_like(S_ref, float("nan"))
        g.gdn2_chunk_fwd_noalloc(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["b"], xd["w"], S0, o, S_T)
        torch.cuda.synchronize()
        assert_close(f"o (call {call + 1})", f64(o), f64(o_ref), TOL[dtype])
        assert_close(f"S_T (call {call + 1})", f64(S_T), f64(S_ref), TOL[dtype])
        assert np.isfinite(f64(o)).all()
