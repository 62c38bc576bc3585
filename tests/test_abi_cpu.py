"""C-ABI checks that need no GPU: the library loads, exports every symbol the header
declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

import gated_delta_rule_96_b200 as g

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn2.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"GDN2_API\s+[\w\s\*]+?\b(gdn2_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    return g.load_library()


def test_header_declares_entry_points():
    syms = declared_symbols()
    for name in ("gdn2_chunk_fwd", "gdn2_decode_step", "gdn2_chunk_fwd_workspace_bytes", "gdn2_status_str",
                 "gdn2_workspace_status", "gdn2_chunk_fwd_path", "gdn2_chunk_fwd_edges",
                 "gdn2_chunk_fwd_edges_workspace_bytes", "gdn2_chunk_bwd", "gdn2_chunk_bwd_workspace_bytes",
                 "gdn2_chunk_fwd_noalloc", "gdn2_gemm_phase_probe", "gdn2_layer_edge_maps", "gdn2_rms_norm",
                 "gdn2_chunk_bwd_tc", "gdn2_chunk_bwd_tc_workspace_bytes"):
        assert name in syms


def test_every_declared_symbol_is_exported(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), f"{name} declared in gdn2.h but not exported"


def test_status_strings(lib):
    for code in range(-8, 1):
        assert g.gdn2_status_str(code)
    assert g.gdn2_status_str(0) == "ok"
    assert g.gdn2_status_str(12345) == "unknown status"


def test_workspace_bytes():
    # the status header is always required
    assert g.gdn2_chunk_fwd_workspace_bytes(0, 0, 0, 128, 128) >= 256
    n1 = g.gdn2_chunk_fwd_workspace_bytes(1, 1, 64, 128, 128, 64, g.GDN2_F32)
    n2 = g.gdn2_chunk_fwd_workspace_bytes(1, 1, 128, 128, 128, 64, g.GDN2_F32)
    n3 = g.gdn2_chunk_fwd_workspace_bytes(2, 3, 128, 128, 128, 64, g.GDN2_F32)
    assert n2 - 256 == 2 * (n1 - 256) and n3 - 256 == 6 * (n2 - 256)
    # a ragged tail costs a whole chunk
    assert g.gdn2_chunk_fwd_workspace_bytes(1, 1, 65, 128, 128, 64, g.GDN2_F32) == n2


def test_workspace_bytes_tensor_core_path():
    # many chains: the two-stage path keeps one 75,776-byte record per chunk-head of a window of at
    # most 64 chunks
    rec = 75776
    assert g.gdn2_chunk_fwd_workspace_bytes(8, 16, 4096, 128, 128, 64, g.GDN2_BF16) == 256 + 8 * 16 * 64 * rec
    # a window holds at most 16,384 chunk-heads but at least 64 chunks: 65 chains take 252 chunks at once
    assert g.gdn2_chunk_fwd_workspace_bytes(1, 65, 64 * 70 + 5, 128, 128, 64, g.GDN2_BF16) == 256 + 65 * 71 * rec
    assert g.gdn2_chunk_fwd_workspace_bytes(1, 65, 64 * 260, 128, 128, 64, g.GDN2_BF16) == 256 + 65 * 252 * rec
    assert g.gdn2_chunk_fwd_workspace_bytes(2, 33, 65, 128, 128, 64, g.GDN2_BF16) == 256 + 66 * 2 * rec
    assert g.gdn2_chunk_fwd_path(8, 16, 4096, 128, 128, 64, g.GDN2_BF16) == 2
    assert g.gdn2_chunk_fwd_path(4, 16, 1024, 128, 128, 64, g.GDN2_BF16) == 1
    assert g.gdn2_chunk_fwd_workspace_bytes(4, 16, 1024, 128, 128, 64, g.GDN2_BF16) == 256
    assert g.gdn2_chunk_fwd_path(8, 16, 4096, 128, 128, 64, g.GDN2_F32) == 0
    # few long chains: the two-stage path over a window of up to 16,384 chunk-heads, each chain cut into
    # segments walked in parallel (three fp32 states per chain and segment)
    state = 4 * 128 * 128
    # B1 H16 T65536: 1,024 chunks in one window, 148 // 16 = 9 segments (one walk per SM)
    assert g.gdn2_chunk_fwd_path(1, 16, 65536, 128, 128, 64, g.GDN2_BF16) == 2
    assert g.gdn2_chunk_fwd_workspace_bytes(1, 16, 65536, 128, 128, 64, g.GDN2_BF16) == \
        256 + 16 * 1024 * rec + 3 * 16 * 9 * state
    # B1 H2, 41 chunks: at most 74 segments by chains, at least 8 chunks each -> 5 segments of 9 chunks
    assert g.gdn2_chunk_fwd_workspace_bytes(1, 2, 64 * 40 + 37, 128, 128, 64, g.GDN2_BF16) == \
        256 + 2 * 41 * rec + 3 * 2 * 5 * state
    # up to 64 chains of fewer than 32 chunks: the fused kernel, status header only
    assert g.gdn2_chunk_fwd_path(1, 2, 64 * 31, 128, 128, 64, g.GDN2_BF16) == 1
    assert g.gdn2_chunk_fwd_workspace_bytes(1, 2, 64 * 31, 128, 128, 64, g.GDN2_BF16) == 256


P = ctypes.c_void_p
FAKE = P(0x10000)       # never dereferenced: every case below fails validation first


def call_fwd(lib, B=1, H=1, T=8, K=128, V=128, C=64, dtype=1, ptr=FAKE, ST=FAKE, ws=FAKE, ws_bytes=1 << 30,
             o=FAKE):
    return lib.gdn2_chunk_fwd(ptr, ptr, ptr, ptr, ptr, ptr, None, o, ST, B, H, T, K, V, C, dtype, ws, ws_bytes,
                              None)


def test_chunk_fwd_validation(lib):
    assert call_fwd(lib, T=-1) == -2
    assert call_fwd(lib, B=-1) == -2
    assert call_fwd(lib, dtype=7) == -3
    assert call_fwd(lib, K=96) == -4
    assert call_fwd(lib, V=32) == -4
    assert call_fwd(lib, C=32) == -4
    assert call_fwd(lib, ptr=None) == -1
    assert call_fwd(lib, o=None) == -1
    assert call_fwd(lib, ST=None) == -1
    assert call_fwd(lib, ptr=P(0x10004)) == -7
    assert call_fwd(lib, ws=None) == -5
    assert call_fwd(lib, ws=P(0x10008)) == -7
    assert call_fwd(lib, ws_bytes=16) == -5
    # empty batch: nothing to launch
    assert call_fwd(lib, B=0) == 0
    assert call_fwd(lib, H=0) == 0


def test_decode_validation(lib):
    f = lambda **kw: lib.gdn2_decode_step(*(kw.get("ptr", FAKE),) * 6, kw.get("S", FAKE), kw.get("o", FAKE),
                                         kw.get("B", 1), kw.get("H", 1), kw.get("K", 128), kw.get("V", 128),
                                         kw.get("dtype", 1), None)
    assert f(B=-1) == -2
    assert f(dtype=2) == -3
    assert f(K=256) == -4
    assert f(ptr=None) == -1
    assert f(S=None) == -1
    assert f(S=P(0x10002)) == -7
    assert f(B=0) == 0


def test_workspace_status_null(lib):
    out = ctypes.c_int(0)
    assert lib.gdn2_workspace_status(None, 0, ctypes.byref(out), None) == -1


def test_binding_refuses_cpu_tensors():
    torch = pytest.importorskip("torch")
    x = torch.zeros((1, 4, 1, 64), dtype=torch.bfloat16)
    a = torch.zeros((1, 4, 1, 64))
    with pytest.raises(ValueError, match="CUDA"):
        g.gdn2_chunk_fwd(x, x, x, a, x, x, None, x, torch.zeros(1, 1, 64, 64))


def test_bwd_workspace_bytes():
    a = lambda n: (n + 255) // 256 * 256
    ntok, state = 8 * 4096 * 16, 4 * 128 * 128
    # two fp32 [B,T,H,d_v] buffers, the state every 64 steps, one d_k vector every 64 steps
    assert g.gdn2_chunk_bwd_workspace_bytes(8, 16, 4096, 128, 128) == \
        2 * a(4 * ntok * 128) + a(128 * 64 * state) + a(128 * 64 * 4 * 128)
    # a ragged tail costs a whole chunk of checkpoints; a single chain splits its value columns over
    # several blocks, which adds the partial row sums of the last pass (fp32 [B,T,H,d_k])
    assert g.gdn2_chunk_bwd_workspace_bytes(1, 1, 65, 64, 128) == \
        2 * a(4 * 65 * 128) + a(2 * 4 * 64 * 128) + a(2 * 4 * 64) + a(4 * 65 * 64)
    assert g.gdn2_chunk_bwd_workspace_bytes(1, 1, 8, 96, 128) == 0


def call_bwd(lib, B=1, H=1, T=8, K=128, V=128, dtype=1, ptr=FAKE, grad=FAKE, ws=FAKE, ws_bytes=1 << 30):
    return lib.gdn2_chunk_bwd(*(ptr,) * 6, None, ptr, None, *(grad,) * 6, None, B, H, T, K, V, dtype, ws,
                              ws_bytes, None)


def test_chunk_bwd_validation(lib):
    assert call_bwd(lib, T=-1) == -2
    assert call_bwd(lib, H=-1) == -2
    assert call_bwd(lib, dtype=5) == -3
    assert call_bwd(lib, K=32) == -4
    assert call_bwd(lib, ptr=None) == -1
    assert call_bwd(lib, grad=None) == -1
    assert call_bwd(lib, ptr=P(0x10004)) == -7
    assert call_bwd(lib, grad=P(0x10008)) == -7
    assert call_bwd(lib, ws=None) == -5
    assert call_bwd(lib, ws_bytes=64) == -5
    assert call_bwd(lib, B=0) == 0
    # no tokens and no dS0 wanted: nothing to do, no pointer read
    assert call_bwd(lib, T=0, ptr=None, grad=None, ws=None, ws_bytes=0) == 0


def test_bwd_tc_workspace_bytes():
    rec, side, state = 75776, 124928, 4 * 128 * 128
    # status header, a record and a side record per chunk-head, the end state of every chain
    assert g.gdn2_chunk_bwd_tc_workspace_bytes(8, 16, 4096, 128, 128) == 256 + 8 * 16 * 64 * (rec + side) + 128 * state
    assert g.gdn2_chunk_bwd_tc_workspace_bytes(2, 3, 65, 128, 128) == 256 + 6 * 2 * (rec + side) + 6 * state
    # few long chains: the replay walks 41 chunks in min(128 / 2, 41 // 8) = 5 segments per chain, three
    # fp32 states per segment
    assert g.gdn2_chunk_bwd_tc_workspace_bytes(1, 2, 64 * 40 + 37, 128, 128) == \
        256 + 2 * 41 * (rec + side) + 2 * state + 3 * state * 2 * 5
    assert g.gdn2_chunk_bwd_tc_workspace_bytes(1, 1, 8, 64, 128) == 0
    assert g.gdn2_chunk_bwd_tc_workspace_bytes(1, 1, 0, 128, 128) == 256


def call_bwd_tc(lib, B=1, H=1, T=8, K=128, V=128, dtype=1, ptr=FAKE, grad=FAKE, ws=FAKE, ws_bytes=1 << 30):
    return lib.gdn2_chunk_bwd_tc(*(ptr,) * 6, None, ptr, None, *(grad,) * 6, None, B, H, T, K, V, dtype, ws,
                                 ws_bytes, None)


def test_chunk_bwd_tc_validation(lib):
    assert call_bwd_tc(lib, T=-1) == -2
    assert call_bwd_tc(lib, dtype=5) == -3
    assert call_bwd_tc(lib, dtype=0) == -4     # fp32 tokens: gdn2_chunk_bwd
    assert call_bwd_tc(lib, K=64) == -4
    assert call_bwd_tc(lib, V=64) == -4
    assert call_bwd_tc(lib, ptr=None) == -1
    assert call_bwd_tc(lib, grad=None) == -1
    assert call_bwd_tc(lib, ptr=P(0x10004)) == -7
    assert call_bwd_tc(lib, grad=P(0x10008)) == -7
    assert call_bwd_tc(lib, ws=None) == -5
    assert call_bwd_tc(lib, ws_bytes=1024) == -5
    assert call_bwd_tc(lib, B=0) == 0
    assert call_bwd_tc(lib, T=0, ptr=None, grad=None, ws=None, ws_bytes=0) == 0


def test_edges_workspace_bytes():
    # on the two-stage path the edge-fused prefill needs exactly the plain prefill's workspace
    for shape in ((8, 16, 4096), (1, 16, 65536), (1, 65, 64 * 70 + 5)):
        assert g.gdn2_chunk_fwd_edges_workspace_bytes(*shape, 128, 128) == \
            g.gdn2_chunk_fwd_workspace_bytes(*shape, 128, 128, 64, g.GDN2_BF16)
    # on the fused kernel (up to 64 chains of fewer than 32 chunks): one decay ring per block
    ring = 4 * 64 * 128 * 4   # four slots of a chunk's decay rows (fp32)
    assert ring == 128 * 1024
    assert g.gdn2_chunk_fwd_edges_workspace_bytes(4, 16, 1024, 128, 128) == 256 + 64 * ring
    # unsupported shapes need only the status header (the call itself is refused)
    assert g.gdn2_chunk_fwd_edges_workspace_bytes(1, 1, 64, 64, 64) == 256


def test_bwd_column_split_threshold():
    """The backward splits a chain's value columns while 2 x blocks still fit the 148 SMs: the split
    adds the fp32 [B,T,H,d_k] partial row sums to the workspace."""
    a = lambda n: (n + 255) // 256 * 256
    T, K, V = 128, 128, 128

    def base(chains):
        ntok = chains * T
        return 2 * a(4 * ntok * V) + a(chains * 2 * 4 * K * V) + a(chains * 2 * 4 * K)

    for chains, split in ((74, True), (75, False), (128, False), (1, True)):
        extra = a(4 * chains * T * K) if split else 0
        assert g.gdn2_chunk_bwd_workspace_bytes(1, chains, T, K, V) == base(chains) + extra, chains


def call_edges(lib, B=1, H=1, T=100, K=128, V=128, C=64, dtype=1, ptr=FAKE, weight=None, ST=FAKE, ws=FAKE,
               ws_bytes=1 << 30, o=FAKE):
    return lib.gdn2_chunk_fwd_edges(ptr, ptr, ptr, ptr, ptr, ptr, None, weight, o, ST, B, H, T, K, V, C, dtype, ws,
                                    ws_bytes, None)


def test_chunk_fwd_edges_validation(lib):
    assert call_edges(lib, T=-1) == -2
    assert call_edges(lib, B=-1) == -2
    assert call_edges(lib, dtype=9) == -3
    assert call_edges(lib, ptr=None) == -1
    assert call_edges(lib, o=None) == -1
    assert call_edges(lib, ST=None) == -1
    # the edges are fused into the tensor-core kernel only: bf16 tokens, d_k = d_v = 128, C = 64
    assert call_edges(lib, K=64) == -4
    assert call_edges(lib, V=64) == -4
    assert call_edges(lib, C=32) == -4
    assert call_edges(lib, dtype=0) == -4
    assert call_edges(lib, ptr=P(0x10004)) == -7
    assert call_edges(lib, weight=P(0x10008)) == -7
    assert call_edges(lib, ws=None) == -5
    assert call_edges(lib, ws=P(0x10004)) == -7
    # the ring (128 KB per block) is part of the workspace: the plain prefill's size is too small
    plain = g.gdn2_chunk_fwd_workspace_bytes(1, 1, 100, 128, 128, 64, g.GDN2_BF16)
    assert plain < g.gdn2_chunk_fwd_edges_workspace_bytes(1, 1, 100, 128, 128)
    assert call_edges(lib, ws_bytes=plain) == -5
    assert call_edges(lib, B=0) == 0
    assert call_edges(lib, H=0, weight=FAKE) == 0


def call_noalloc(lib, B=1, H=1, T=8, K=128, V=128, C=64, dtype=1, ptr=FAKE, ST=FAKE, o=FAKE):
    return lib.gdn2_chunk_fwd_noalloc(ptr, ptr, ptr, ptr, ptr, ptr, None, o, ST, B, H, T, K, V, C, dtype, None)


def test_chunk_fwd_noalloc_validation(lib):
    assert call_noalloc(lib, T=-1) == -2
    assert call_noalloc(lib, H=-1) == -2
    assert call_noalloc(lib, dtype=4) == -3
    assert call_noalloc(lib, K=32) == -4
    assert call_noalloc(lib, C=128) == -4
    assert call_noalloc(lib, ST=None) == -1
    assert call_noalloc(lib, ptr=None) == -1
    assert call_noalloc(lib, o=None) == -1
    assert call_noalloc(lib, ST=P(0x10004)) == -7
    assert call_noalloc(lib, ptr=P(0x10002)) == -7
    # more scratch than the fixed array holds is refused before any device call
    assert call_noalloc(lib, B=64, H=64, T=1 << 16) == -9


def test_library_is_standalone():
    """libgdn2.so depends on no Python or torch library (the CUDA runtime is linked statically): the
    boundary is plain C, usable from any host program."""
    import shutil
    import subprocess
    readelf = shutil.which("readelf")
    if readelf is None:
        pytest.skip("readelf not available")
    out = subprocess.run([readelf, "-d", g.library_path()], capture_output=True, text=True, check=True).stdout
    needed = re.findall(r"\(NEEDED\).*\[(.+?)\]", out)
    assert needed, out
    for lib_name in needed:
        assert not re.search(r"torch|c10|python|cudart", lib_name), lib_name


def test_phase_probe_validation(lib):
    ws = ctypes.c_void_p(0x10000)   # never dereferenced: every case fails validation first
    assert lib.gdn2_gemm_phase_probe(2, 1, 1, ws, 256, None) == -2
    assert lib.gdn2_gemm_phase_probe(0, 0, 1, ws, 256, None) == -2
    assert lib.gdn2_gemm_phase_probe(0, 1, 0, ws, 256, None) == -2
    assert lib.gdn2_gemm_phase_probe(0, 1, 1, None, 256, None) == -5
    assert lib.gdn2_gemm_phase_probe(0, 1, 1, ws, 255, None) == -5
    assert lib.gdn2_gemm_phase_probe(1, 1, 1, ctypes.c_void_p(0x10004), 256, None) == -7


def test_edge_maps_and_rms_norm_validation(lib):
    f = ctypes.c_void_p(0x10000)   # never dereferenced: every case fails validation first
    assert lib.gdn2_layer_edge_maps(*(f,) * 10, -1, 1, 1, 128, 128, None) == -2
    assert lib.gdn2_layer_edge_maps(*(f,) * 10, 1, 1, 1, 96, 128, None) == -4
    assert lib.gdn2_layer_edge_maps(*(f,) * 9, None, 1, 1, 1, 128, 128, None) == -1
    assert lib.gdn2_layer_edge_maps(*(f,) * 9, ctypes.c_void_p(0x10008), 1, 1, 1, 128, 128, None) == -7
    assert lib.gdn2_layer_edge_maps(*(f,) * 10, 0, 1, 1, 128, 128, None) == 0
    assert lib.gdn2_rms_norm(f, f, -1, 128, None) == -2
    assert lib.gdn2_rms_norm(f, f, 1, 32, None) == -4
    assert lib.gdn2_rms_norm(None, f, 1, 128, None) == -1
    assert lib.gdn2_rms_norm(f, ctypes.c_void_p(0x10004), 1, 128, None) == -7
    assert lib.gdn2_rms_norm(f, f, 0, 128, None) == 0
