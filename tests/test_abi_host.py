"""Host-side checks of the C ABI (no GPU needed, no compute launched).

The library must load, export every function include/g3attn.h declares and
reject bad arguments on the host before touching the device.
"""
import ctypes
import os

import numpy as np
import pytest

import global_gqa_b200 as g3
from global_gqa_b200 import metrics
from oracle import attention as O

FAKE = 0x1000  # never dereferenced: every call below fails validation first


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(g3.LIB_PATH):
        from global_gqa_b200 import build
        build.build()
    return g3.lib()


def test_exports_every_declared_symbol(lib):
    names = g3.header_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(g3._SIGS), "binding and header disagree"


def test_status_strings(lib):
    for code in range(6):
        s = lib.g3attn_status_string(code)
        assert s and s != b"unknown status"
    assert lib.g3attn_status_string(99) == b"unknown status"


def test_workspace_sizes(lib):
    assert lib.g3attn_prefill_workspace_size(0, 1, 1, 1, 64) == 0
    n = lib.g3attn_prefill_workspace_size(1, 8192, 32, 16, 128)
    assert n >= 8192 * (32 + 16) * 128 * 2 + 2 * 8192 * 4
    assert n % 1024 == 0
    d = lib.g3attn_decode_workspace_size(64, 32, 16, 128, 131072)
    assert d >= 64 * 32 * 256 * 128 * 4
    assert lib.g3attn_decode_workspace_size(1, 1, 1, 64, 0) == 0


def _prefill(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, qg=FAKE, kg=FAKE, pos=FAKE, kind=0, window=1024, base=1e4, interp=1.0,
             spans=None, n_spans=0, B=1, S=128, Hq=4, Hkv=2, D=64, out=FAKE, lse=None, kc=None, vc=None,
             cap=0, ws=FAKE * 256, wsb=1 << 40, stream=None)
    a.update(kw)
    return lib.g3attn_prefill(a["q"], a["k"], a["v"], a["qg"], a["kg"], a["pos"], a["kind"], a["window"],
                              a["base"], a["interp"], a["spans"], a["n_spans"], a["B"], a["S"], a["Hq"],
                              a["Hkv"], a["D"], a["out"], a["lse"], a["kc"], a["vc"], a["cap"], a["ws"],
                              a["wsb"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), 1), (dict(out=None), 1), (dict(B=0), 1), (dict(S=0), 1),
    (dict(Hq=3, Hkv=2), 1), (dict(kind=7), 1), (dict(window=0), 1), (dict(base=0.0), 1),
    (dict(base=float("inf")), 1), (dict(interp=0.0), 1), (dict(n_spans=2), 1),
    (dict(spans=FAKE, n_spans=0), 1), (dict(q=FAKE + 2), 1), (dict(kc=FAKE), 1),
    (dict(kc=FAKE, vc=FAKE, cap=100), 1), (dict(kind=1, kc=FAKE, vc=FAKE, cap=64), 1),
    (dict(D=96), 2), (dict(D=512), 2), (dict(ws=None), 3), (dict(ws=FAKE * 256 + 16), 3), (dict(wsb=100), 3),
])
def test_prefill_rejects_on_host(lib, kw, code):
    assert _prefill(lib, **kw) == code
    assert lib.g3attn_last_error() != b""


def _decode(lib, **kw):
    a = dict(q=FAKE, kn=FAKE, vn=FAKE, qg=FAKE, kg=FAKE, kc=FAKE, vc=FAKE, cap=1024, lens=FAKE, maxlen=4096,
             kind=0, window=1024, base=1e4, interp=1.0, B=2, Hq=4, Hkv=2, D=128, out=FAKE, ws=FAKE * 256,
             wsb=1 << 40, stream=None)
    a.update(kw)
    return lib.g3attn_decode(a["q"], a["kn"], a["vn"], a["qg"], a["kg"], a["kc"], a["vc"], a["cap"], a["lens"],
                             a["maxlen"], a["kind"], a["window"], a["base"], a["interp"], a["B"], a["Hq"],
                             a["Hkv"], a["D"], a["out"], a["ws"], a["wsb"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(kc=None), 1), (dict(lens=None), 1), (dict(B=0), 1), (dict(maxlen=0), 1), (dict(cap=512), 1),
    (dict(Hq=6, Hkv=4), 1), (dict(kind=3), 1), (dict(interp=-1.0), 1), (dict(kc=FAKE + 8), 1),
    (dict(D=80), 2), (dict(Hq=16, Hkv=2), 2), (dict(wsb=64), 3), (dict(ws=None), 3),
])
def test_decode_rejects_on_host(lib, kw, code):
    assert _decode(lib, **kw) == code


def _chunk(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, qg=FAKE, kg=FAKE, pos=FAKE, kc=FAKE, vc=FAKE, cap=1024, start=100, kind=0,
             window=1024, base=1e4, interp=1.0, spans=None, n_spans=0, B=1, C=128, Hq=4, Hkv=2, D=128, out=FAKE,
             lse=None, ws=FAKE * 256, wsb=1 << 40, stream=None)
    a.update(kw)
    return lib.g3attn_prefill_chunk(a["q"], a["k"], a["v"], a["qg"], a["kg"], a["pos"], a["kc"], a["vc"], a["cap"],
                                    a["start"], a["kind"], a["window"], a["base"], a["interp"], a["spans"],
                                    a["n_spans"], a["B"], a["C"], a["Hq"], a["Hkv"], a["D"], a["out"], a["lse"],
                                    a["ws"], a["wsb"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(kc=None), 1), (dict(start=-1), 1), (dict(C=0), 1), (dict(cap=512), 1),
    (dict(kind=1, cap=200), 1), (dict(Hq=3), 1), (dict(vc=FAKE + 8), 1), (dict(n_spans=1), 1),
    (dict(D=96), 2), (dict(ws=None), 3), (dict(wsb=1000), 3),
])
def test_prefill_chunk_rejects_on_host(lib, kw, code):
    assert _chunk(lib, **kw) == code
    assert lib.g3attn_last_error() != b""


def test_prefill_chunk_workspace_sizes(lib):
    assert lib.g3attn_prefill_chunk_workspace_size(1, 0, 4, 2, 128, 0, 0, 1024) == 0
    assert lib.g3attn_prefill_chunk_workspace_size(1, 16, 4, 2, 128, -1, 0, 1024) == 0
    loc = lib.g3attn_prefill_chunk_workspace_size(1, 2048, 32, 16, 128, 6144, 0, 1024)
    glb = lib.g3attn_prefill_chunk_workspace_size(1, 2048, 32, 16, 128, 6144, 1, 1024)
    # a local chunk also holds its context: 1023 ring rows + the chunk, K and V
    assert loc >= glb + 2 * 16 * (1023 + 2048) * 128 * 2
    assert glb >= 2048 * 32 * 128 * 2 and glb % 1024 == 0


def _backward(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, qg=FAKE, kg=FAKE, pos=FAKE, kind=0, window=1024, base=1e4, interp=1.0,
             spans=None, n_spans=0, B=1, S=256, Hq=4, Hkv=2, D=128, out=FAKE, lse=FAKE, dout=FAKE, dq=FAKE,
             dk=FAKE, dv=FAKE, dqg=FAKE, dkg=FAKE, ws=FAKE * 256, wsb=1 << 40, stream=None)
    a.update(kw)
    return lib.g3attn_prefill_backward(a["q"], a["k"], a["v"], a["qg"], a["kg"], a["pos"], a["kind"], a["window"],
                                       a["base"], a["interp"], a["spans"], a["n_spans"], a["B"], a["S"], a["Hq"],
                                       a["Hkv"], a["D"], a["out"], a["lse"], a["dout"], a["dq"], a["dk"], a["dv"],
                                       a["dqg"], a["dkg"], a["ws"], a["wsb"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(lse=None), 1), (dict(dout=None), 1), (dict(dq=None), 1), (dict(dk_gamma=None, dkg=None), 1),
    (dict(B=0), 1), (dict(Hq=3), 1), (dict(kind=5), 1), (dict(window=0), 1), (dict(interp=float("nan")), 1),
    (dict(n_spans=1), 1), (dict(dv=FAKE + 8), 1), (dict(dout=FAKE + 2), 1),
    (dict(D=512), 2), (dict(D=96), 2), (dict(ws=None), 3), (dict(ws=FAKE * 256 + 64), 3), (dict(wsb=4096), 3),
])
def test_prefill_backward_rejects_on_host(lib, kw, code):
    kw.pop("dk_gamma", None)
    assert _backward(lib, **kw) == code
    assert lib.g3attn_last_error() != b""


def test_prefill_backward_workspace_sizes(lib):
    assert lib.g3attn_prefill_backward_workspace_size(1, 0, 4, 2, 128) == 0
    fwd = lib.g3attn_prefill_workspace_size(1, 8192, 32, 16, 128)
    bwd = lib.g3attn_prefill_backward_workspace_size(1, 8192, 32, 16, 128)
    # the forward buffers plus fp32 gradients of the rotated q and k
    assert bwd >= fwd + 8192 * (32 + 16) * 128 * 4
    assert bwd % 1024 == 0


def _soft(lib, **kw):
    a = dict(p=FAKE, g=FAKE, B=2, gh=64, gw=64, F=1152, pool=4, out=FAKE, stream=None)
    a.update(kw)
    return lib.g3attn_soft_tokens(a["p"], a["g"], a["B"], a["gh"], a["gw"], a["F"], a["pool"], a["out"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(p=None), 1), (dict(out=None), 1), (dict(B=0), 1), (dict(F=4), 1), (dict(gh=62), 1),
    (dict(g=FAKE + 4), 1), (dict(F=12), 2), (dict(F=8200), 2), (dict(pool=3, gh=63, gw=63), 2),
])
def test_soft_tokens_rejects_on_host(lib, kw, code):
    assert _soft(lib, **kw) == code
    assert lib.g3attn_last_error() != b""


def test_check_device_error_null(lib):
    assert lib.g3attn_check_device_error(None, None) == 3


def test_trace_toggle(lib):
    assert lib.g3attn_trace_enable(1) == 0
    assert lib.g3attn_trace_collect(None, 0) == 0
    assert lib.g3attn_trace_enable(0) == 0


def test_python_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(1, 4, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        g3.prefill(q, q[:, :, :1], q[:, :, :1], torch.ones(64), torch.ones(64),
                   torch.zeros(1, 4, dtype=torch.int32), 0, 1024, 1e4, 1.0)


# ---------------------------------------------------- FLOP accounting vs oracle
@pytest.mark.parametrize("S,kind,W,spans", [
    (50, 0, 7, None), (50, 1, 7, None), (64, 0, 5, [[3, 20], [20, 22], [40, 64]]),
    (33, 1, 1, [[0, 33]]), (70, 0, 1000, [[10, 11]]),
])
def test_visible_pairs_match_oracle_enumeration(S, kind, W, spans):
    assert metrics.visible_pairs(S, kind, W, spans) == O.unmasked_pairs(S, kind, W, spans)


def test_block_flops_of_8k_block():
    import inputs
    c = inputs.BLOCK_8K
    f = metrics.block_flops(c.B, c.S, c.Hq, c.D, c.block())
    local = 8192 * 1024 - 1023 * 1024 // 2
    glob = 8192 * 8193 // 2
    assert f == 4 * 128 * 32 * (5 * local + glob)


def test_fault_injection_only_in_the_test_build(lib):
    """The withheld-arrival hook and the 20 ms wait limit exist only in the
    test-only library under _build/; the product library has neither."""
    from global_gqa_b200 import build as B
    assert not hasattr(lib, "g3attn_test_withhold_s_commit")
    assert not any("FAULT" in f or "TIMEOUT" in f for f in B.FLAGS)
    assert os.path.dirname(B.FAULT_LIB) != os.path.dirname(B.LIB)
    path = B.build_fault_inject()
    test_lib = ctypes.CDLL(path)
    assert hasattr(test_lib, "g3attn_test_withhold_s_commit")
