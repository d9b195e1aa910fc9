"""g3attn_decode_no_alloc: decode for callers that cannot allocate device memory.

Some callers cannot hand the library a workspace: plugins whose host framework
owns all device memory, serving loops where a cudaMalloc (which can
synchronise the device) is forbidden, C callers without an allocator.  For
them the library keeps the decode scratch in a static device array.  This test
calls that entry point through the C ABI twice in a row and checks each result
against the regular g3attn_decode (which uses a caller workspace) within the
decode parity tolerance.  The file is named so pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import global_gqa_b200 as g3
import inputs

pytestmark = pytest.mark.gpu

ATOL, REL_L2 = 2e-2, 5e-3


def _close(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    assert np.isfinite(a).all()
    assert np.abs(a - b).max() <= ATOL
    assert np.linalg.norm(a - b) / np.linalg.norm(b) <= REL_L2


def _call_no_alloc(x, kc, vc, sl, max_len, kind, W, base, interp, out):
    B, Hq, D = x["q"].shape
    Hkv = x["k_new"].shape[1]
    st = torch.cuda.current_stream().cuda_stream
    return g3.lib().g3attn_decode_no_alloc(
        x["q"].data_ptr(), x["k_new"].data_ptr(), x["v_new"].data_ptr(), x["q_gamma"].data_ptr(),
        x["k_gamma"].data_ptr(), kc.data_ptr(), vc.data_ptr(), kc.shape[2], sl.data_ptr(), max_len, kind, W,
        ctypes.c_float(base), ctypes.c_float(interp), B, Hq, Hkv, D, out.data_ptr(), st)


@pytest.mark.parametrize("kind,W,base,interp,lens,cap", [
    (1, 1024, 1e6, 8.0, [700, 1500, 64], 2048),
    (0, 1024, 1e4, 1.0, [3000, 999, 1025], 1024),
])
def test_decode_no_alloc_matches_workspace_decode(kind, W, base, interp, lens, cap):
    dev = torch.device("cuda", 0)
    B, Hq, Hkv, D = len(lens), 4, 2, 128
    max_len = 4096
    x = {k: v.to(dev) for k, v in inputs.decode_step_inputs(B, Hq, Hkv, D, seed=21, layer=kind).items()}
    kc0 = torch.empty(B, Hkv, cap, D, dtype=torch.bfloat16, device=dev)
    vc0 = torch.empty_like(kc0)
    inputs.device_fill_normal_bf16(kc0, 5)
    inputs.device_fill_normal_bf16(vc0, 6)
    sl = torch.tensor(lens, dtype=torch.int32, device=dev)

    # regular entry point with a caller workspace
    kc_ref, vc_ref = kc0.clone(), vc0.clone()
    ref = g3.decode(x["q"], x["k_new"], x["v_new"], x["q_gamma"], x["k_gamma"], kc_ref, vc_ref, sl, max_len,
                    kind, W, base, interp)
    torch.cuda.synchronize()

    kc, vc = kc0.clone(), vc0.clone()
    for call in range(2):
        out = torch.full((B, Hq, D), float("nan"), dtype=torch.bfloat16, device=dev)
        st = _call_no_alloc(x, kc, vc, sl, max_len, kind, W, base, interp, out)
        assert st == 0, g3.lib().g3attn_last_error()
        torch.cuda.synchronize()
        _close(out, ref)
        assert torch.equal(kc, kc_ref) and torch.equal(vc, vc_ref)


def test_decode_no_alloc_local_layer_at_batched_decode_sizes():
    """A local layer of the 64-sequence decode (32/16 heads, contexts up to 128K):
    a query sees at most the 1024 ring slots, so the scratch is a couple of MB
    whatever max_seq_len is, and the call is accepted."""
    dev = torch.device("cuda", 0)
    B, Hq, Hkv, D, W, max_len = 64, 32, 16, 128, 1024, 131072
    x = {k: v.to(dev) for k, v in inputs.decode_step_inputs(B, Hq, Hkv, D, seed=4, layer=0).items()}
    kc0 = torch.empty(B, Hkv, W, D, dtype=torch.bfloat16, device=dev)
    vc0 = torch.empty_like(kc0)
    inputs.device_fill_normal_bf16(kc0, 7)
    inputs.device_fill_normal_bf16(vc0, 8)
    sl = inputs.decode_lengths(B, 4096, max_len, seed=4).to(dev)
    kc_ref, vc_ref = kc0.clone(), vc0.clone()
    ref = g3.decode(x["q"], x["k_new"], x["v_new"], x["q_gamma"], x["k_gamma"], kc_ref, vc_ref, sl, max_len,
                    0, W, 1e4, 1.0)
    torch.cuda.synchronize()
    kc, vc = kc0.clone(), vc0.clone()
    for call in range(2):
        out = torch.full((B, Hq, D), float("nan"), dtype=torch.bfloat16, device=dev)
        st = _call_no_alloc(x, kc, vc, sl, max_len, 0, W, 1e4, 1.0, out)
        assert st == 0, g3.lib().g3attn_last_error()
        torch.cuda.synchronize()
        _close(out, ref)
        assert torch.equal(kc, kc_ref) and torch.equal(vc, vc_ref)


def test_decode_no_alloc_rejects_sizes_beyond_its_array():
    dev = torch.device("cuda", 0)
    B, Hq, Hkv, D = 64, 32, 16, 128
    x = {k: v.to(dev) for k, v in inputs.decode_step_inputs(B, Hq, Hkv, D, seed=1).items()}
    kc = torch.zeros(B, Hkv, 16, D, dtype=torch.bfloat16, device=dev)
    sl = torch.ones(B, dtype=torch.int32, device=dev)
    out = torch.zeros(B, Hq, D, dtype=torch.bfloat16, device=dev)
    st = _call_no_alloc(x, kc, kc, sl, 131072, 1, 1024, 1e6, 8.0, out)
    assert st == 2
    assert b"static array" in g3.lib().g3attn_last_error()
