"""Failure detection without a GPU fault: a bounded wait that runs out.

Every mbarrier wait of the attention kernels gives up after a time limit,
raises the CTA's abort flag, records G3_ERR_TIMEOUT in the workspace header,
waits (again with a limit) for its own copies and products in flight, frees
its tensor memory and returns.  The test-only build of the library (compiled
with G3_FAULT_INJECT and a 20 ms limit, never the product library) exports
g3attn_test_withhold_s_commit(cta): the next prefill makes the MMA thread of
that CTA skip one "S ready" arrival, a missing arrival and nothing else, so
the softmax warps of that CTA wait for a phase that never completes.  The
call must report G3_ERR_TIMEOUT, and the GPU must stay usable: a normal
prefill in the same process, with the same library, then matches the oracle.
"""
import ctypes
import os

import numpy as np
import pytest
import torch

import global_gqa_b200 as g3
import inputs
from global_gqa_b200 import build as B
from gpu_helpers import assert_close, dev, oracle_rows, run_prefill, to_dev

pytestmark = pytest.mark.gpu

G3_ERR_TIMEOUT = 5


@pytest.fixture()
def fault_lib():
    path = B.build_fault_inject()
    saved_lib, saved_path = g3._lib, g3.LIB_PATH
    g3._lib, g3.LIB_PATH = None, path
    try:
        h = g3.lib()
        h.g3attn_test_withhold_s_commit.argtypes = [ctypes.c_int32]
        h.g3attn_test_withhold_s_commit.restype = None
        yield h
    finally:
        g3._lib, g3.LIB_PATH = saved_lib, saved_path


@pytest.mark.parametrize("kind,base,interp", [(0, 1e4, 1.0), (1, 1e6, 8.0)], ids=["local", "global"])
def test_withheld_arrival_times_out_and_gpu_stays_usable(fault_lib, kind, base, interp):
    Bt, S, Hq, Hkv, D, W = 1, 1025, 4, 2, 128, 256
    xc = inputs.prefill_layer_inputs(Bt, S, Hq, Hkv, D, seed=3, layer=kind)
    xd = to_dev(xc)
    ws = torch.empty(g3.prefill_workspace_size(Bt, S, Hq, Hkv, D), dtype=torch.uint8, device=dev())
    assert os.path.samefile(g3.LIB_PATH, B.FAULT_LIB)

    fault_lib.g3attn_test_withhold_s_commit(3)          # CTA 3 exists: the grid has 18 CTAs here
    run_prefill(xd, kind, W, base, interp, return_lse=False, ws=ws)
    assert g3.check_device_error(ws) == G3_ERR_TIMEOUT

    # The hook is one-shot: the next call is a normal prefill, and it is right.
    out, lse = run_prefill(xd, kind, W, base, interp, ws=ws)
    assert g3.check_device_error(ws) == 0
    ref, ref_lse = oracle_rows(xc, kind, W, base, interp)
    assert_close(out, ref, what="prefill after a timed-out call")
    assert np.abs(lse.double().cpu().numpy() - ref_lse).max() <= 2e-2
