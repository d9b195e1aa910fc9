"""Chunked prefill parity: g3attn_prefill_chunk against the float64 oracle.

A chunk's rows must equal rows start .. start+C-1 of the whole prefill over
start + C tokens (the oracle's definition), and the cache it leaves behind must
equal the one a whole prefill with cache fill writes.  Tolerances as for
prefill: max |err| <= 2e-2, relative L2 <= 5e-3, lse within 2e-2.
"""
import numpy as np
import pytest
import torch

import global_gqa_b200 as g3
import inputs
from oracle import attention as O
from gpu_helpers import assert_close, dev, oracle_rows, to_dev, LSE_ATOL

pytestmark = pytest.mark.gpu

LOC, GLB = O.LOCAL, O.GLOBAL


def _spans(spans, B):
    if not spans:
        return None
    return torch.tensor([spans] * B, dtype=torch.int32)


def _caches(B, Hkv, D, kind, W, T):
    cap = W if kind == LOC else T + 37  # a global cache larger than needed
    k = torch.full((B, Hkv, cap, D), float("nan"), dtype=torch.bfloat16, device=dev())
    v = torch.full_like(k, float("nan"))
    return k, v


def _slice(xd, a, b):
    return {key: (t[:, a:b].contiguous() if key in ("q", "k", "v", "positions") else t) for key, t in xd.items()
            if key != "spans"}


def _run_chunks(xd, kind, W, base, interp, cuts, spans_all):
    """Prefill the first cut with g3attn_prefill (cache fill), then each later
    piece with g3attn_prefill_chunk; returns the concatenated outputs of the
    chunks (rows cuts[0]..T-1), their lse, and the caches."""
    B, T, Hq, D = xd["q"].shape
    Hkv = xd["k"].shape[2]
    kc, vc = _caches(B, Hkv, D, kind, W, T)
    outs, lses = [], []
    first = cuts[0]
    if first > 0:
        hist = [s for s in spans_all if s[1] <= first]
        x0 = _slice(xd, 0, first)
        g3.prefill(x0["q"], x0["k"], x0["v"], x0["q_gamma"], x0["k_gamma"], x0["positions"], kind, W, base,
                   interp, _spans(hist, B).to(dev()) if hist else None, k_cache=kc, v_cache=vc)
    bounds = list(cuts) + [T]
    for a, b in zip(bounds[:-1], bounds[1:]):
        xc = _slice(xd, a, b)
        sp = [s for s in spans_all if s[1] <= b]
        out, lse = g3.prefill_chunk(xc["q"], xc["k"], xc["v"], xc["q_gamma"], xc["k_gamma"], xc["positions"],
                                    kc, vc, a, kind, W, base, interp,
                                    _spans(sp, B).to(dev()) if sp else None, return_lse=True)
        assert g3.check_device_error(g3.workspace(0, dev())) == 0
        outs.append(out)
        lses.append(lse)
    return torch.cat(outs, dim=1), torch.cat(lses, dim=2), kc, vc


CASES = [
    # B, T, Hq, Hkv, D, kind, W, cuts (first = tokens prefilled whole), spans
    (1, 700, 4, 2, 128, LOC, 256, [300], []),
    (2, 1500, 4, 2, 128, LOC, 1024, [0, 700], [[100, 356], [760, 1016]]),
    (1, 2600, 8, 2, 128, LOC, 1024, [1100, 1300, 2599], []),
    (1, 2000, 4, 2, 128, GLB, 1024, [1000, 1777], [[300, 556]]),
    (2, 900, 4, 1, 64, GLB, 1024, [0, 129], []),
    (1, 1200, 4, 4, 64, LOC, 300, [500, 501], [[600, 700]]),
    (1, 1300, 4, 1, 256, LOC, 512, [640], []),
    (1, 1300, 4, 1, 256, GLB, 1024, [700], [[800, 1056]]),
]


@pytest.mark.parametrize("case", CASES, ids=[f"T{c[1]}_H{c[2]}x{c[3]}_D{c[4]}_k{c[5]}_W{c[6]}_cuts{len(c[7])}"
                                             for c in CASES])
def test_chunked_prefill(case):
    B, T, Hq, Hkv, D, kind, W, cuts, spans = case
    base, interp = (1e4, 1.0) if kind == LOC else (1e6, 8.0)
    xc = inputs.prefill_layer_inputs(B, T, Hq, Hkv, D, seed=11, layer=T % 7)
    xc["spans"] = _spans(spans, B)
    xd = to_dev(xc)
    out, lse, kc, vc = _run_chunks(xd, kind, W, base, interp, cuts, spans)
    rows = list(range(cuts[0], T))
    ref, ref_lse = oracle_rows(xc, kind, W, base, interp, rows=rows)
    assert_close(out, ref, what="chunk out")
    assert_close(lse, ref_lse, atol=LSE_ATOL, rel_l2=np.inf, what="chunk lse")

    # The cache equals the one a whole prefill with cache fill leaves.
    kw, vw = _caches(B, Hkv, D, kind, W, T)
    g3.prefill(xd["q"], xd["k"], xd["v"], xd["q_gamma"], xd["k_gamma"], xd["positions"], kind, W, base, interp,
               xd.get("spans"), k_cache=kw, v_cache=vw)
    n = min(T, W) if kind == LOC else T
    slots = [t % W for t in range(T - n, T)] if kind == LOC else list(range(T))
    idx = torch.as_tensor(slots, device=dev())
    assert torch.equal(kc[:, :, idx], kw[:, :, idx])
    assert torch.equal(vc[:, :, idx], vw[:, :, idx])


def test_chunk_equals_whole_prefill_on_gpu():
    """Chunks of a long local-layer prompt reproduce the whole prefill's rows."""
    B, T, Hq, Hkv, D, W = 1, 3000, 4, 2, 128, 1024
    xc = inputs.prefill_layer_inputs(B, T, Hq, Hkv, D, seed=5, layer=0)
    xd = to_dev(xc)
    whole = g3.prefill(xd["q"], xd["k"], xd["v"], xd["q_gamma"], xd["k_gamma"], xd["positions"], LOC, W, 1e4, 1.0)
    out, _, _, _ = _run_chunks(xd, LOC, W, 1e4, 1.0, [0, 512, 1024, 2047], [])
    assert_close(out, whole.double().cpu().numpy(), atol=2e-2, rel_l2=5e-3, what="chunks vs whole")


def test_chunk_rejects_span_across_boundary():
    """An image span with tokens on both sides of the chunk's end is reported."""
    B, T, Hq, Hkv, D, W = 1, 600, 2, 1, 64, 1024
    xc = inputs.prefill_layer_inputs(B, T, Hq, Hkv, D, seed=2, layer=0)
    xd = to_dev(xc)
    kc, vc = _caches(B, Hkv, D, GLB, W, T)
    x0 = _slice(xd, 0, 300)
    g3.prefill(x0["q"], x0["k"], x0["v"], x0["q_gamma"], x0["k_gamma"], x0["positions"], GLB, W, 1e6, 8.0,
               k_cache=kc, v_cache=vc)
    x1 = _slice(xd, 300, 400)
    bad = torch.tensor([[[350, 450]]], dtype=torch.int32, device=dev())
    g3.prefill_chunk(x1["q"], x1["k"], x1["v"], x1["q_gamma"], x1["k_gamma"], x1["positions"], kc, vc, 300, GLB,
                     W, 1e6, 8.0, bad)
    assert g3.check_device_error(g3.workspace(0, dev())) != 0
