"""Prefill parity: the CUDA path through the C ABI against the float64 oracle.

Tolerances (bf16 inputs, fp32 accumulation): max |err| <= 2e-2 and relative
L2 <= 5e-3 on outputs; lse within 2e-2.  Full-size workloads compare sampled
rows (first and last tiles, window/tile/span edges, whole spans, random rows)
over all heads, in the launch configuration the benchmark uses.
"""
import numpy as np
import pytest
import torch

import global_gqa_b200 as g3
import inputs
from oracle import attention as O
from gpu_helpers import assert_close, dev, oracle_rows, run_prefill, sampled_rows, to_dev, LSE_ATOL

pytestmark = pytest.mark.gpu

LOC, GLB = O.LOCAL, O.GLOBAL

SWEEP = [
    # B, S, Hq, Hkv, D, kind, W, spans, base, interp
    (1, 1, 2, 1, 64, LOC, 1024, None, 1e4, 1.0),
    (1, 2, 2, 2, 128, GLB, 1024, None, 1e6, 8.0),
    (2, 127, 4, 2, 64, LOC, 7, None, 1e4, 1.0),
    (1, 128, 4, 2, 128, GLB, 1024, None, 1e6, 8.0),
    (1, 129, 4, 1, 128, LOC, 128, None, 1e4, 1.0),
    (2, 300, 2, 2, 64, LOC, 1, None, 1e4, 1.0),
    (1, 300, 4, 2, 128, LOC, 1, [[10, 40], [40, 41], [100, 299]], 1e4, 1.0),
    (1, 1023, 8, 2, 64, LOC, 1024, None, 1e4, 1.0),
    (1, 1025, 4, 2, 128, LOC, 1024, [[0, 256], [700, 956]], 1e4, 1.0),
    (2, 1025, 6, 3, 128, GLB, 1024, [[129, 385], [769, 1025]], 1e6, 8.0),
    (1, 3000, 4, 2, 128, LOC, 1024, None, 1e4, 1.0),
    (1, 3000, 4, 2, 64, GLB, 1024, [[1000, 1256]], 1e6, 1.0),
    (1, 777, 4, 4, 64, LOC, 300, None, 1e4, 1.0),
    (1, 2048, 8, 2, 128, GLB, 1024, None, 1e6, 8.0),
    # Gemma 3 1B attention shapes: 4 query heads, 1 kv head, head_dim 256
    (1, 300, 4, 1, 256, LOC, 512, [[10, 40], [100, 299]], 1e4, 1.0),
    (2, 1025, 4, 1, 256, LOC, 1024, [[0, 256]], 1e4, 1.0),
    (1, 2048, 4, 1, 256, GLB, 1024, None, 1e6, 8.0),
    (1, 129, 2, 2, 256, GLB, 1024, None, 1e6, 1.0),
]


def _spans_tensor(spans, B):
    if spans is None:
        return None
    return torch.tensor([spans] * B, dtype=torch.int32)


@pytest.mark.parametrize("case", SWEEP, ids=[f"B{c[0]}_S{c[1]}_H{c[2]}x{c[3]}_D{c[4]}_k{c[5]}_W{c[6]}"
                                             f"_sp{0 if c[7] is None else len(c[7])}" for c in SWEEP])
def test_prefill_sweep(case):
    B, S, Hq, Hkv, D, kind, W, spans, base, interp = case
    xc = inputs.prefill_layer_inputs(B, S, Hq, Hkv, D, seed=7, layer=S % 11)
    xc["spans"] = _spans_tensor(spans, B)
    xd = to_dev(xc)
    out, lse = run_prefill(xd, kind, W, base, interp)
    assert g3.check_device_error(g3.workspace(0, dev())) == 0
    ref, ref_lse = oracle_rows(xc, kind, W, base, interp)
    assert_close(out, ref)
    assert_close(lse, ref_lse, atol=LSE_ATOL, rel_l2=np.inf, what="lse")


WORK_ORDER = [
    # B, S, Hq, Hkv, D, spans: causal layers whose grid has both parts of the work order
    (2, 4000, 16, 8, 128, [[100, 356], [2000, 2256]]),   # two-head CTAs, 16 units, ragged last tile
    (1, 6100, 16, 4, 64, None),                          # two-head CTAs, G = 4: two head groups per kv head
    (1, 6100, 8, 2, 256, [[5000, 5256]]),                # one-head CTAs (head dim 256)
]


@pytest.mark.parametrize("case", WORK_ORDER, ids=[f"B{c[0]}_S{c[1]}_H{c[2]}x{c[3]}_D{c[4]}" for c in WORK_ORDER])
def test_causal_work_order_heavy_and_light_tiles(case):
    """On a causal layer the heavy query tiles of each (sequence, kv head, head
    group) unit run unit by unit and the light tiles of all units follow.
    These shapes have more query tiles per unit than the light tail holds on
    this GPU (at most one CTA per SM for these kernels, so the tail is at most
    sqrt(2 * tiles * SMs / units) tiles), so both parts run; every row of every
    head is compared."""
    B, S, Hq, Hkv, D, spans = case
    G = Hq // Hkv
    units = B * Hkv * (G // 2 if D <= 128 else G)
    nq = (S + 127) // 128
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert np.sqrt(2.0 * nq * sms / units) < nq - 2, "the case must reach the heavy part of the order"
    xc = inputs.prefill_layer_inputs(B, S, Hq, Hkv, D, seed=11, layer=5)
    xc["spans"] = _spans_tensor(spans, B)
    xd = to_dev(xc)
    out, lse = run_prefill(xd, GLB, 1024, 1e6, 8.0)
    assert g3.check_device_error(g3.workspace(0, dev())) == 0
    ref, ref_lse = oracle_rows(xc, GLB, 1024, 1e6, 8.0)
    assert_close(out, ref)
    assert_close(lse, ref_lse, atol=LSE_ATOL, rel_l2=np.inf, what="lse")


def test_prefill_positions_shifted():
    """Shifting every position by a constant leaves the output unchanged."""
    B, S, Hq, Hkv, D = 1, 600, 4, 2, 128
    xc = inputs.prefill_layer_inputs(B, S, Hq, Hkv, D, seed=3, layer=1)
    xd = to_dev(xc)
    a = run_prefill(xd, GLB, 1024, 1e6, 8.0, return_lse=False)
    xd2 = dict(xd)
    xd2["positions"] = (xd["positions"] + 4096).contiguous()
    b = run_prefill(xd2, GLB, 1024, 1e6, 8.0, return_lse=False)
    assert_close(b, a.double().cpu().numpy(), atol=2e-2, rel_l2=5e-3)


def _block_parity(cfg, rows_fn, layers=range(6)):
    blk = cfg.block()
    for li in layers:
        L = blk[li]
        xc = inputs.config_layer_inputs(cfg, li)
        xd = to_dev(xc)
        out, lse = run_prefill(xd, L.kind, L.window, L.rope_base, L.interp)
        assert g3.check_device_error(g3.workspace(0, dev())) == 0
        rows = rows_fn(cfg, xc)
        ref, ref_lse = oracle_rows(xc, L.kind, L.window, L.rope_base, L.interp, rows=rows)
        got = out[:, torch.as_tensor(rows, device=out.device)]
        assert_close(got, ref, what=f"{cfg.name} layer {li} out")
        assert_close(lse[:, :, torch.as_tensor(rows, device=out.device)], ref_lse, atol=LSE_ATOL,
                     rel_l2=np.inf, what=f"{cfg.name} layer {li} lse")
        del xd, out, lse


def test_tiny_block_all_rows():
    _block_parity(inputs.TINY_BLOCK, lambda c, x: np.arange(c.S))


def test_8k_block_sampled_rows():
    _block_parity(inputs.BLOCK_8K, lambda c, x: sampled_rows(c.S, 1024, n_random=512))


def test_mixed_32k_sampled_rows():
    def rows(c, x):
        sp = x["spans"][0].numpy()
        r = sampled_rows(c.S, 1024, sp, n_random=1024)
        return r
    _block_parity(inputs.MIXED_32K, rows, layers=[0, 5])


@pytest.mark.parametrize("layer", [0, 5])
def test_long_128k_sampled_rows(layer):
    _block_parity(inputs.LONG_128K, lambda c, x: sampled_rows(c.S, 1024, n_random=1024), layers=[layer])


# -------------------------------------------------------------- cache fill
@pytest.mark.parametrize("kind,S,W", [(LOC, 3000, 1024), (LOC, 500, 1024), (GLB, 700, 1024)])
def test_prefill_fills_cache(kind, S, W):
    B, Hq, Hkv, D = 2, 4, 2, 128
    base, interp = (1e4, 1.0) if kind == LOC else (1e6, 8.0)
    xc = inputs.prefill_layer_inputs(B, S, Hq, Hkv, D, seed=5, layer=2)
    xd = to_dev(xc)
    cap = W if kind == LOC else S + 37
    kc = torch.full((B, Hkv, cap, D), 7.0, dtype=torch.bfloat16, device=dev())
    vc = torch.full_like(kc, 7.0)
    run_prefill(xd, kind, W, base, interp, return_lse=False, k_cache=kc, v_cache=vc)
    torch.cuda.synchronize()
    kh = O.rope(O.qk_rmsnorm(xc["k"], xc["k_gamma"]), xc["positions"].double().numpy(), base, interp)
    kcc, vcc = kc.double().cpu().numpy(), vc.double().cpu().numpy()
    tokens = range(S) if kind == GLB else range(max(0, S - W), S)
    for t in tokens:
        slot = t if kind == GLB else t % W
        np.testing.assert_allclose(kcc[:, :, slot], kh[:, t], atol=3e-2, rtol=1e-2)
        np.testing.assert_array_equal(vcc[:, :, slot], xc["v"][:, t].double().numpy())
    untouched = range(S, cap) if kind == GLB else range(S, W)
    for slot in untouched:
        assert (kcc[:, :, slot] == 7.0).all() and (vcc[:, :, slot] == 7.0).all()


# -------------------------------------------- inputs written just before
@pytest.mark.parametrize("kind", [LOC, GLB], ids=["local", "global"])
def test_prefill_reads_inputs_written_just_before(kind):
    """The prologue and attention kernels start as programmatic dependents of
    the work before them; whatever kernel produced q, k and v right before the
    call (here an elementwise torch kernel on the same stream, no
    synchronisation) must be complete before they are read.  Two input sets
    alternate over 20 calls and every output must equal its set's reference
    bit for bit."""
    B, S, Hq, Hkv, D = 1, 2048, 8, 4, 128
    base, interp = (1e4, 1.0) if kind == LOC else (1e6, 8.0)
    srcs = [to_dev(inputs.prefill_layer_inputs(B, S, Hq, Hkv, D, seed=s, layer=3)) for s in (11, 12)]
    x = {k: (torch.empty_like(v) if k in ("q", "k", "v") else v) for k, v in srcs[0].items()}
    refs = []
    for src in srcs:
        for k in ("q", "k", "v"):
            x[k].copy_(src[k])
        refs.append(run_prefill(x, kind, 1024, base, interp, return_lse=False).clone())
    torch.cuda.synchronize()
    assert not torch.equal(refs[0], refs[1])
    outs = []
    for i in range(20):
        src = srcs[i % 2]
        for k in ("q", "k", "v"):
            torch.add(src[k], 0, out=x[k])  # a kernel on the call's stream, not a copy-engine transfer
        outs.append(run_prefill(x, kind, 1024, base, interp, return_lse=False))
    torch.cuda.synchronize()
    assert g3.check_device_error(g3.workspace(0, dev())) == 0
    for i, out in enumerate(outs):
        assert torch.equal(out, refs[i % 2]), f"call {i} read inputs of the wrong set"


# ------------------------------------------------------- device-side errors
def test_bad_spans_reported_on_device():
    B, S, Hq, Hkv, D = 1, 256, 2, 1, 64
    xc = inputs.prefill_layer_inputs(B, S, Hq, Hkv, D, seed=1)
    xc["spans"] = torch.tensor([[[10, 50], [40, 60]]], dtype=torch.int32)   # overlapping
    xd = to_dev(xc)
    ws = torch.empty(g3.prefill_workspace_size(B, S, Hq, Hkv, D), dtype=torch.uint8, device=dev())
    run_prefill(xd, LOC, 16, 1e4, 1.0, ws=ws)
    assert g3.check_device_error(ws) == 1
    assert g3.check_device_error(ws) == 0   # read-and-clear


def test_cache_fill_with_positions_other_than_token_index_is_reported():
    """Decode rotates a new token by its index, so a prefill that fills a cache
    must have positions[b, t] == t; the prologue records anything else."""
    B, S, Hq, Hkv, D, W = 1, 300, 2, 1, 64, 128
    xc = inputs.prefill_layer_inputs(B, S, Hq, Hkv, D, seed=2)
    xc["positions"] = (xc["positions"] + 5).contiguous()
    xd = to_dev(xc)
    ws = torch.empty(g3.prefill_workspace_size(B, S, Hq, Hkv, D), dtype=torch.uint8, device=dev())
    kc = torch.zeros(B, Hkv, W, D, dtype=torch.bfloat16, device=dev())
    vc = torch.zeros_like(kc)
    run_prefill(xd, LOC, W, 1e4, 1.0, return_lse=False, ws=ws, k_cache=kc, v_cache=vc)
    assert g3.check_device_error(ws) == 1
    run_prefill(xd, LOC, W, 1e4, 1.0, return_lse=False, ws=ws)   # no cache: any positions are fine
    assert g3.check_device_error(ws) == 0


@pytest.mark.parametrize("kind", [LOC, GLB], ids=["local", "global"])
def test_prefill_1b_shapes_32k(kind):
    """Gemma 3 1B attention shapes (4 query heads, 1 kv head, head_dim 256) at a
    32K context, on sampled rows of all heads."""
    B, S, Hq, Hkv, D, W = 1, 32768, 4, 1, 256, 1024
    base, interp = (1e4, 1.0) if kind == LOC else (1e6, 8.0)
    xc = inputs.prefill_layer_inputs(B, S, Hq, Hkv, D, seed=0, layer=0 if kind == LOC else 5)
    xd = to_dev(xc)
    out, lse = run_prefill(xd, kind, W, base, interp)
    assert g3.check_device_error(g3.workspace(0, dev())) == 0
    rows = sampled_rows(S, W, n_random=128)
    ref, ref_lse = oracle_rows(xc, kind, W, base, interp, rows=rows)
    idx = torch.as_tensor(rows, device=out.device)
    assert_close(out[:, idx], ref, what="1B-shaped out")
    assert_close(lse[:, :, idx], ref_lse, atol=LSE_ATOL, rel_l2=np.inf, what="1B-shaped lse")
