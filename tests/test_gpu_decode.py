"""Decode parity: split-KV decode through the C ABI against the float64 oracle.

Caches hold arbitrary seeded rows (standing for already rotated keys); the
oracle receives the same rows as a token-indexed history.  Local layers use a
ring of W slots (token t in slot t % W); slots that hold no visible token are
filled with a large constant, so reading one would break parity.
"""
import numpy as np
import pytest
import torch

import global_gqa_b200 as g3
import inputs
from oracle import attention as O
from gpu_helpers import assert_close, dev, to_dev

pytestmark = pytest.mark.gpu

JUNK = 300.0


def _build_cache(B, Hkv, D, lens, kind, W, cap, seed, layer):
    """Device caches plus the per-sequence histories the oracle sees."""
    kc = torch.full((B, Hkv, cap, D), JUNK, dtype=torch.bfloat16)
    vc = torch.full((B, Hkv, cap, D), JUNK, dtype=torch.bfloat16)
    hist_k, hist_v, starts = [], [], []
    for b in range(B):
        L = int(lens[b])
        t0 = 0 if kind == O.GLOBAL else max(0, L - W)
        h = inputs.cache_history(L - 1 - t0, Hkv, D, seed=seed, layer=layer, batch=b)
        for i, t in enumerate(range(t0, L - 1)):
            slot = t if kind == O.GLOBAL else t % W
            kc[b, :, slot] = h["k"][i]
            vc[b, :, slot] = h["v"][i]
        hist_k.append(h["k"])
        hist_v.append(h["v"])
        starts.append(t0)
    return kc, vc, hist_k, hist_v, starts


def _run_case(B, Hq, Hkv, D, lens, kind, W, base, interp, seed=0, layer=0, cap=None, max_len=None):
    lens = np.asarray(lens)
    cap = cap or (W if kind == O.LOCAL else int(lens.max()) + 5)
    max_len = max_len or int(lens.max())
    x = inputs.decode_step_inputs(B, Hq, Hkv, D, seed=seed, layer=layer)
    kc, vc, hk, hv, starts = _build_cache(B, Hkv, D, lens, kind, W, cap, seed, layer)
    xd = to_dev(x)
    kcd, vcd = kc.to(dev()), vc.to(dev())
    sl = torch.tensor(lens, dtype=torch.int32, device=dev())
    out = g3.decode(xd["q"], xd["k_new"], xd["v_new"], xd["q_gamma"], xd["k_gamma"], kcd, vcd, sl, max_len,
                    kind, W, base, interp)
    assert g3.check_device_error(g3.workspace(0, dev(), tag="decode")) == 0
    ref, k_hat = O.decode(x["q"], x["k_new"], x["v_new"], x["q_gamma"], x["k_gamma"], lens, hk, hv, starts,
                          kind, W, base, interp)
    assert_close(out, ref)
    # the new token's rotated key and its value were written to its slot
    kcc = kcd.double().cpu().numpy()
    vcc = vcd.double().cpu().numpy()
    for b in range(B):
        slot = (lens[b] - 1) if kind == O.GLOBAL else (lens[b] - 1) % W
        np.testing.assert_allclose(kcc[b, :, slot], k_hat[b], atol=3e-2, rtol=1e-2)
        np.testing.assert_array_equal(vcc[b, :, slot], x["v_new"][b].double().numpy())
    return out, kcd, vcd


SWEEP = [
    # B, Hq, Hkv, D, lens, kind, W
    (3, 4, 2, 128, [1, 2, 511], O.GLOBAL, 1024),
    (3, 4, 2, 128, [512, 513, 1025], O.GLOBAL, 1024),
    (2, 4, 1, 64, [5000, 2049], O.GLOBAL, 1024),
    (2, 2, 2, 64, [1, 1023], O.LOCAL, 1024),
    (3, 4, 2, 128, [1024, 1025, 2049], O.LOCAL, 1024),
    (2, 8, 2, 128, [3, 100], O.LOCAL, 7),
    (2, 4, 4, 128, [700, 9000], O.LOCAL, 1024),
    # Gemma 3 1B attention shapes: 4 query heads, 1 kv head, head_dim 256
    (2, 4, 1, 256, [1, 4097], O.GLOBAL, 512),
    (3, 4, 1, 256, [511, 1025, 2000], O.LOCAL, 512),
]


@pytest.mark.parametrize("case", SWEEP, ids=[f"D{c[3]}_G{c[1]//c[2]}_k{c[5]}_W{c[6]}_L{c[4][-1]}" for c in SWEEP])
def test_decode_sweep(case):
    B, Hq, Hkv, D, lens, kind, W = case
    base, interp = (1e4, 1.0) if kind == O.LOCAL else (1e6, 8.0)
    _run_case(B, Hq, Hkv, D, lens, kind, W, base, interp, seed=1, layer=len(lens))


def test_decode_ring_permutation_invariant():
    """Permuting the ring's slots (except the one the new token takes) changes nothing."""
    B, Hq, Hkv, D, W = 2, 4, 2, 128, 1024
    lens = np.array([3000, 1500])
    out, kcd, vcd = _run_case(B, Hq, Hkv, D, lens, O.LOCAL, W, 1e4, 1.0, seed=2)
    x = to_dev(inputs.decode_step_inputs(B, Hq, Hkv, D, seed=2, layer=0))
    rng = np.random.default_rng(0)
    kp, vp = kcd.clone(), vcd.clone()
    for b in range(B):
        fixed = (lens[b] - 1) % W
        others = np.array([s for s in range(W) if s != fixed])
        perm = others[rng.permutation(others.size)]
        idx = torch.as_tensor(others, device=dev())
        src = torch.as_tensor(perm, device=dev())
        kp[b][:, idx] = kcd[b][:, src]
        vp[b][:, idx] = vcd[b][:, src]
    sl = torch.tensor(lens, dtype=torch.int32, device=dev())
    out2 = g3.decode(x["q"], x["k_new"], x["v_new"], x["q_gamma"], x["k_gamma"], kp, vp, sl, int(lens.max()),
                     O.LOCAL, W, 1e4, 1.0)
    d = (out2.float() - out.float()).abs().max().item()
    assert d <= 1e-2, d


def test_decode_equals_last_prefill_row():
    """GPU decode at L equals row L-1 of a GPU prefill over the same L tokens."""
    B, S, Hq, Hkv, D = 2, 1500, 4, 2, 128
    for kind, W, base, interp in [(O.LOCAL, 1024, 1e4, 1.0), (O.GLOBAL, 1024, 1e6, 8.0)]:
        x = to_dev(inputs.prefill_layer_inputs(B, S, Hq, Hkv, D, seed=9))
        full = g3.prefill(x["q"], x["k"], x["v"], x["q_gamma"], x["k_gamma"], x["positions"], kind, W, base,
                          interp)
        cap = W if kind == O.LOCAL else S
        kc = torch.zeros(B, Hkv, cap, D, dtype=torch.bfloat16, device=dev())
        vc = torch.zeros_like(kc)
        g3.prefill(x["q"][:, :S - 1].contiguous(), x["k"][:, :S - 1].contiguous(), x["v"][:, :S - 1].contiguous(),
                   x["q_gamma"], x["k_gamma"], x["positions"][:, :S - 1].contiguous(), kind, W, base, interp,
                   k_cache=kc, v_cache=vc)
        sl = torch.full((B,), S, dtype=torch.int32, device=dev())
        dec = g3.decode(x["q"][:, S - 1].contiguous(), x["k"][:, S - 1].contiguous(),
                        x["v"][:, S - 1].contiguous(), x["q_gamma"], x["k_gamma"], kc, vc, sl, S, kind, W,
                        base, interp)
        d = (dec.float() - full[:, S - 1].float()).abs().max().item()
        assert d <= 2e-2, (kind, d)


def test_decode_bad_lengths_zero_rows_and_status():
    B, Hq, Hkv, D, W = 3, 4, 2, 64, 1024
    x = to_dev(inputs.decode_step_inputs(B, Hq, Hkv, D, seed=4))
    cap = 600
    kc = torch.ones(B, Hkv, cap, D, dtype=torch.bfloat16, device=dev())
    vc = torch.ones_like(kc)
    sl = torch.tensor([0, 601, 10], dtype=torch.int32, device=dev())
    ws = torch.empty(g3.decode_workspace_size(B, Hq, Hkv, D, 700), dtype=torch.uint8, device=dev())
    out = g3.decode(x["q"], x["k_new"], x["v_new"], x["q_gamma"], x["k_gamma"], kc, vc, sl, 700, O.GLOBAL, W,
                    1e6, 8.0, ws=ws)
    assert g3.check_device_error(ws) == 1
    o = out.float().cpu()
    assert (o[0] == 0).all() and (o[1] == 0).all() and o[2].abs().sum() > 0
    assert (kc[1].float() == 1).all()


def test_decode_full_size_sampled():
    """The 64-sequence, up-to-128K-token decode workload, every layer of the block.

    All sequences run; six of them are checked against the oracle.
    """
    cfg = inputs.DECODE_B64
    B, Hq, Hkv, D = cfg.B, cfg.Hq, cfg.Hkv, cfg.D
    lens = inputs.decode_lengths(B, cfg.len_lo, cfg.len_hi, cfg.seed)
    check = [int(i) for i in np.argsort(lens.numpy())[[0, 1, B // 2, B - 2, B - 1]]] + [7]
    blk = cfg.block()
    sl = lens.to(dev())
    for li in (0, 5):
        L = blk[li]
        cap = cfg.window if L.kind == O.LOCAL else cfg.global_capacity
        kc = torch.empty(B, Hkv, cap, D, dtype=torch.bfloat16, device=dev())
        vc = torch.empty_like(kc)
        inputs.device_fill_normal_bf16(kc, inputs.seed_for(cfg.seed, li, inputs.T_KC))
        inputs.device_fill_normal_bf16(vc, inputs.seed_for(cfg.seed, li, inputs.T_VC))
        x = inputs.decode_step_inputs(B, Hq, Hkv, D, seed=cfg.seed, layer=li)
        hk, hv, starts = [], [], []
        for b in check:
            Lb = int(lens[b])
            t0 = 0 if L.kind == O.GLOBAL else max(0, Lb - cfg.window)
            toks = np.arange(t0, Lb - 1)
            slots = toks if L.kind == O.GLOBAL else toks % cfg.window
            idx = torch.as_tensor(slots, device=dev())
            hk.append(kc[b][:, idx].permute(1, 0, 2).cpu())
            hv.append(vc[b][:, idx].permute(1, 0, 2).cpu())
            starts.append(t0)
        xd = to_dev(x)
        out = g3.decode(xd["q"], xd["k_new"], xd["v_new"], xd["q_gamma"], xd["k_gamma"], kc, vc, sl,
                        cfg.len_hi, L.kind, L.window, L.rope_base, L.interp)
        assert g3.check_device_error(g3.workspace(0, dev(), tag="decode")) == 0
        sub = {k: v[check] for k, v in x.items() if k in ("q", "k_new", "v_new")}
        ref, _ = O.decode(sub["q"], sub["k_new"], sub["v_new"], x["q_gamma"], x["k_gamma"], lens[check].numpy(),
                          hk, hv, starts, L.kind, L.window, L.rope_base, L.interp)
        assert_close(out[check], ref, what=f"decode layer {li}")
        del kc, vc
        torch.cuda.empty_cache()


def test_decode_medium_global():
    """8 sequences of 16K-32K tokens on a global layer (~2 GB of cache, larger than
    L2): the DRAM traffic of this call is what the decode profile scales; three
    sequences are checked against the oracle."""
    B, Hq, Hkv, D, cap = 8, 32, 16, 128, 32768
    lens = inputs.decode_lengths(B, 16384, cap, seed=3)
    sl = lens.to(dev())
    kc = torch.empty(B, Hkv, cap, D, dtype=torch.bfloat16, device=dev())
    vc = torch.empty_like(kc)
    inputs.device_fill_normal_bf16(kc, 31)
    inputs.device_fill_normal_bf16(vc, 32)
    x = inputs.decode_step_inputs(B, Hq, Hkv, D, seed=3, layer=5)
    xd = to_dev(x)
    out = g3.decode(xd["q"], xd["k_new"], xd["v_new"], xd["q_gamma"], xd["k_gamma"], kc, vc, sl, cap, O.GLOBAL,
                    cap, 1e6, 8.0)
    assert g3.check_device_error(g3.workspace(0, dev(), tag="decode")) == 0
    check = [0, 3, 7]
    hk = [kc[b][:, :int(lens[b]) - 1].permute(1, 0, 2).cpu() for b in check]
    hv = [vc[b][:, :int(lens[b]) - 1].permute(1, 0, 2).cpu() for b in check]
    sub = {k: v[check] for k, v in x.items() if k in ("q", "k_new", "v_new")}
    ref, _ = O.decode(sub["q"], sub["k_new"], sub["v_new"], x["q_gamma"], x["k_gamma"], lens[check].numpy(), hk, hv,
                      [0] * len(check), O.GLOBAL, cap, 1e6, 8.0)
    assert_close(out[check], ref, what="decode medium")
