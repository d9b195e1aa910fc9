"""Pins for the CPU oracle: checks against facts other than the oracle itself.

The pages print no worked numeric example for this attention, so the oracle
is pinned by the constants they print (tests/golden/gemma3_constants.txt),
closed forms, invariants the method must satisfy, brute-force enumeration on
tiny inputs and a library routine (torch SDPA in float64 with an explicit
boolean mask).  Each check_* function is also run against deliberately broken
copies of the oracle in test_oracle_mutations.py, to show the pins catch
plausible mistakes.
"""
import math
import os

import numpy as np
import pytest
import torch

import inputs
from oracle import attention as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "gemma3_constants.txt")
RNG = np.random.default_rng(1234)


def golden():
    vals = {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            name, value = line.split("|")[0].split()
            vals[name] = value
    return vals


def _bf16(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g).to(torch.bfloat16)


def _layer(B, S, Hq, Hkv, D, seed):
    q = _bf16((B, S, Hq, D), seed)
    k = _bf16((B, S, Hkv, D), seed + 1)
    v = _bf16((B, S, Hkv, D), seed + 2)
    g = torch.Generator().manual_seed(seed + 3)
    qg = 1 + 0.1 * torch.randn(D, generator=g)
    kg = 1 + 0.1 * torch.randn(D, generator=g)
    pos = torch.arange(S, dtype=torch.int32).repeat(B, 1)
    return q, k, v, qg, kg, pos


def _mask_by_words(S, kind, W, spans_b):
    """Visible sets built by enumeration from the sentences, not the oracle."""
    vis = np.zeros((S, S), dtype=bool)
    for i in range(S):
        lo = 0 if kind == O.GLOBAL else max(0, i - W + 1)
        for j in range(lo, i + 1):          # causal, within the window
            vis[i, j] = True
    if spans_b is not None:
        for st, en in spans_b:
            for i in range(st, en):         # every token of one image sees every other
                for j in range(st, en):
                    vis[i, j] = True
    return vis


def _sdpa64(qh, kh, v, vis):
    """torch SDPA in float64, kv heads repeated to the query heads."""
    B, S, Hq, D = qh.shape
    Hkv = kh.shape[2]
    G = Hq // Hkv
    qt = torch.from_numpy(qh).permute(0, 2, 1, 3)
    kt = torch.from_numpy(kh).permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    vt = torch.from_numpy(v).permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    m = torch.from_numpy(vis)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=m)
    return o.permute(0, 2, 1, 3).numpy()


# ------------------------------------------------------------------ golden --
def check_golden_block_and_shapes():
    g = golden()
    blk = inputs.gemma3_block()
    assert len(blk) == int(g["local_layers_per_global"]) + 1
    assert blk[0].kind == inputs.LOCAL and g["first_layer_kind"] == "local"
    assert [l.kind for l in blk] == [inputs.LOCAL] * 5 + [inputs.GLOBAL]
    assert all(l.window == int(g["local_window_tokens"]) for l in blk)
    assert blk[0].rope_base == float(g["local_rope_base"])
    assert blk[5].rope_base == float(g["global_rope_base"])
    assert inputs.IMAGE_SPAN_TOKENS == int(g["image_soft_tokens"])
    assert O.EPS == float(g["qk_norm_eps"])
    c = inputs.BLOCK_8K
    assert c.D == int(g["g27b_qk_norm_dim"])
    assert c.Hq == int(g["g27b_q_proj_out"]) // c.D
    assert c.Hkv == int(g["g27b_kv_proj_out"]) // c.D
    assert inputs.LONG_128K.S == int(g["context_tokens_large"])


def check_golden_local_window_edge():
    """A local query sees exactly the last 1024 tokens (itself included)."""
    W = int(golden()["local_window_tokens"])
    S = 2100
    sid = O.span_ids(S, None)
    row = O.allowed_row(2000, S, O.LOCAL, W, sid)
    idx = np.nonzero(row)[0]
    assert idx[0] == 2000 - W + 1 and idx[-1] == 2000 and idx.size == W
    row = O.allowed_row(2000, S, O.GLOBAL, W, sid)
    assert np.nonzero(row)[0].size == 2001


# ----------------------------------------------------------------- rmsnorm --
def check_rmsnorm_unit_rms():
    """mean((x_hat / gamma)^2) = ms / (ms + eps) exactly (closed form)."""
    x = RNG.standard_normal((7, 3, 64)) * 1e-3        # small so eps matters
    gam = 1 + 0.1 * RNG.standard_normal(64)
    y = O.qk_rmsnorm(x, gam)
    ms = np.mean(x * x, axis=-1)
    np.testing.assert_allclose(np.mean((y / gam) ** 2, axis=-1), ms / (ms + 1e-6), rtol=1e-12)


def check_rmsnorm_gamma_is_multiplier():
    x = RNG.standard_normal((5, 2, 32))
    gam = 1 + 0.1 * RNG.standard_normal(32)
    np.testing.assert_allclose(O.qk_rmsnorm(x, gam), O.qk_rmsnorm(x, np.ones(32)) * gam, rtol=1e-14)


# -------------------------------------------------------------------- rope --
def check_rope_position_zero_identity():
    x = RNG.standard_normal((4, 3, 16))
    np.testing.assert_allclose(O.rope(x, np.zeros(4), 10_000.0), x, rtol=0, atol=0)


def check_rope_d2_closed_form():
    """D = 2: score = cos(t)(q0k0+q1k1) + sin(t)(q1k0-q0k1), t = p_j - p_i."""
    q = RNG.standard_normal(2); k = RNG.standard_normal(2)
    pi, pj = 7.0, 3.0
    qr = O.rope(q[None, None], np.array([pi]), 10_000.0)[0, 0]
    kr = O.rope(k[None, None], np.array([pj]), 10_000.0)[0, 0]
    t = pj - pi
    want = math.cos(t) * (q[0] * k[0] + q[1] * k[1]) + math.sin(t) * (q[1] * k[0] - q[0] * k[1])
    assert abs(qr @ kr - want) < 1e-12


def check_rope_d4_pairing_and_frequencies():
    """D = 4: pairs (0,2) turn by p, pairs (1,3) by p * base^(-1/2)."""
    base = 10_000.0
    x = RNG.standard_normal(4)
    p = 5.0
    y = O.rope(x[None, None], np.array([p]), base)[0, 0]
    t0, t1 = p, p * base ** -0.5
    want = np.array([x[0] * math.cos(t0) - x[2] * math.sin(t0),
                     x[1] * math.cos(t1) - x[3] * math.sin(t1),
                     x[0] * math.sin(t0) + x[2] * math.cos(t0),
                     x[1] * math.sin(t1) + x[3] * math.cos(t1)])
    np.testing.assert_allclose(y, want, rtol=1e-13, atol=1e-14)


def check_rope_relative_invariance():
    """Scores depend on positions only through their difference."""
    S, D = 9, 64
    q = RNG.standard_normal((S, 1, D)); k = RNG.standard_normal((S, 1, D))
    pos = np.arange(S, dtype=np.float64) * 3
    for base in (10_000.0, 1_000_000.0):
        s0 = O.rope(q, pos, base)[:, 0] @ O.rope(k, pos, base)[:, 0].T
        s1 = O.rope(q, pos + 1000, base)[:, 0] @ O.rope(k, pos + 1000, base)[:, 0].T
        np.testing.assert_allclose(s0, s1, rtol=1e-9, atol=1e-9)


def check_rope_preserves_norm():
    x = RNG.standard_normal((6, 2, 32))
    y = O.rope(x, np.arange(6) * 11.0, 1_000_000.0, 8.0)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)


def check_rope_interpolation():
    """Interpolation factor s at positions s*p equals factor 1 at positions p."""
    x = RNG.standard_normal((5, 2, 32))
    p = np.arange(5) * 13.0
    np.testing.assert_allclose(O.rope(x, 8 * p, 1e6, 8.0), O.rope(x, p, 1e6, 1.0), rtol=1e-12, atol=1e-13)


# -------------------------------------------------------------------- mask --
def check_mask_matches_enumeration():
    rng = np.random.default_rng(7)
    for trial in range(30):
        S = int(rng.integers(1, 65))
        W = int(rng.integers(1, S + 3))
        kind = int(rng.integers(0, 2))
        n = int(rng.integers(0, 4))
        spans = None
        if n and S >= 2:
            cuts = np.sort(rng.choice(np.arange(S + 1), size=2 * n, replace=False))
            spans = cuts.reshape(n, 2)
        sid = O.span_ids(S, spans)
        ii, jj = np.meshgrid(np.arange(S), np.arange(S), indexing="ij")
        got = O.allowed(ii, jj, kind, W, sid)
        want = _mask_by_words(S, kind, W, None if spans is None else spans.tolist())
        assert np.array_equal(got, want), (S, W, kind, spans)


# ------------------------------------------------------------- attention --
def check_window_ge_S_local_equals_global():
    q, k, v, qg, kg, pos = _layer(1, 40, 4, 2, 16, 11)
    a, la = O.prefill(q, k, v, qg, kg, pos, O.LOCAL, 40, 1e4, 1.0)
    b, lb = O.prefill(q, k, v, qg, kg, pos, O.GLOBAL, 1, 1e4, 1.0)
    np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(la, lb, rtol=1e-13, atol=1e-13)


def check_window_one_returns_v():
    q, k, v, qg, kg, pos = _layer(2, 17, 4, 2, 16, 12)
    out, lse = O.prefill(q, k, v, qg, kg, pos, O.LOCAL, 1, 1e4, 1.0)
    want = np.repeat(v.double().numpy(), 2, axis=2)          # head h reads kv h // 2
    np.testing.assert_allclose(out, want, rtol=1e-14, atol=1e-14)


def check_zero_query_mean_and_count():
    """q = 0: every score is 0, out = mean of v over the visible set, lse = ln|A|."""
    S = 33
    _, k, v, qg, kg, pos = _layer(1, S, 2, 1, 8, 13)
    q = torch.zeros(1, S, 2, 8, dtype=torch.bfloat16)
    spans = np.array([[[5, 12], [20, 21]]])
    out, lse = O.prefill(q, k, v, qg, kg, pos, O.LOCAL, 6, 1e4, 1.0, spans)
    vis = _mask_by_words(S, O.LOCAL, 6, [[5, 12], [20, 21]])
    vv = v.double().numpy()[0, :, 0, :]
    for i in range(S):
        idx = np.nonzero(vis[i])[0]
        np.testing.assert_allclose(out[0, i, 0], vv[idx].mean(axis=0), rtol=1e-13, atol=1e-14)
        assert abs(lse[0, 0, i] - math.log(idx.size)) < 1e-13


def check_rows_sum_to_one():
    q, k, _, qg, kg, pos = _layer(1, 30, 4, 2, 16, 14)
    v = torch.ones(1, 30, 2, 16)
    out, _ = O.prefill(q, k, v, qg, kg, pos, O.GLOBAL, 1, 1e6, 8.0)
    np.testing.assert_allclose(out, 1.0, rtol=1e-14)


def check_span_of_length_one_is_no_op():
    q, k, v, qg, kg, pos = _layer(1, 30, 4, 2, 16, 15)
    a, _ = O.prefill(q, k, v, qg, kg, pos, O.LOCAL, 8, 1e4, 1.0, None)
    b, _ = O.prefill(q, k, v, qg, kg, pos, O.LOCAL, 8, 1e4, 1.0, np.array([[[9, 10]]]))
    np.testing.assert_allclose(a, b, rtol=0, atol=0)


def check_full_span_is_bidirectional():
    S = 24
    q, k, v, qg, kg, pos = _layer(1, S, 4, 2, 16, 16)
    out, _ = O.prefill(q, k, v, qg, kg, pos, O.LOCAL, 4, 1e4, 1.0, np.array([[[0, S]]]))
    qh = O.rope(O.qk_rmsnorm(q, qg), pos.double().numpy(), 1e4)
    kh = O.rope(O.qk_rmsnorm(k, kg), pos.double().numpy(), 1e4)
    want = _sdpa64(qh, kh, v.double().numpy(), np.ones((S, S), dtype=bool))
    np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-12)


def check_equal_positions_is_plain_attention():
    S = 20
    q, k, v, qg, kg, _ = _layer(1, S, 4, 2, 16, 17)
    pos = torch.full((1, S), 37, dtype=torch.int32)
    out, _ = O.prefill(q, k, v, qg, kg, pos, O.GLOBAL, 1, 1e6, 8.0)
    qn, kn = O.qk_rmsnorm(q, qg), O.qk_rmsnorm(k, kg)          # no rotation at all
    want = _sdpa64(qn, kn, v.double().numpy(), _mask_by_words(S, O.GLOBAL, 1, None))
    np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-12)


def check_rows_equal_bruteforce_and_sdpa():
    rng = np.random.default_rng(3)
    for trial, (G, Hkv, D) in enumerate([(1, 2, 8), (2, 2, 16), (4, 1, 16), (2, 3, 8)]):
        S = int(rng.integers(20, 70))
        kind = trial % 2
        W = int(rng.integers(1, 30))
        q, k, v, qg, kg, pos = _layer(2, S, G * Hkv, Hkv, D, 100 + trial)
        spans = np.array([[[3, 9], [9, 14]], [[0, 5], [S - 6, S - 1]]])
        base, interp = (1e4, 1.0) if kind == O.LOCAL else (1e6, 8.0)
        a, la = O.prefill(q, k, v, qg, kg, pos, kind, W, base, interp, spans)
        b, lb = O.prefill_bruteforce(q, k, v, qg, kg, pos, kind, W, base, interp, spans)
        np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(la, lb, rtol=1e-11, atol=1e-12)
        for bb in range(2):
            qh = O.rope(O.qk_rmsnorm(q[bb:bb + 1], qg), pos[bb:bb + 1].double().numpy(), base, interp)
            kh = O.rope(O.qk_rmsnorm(k[bb:bb + 1], kg), pos[bb:bb + 1].double().numpy(), base, interp)
            vis = _mask_by_words(S, kind, W, spans[bb].tolist())
            want = _sdpa64(qh, kh, v[bb:bb + 1].double().numpy(), vis)
            np.testing.assert_allclose(a[bb:bb + 1], want, rtol=1e-11, atol=1e-12)


def check_row_subset_matches_all_rows():
    q, k, v, qg, kg, pos = _layer(1, 90, 4, 2, 16, 18)
    full, lf = O.prefill(q, k, v, qg, kg, pos, O.LOCAL, 7, 1e4, 1.0)
    rows = [0, 5, 44, 89]
    part, lp = O.prefill_rows(q, k, v, qg, kg, pos, O.LOCAL, 7, 1e4, 1.0, rows=rows, row_group=3)
    np.testing.assert_allclose(part, full[:, rows], rtol=1e-14, atol=0)
    np.testing.assert_allclose(lp, lf[:, :, rows], rtol=1e-14, atol=0)


# ------------------------------------------------------------------ decode --
def _decode_case(kind, W, L, seed):
    Hq, Hkv, D = 4, 2, 16
    q, k, v, qg, kg, pos = _layer(1, L, Hq, Hkv, D, seed)
    base, interp = (1e4, 1.0) if kind == O.LOCAL else (1e6, 8.0)
    full, _ = O.prefill(q, k, v, qg, kg, pos, kind, W, base, interp)
    kh = O.rope(O.qk_rmsnorm(k, kg), pos.double().numpy(), base, interp)
    return q, k, v, qg, kg, kh, full, base, interp


def check_decode_equals_last_prefill_row():
    for kind, W, L in [(O.GLOBAL, 1, 37), (O.LOCAL, 8, 37), (O.LOCAL, 64, 20), (O.LOCAL, 1, 5)]:
        q, k, v, qg, kg, kh, full, base, interp = _decode_case(kind, W, L, 40 + L + W)
        out, khat = O.decode(q[:, L - 1], k[:, L - 1], v[:, L - 1], qg, kg, [L],
                             [kh[0, :L - 1]], [v[0, :L - 1]], [0], kind, W, base, interp)
        np.testing.assert_allclose(out[0], full[0, L - 1], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(khat[0], kh[0, L - 1], rtol=1e-13, atol=1e-14)


def check_decode_local_history_tail_suffices():
    kind, W, L = O.LOCAL, 8, 30
    q, k, v, qg, kg, kh, full, base, interp = _decode_case(kind, W, L, 77)
    t0 = L - W
    out, _ = O.decode(q[:, L - 1], k[:, L - 1], v[:, L - 1], qg, kg, [L],
                      [kh[0, t0:L - 1]], [v[0, t0:L - 1]], [t0], kind, W, base, interp)
    np.testing.assert_allclose(out[0], full[0, L - 1], rtol=1e-12, atol=1e-13)


ALL_CHECKS = [v for n, v in sorted(globals().items()) if n.startswith("check_")]


@pytest.mark.parametrize("check", ALL_CHECKS, ids=[c.__name__ for c in ALL_CHECKS])
def test_pin(check):
    check()
