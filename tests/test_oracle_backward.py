"""Pins of the float64 backward oracle (oracle/backward.py), CPU only.

The gradients are checked against things that do not share the oracle's
hand-derived formulas:
- central finite differences of the forward oracle's loss sum(out * dout);
- torch float64 autograd of a separately written torch forward (norm, RoPE,
  a boolean mask built from the visibility rule, scaled_dot_product_attention);
- closed forms: rows of P sum to one (sum_j dv_j = sum_i dout_i over the
  group), identical keys give dq = 0, a window of one gives out_i = v_i;
- invariants: RMSNorm is scale-invariant up to eps (x . dx ~ 0), RoPE's
  gradient is the inverse rotation.
"""
import math

import numpy as np
import pytest
import torch

from oracle import attention as O
from oracle import backward as BW

LOC, GLB = O.LOCAL, O.GLOBAL


def _case(B, S, Hq, Hkv, D, seed, spans=None, positions=None):
    rng = np.random.default_rng(seed)
    x = dict(
        q=rng.standard_normal((B, S, Hq, D)),
        k=rng.standard_normal((B, S, Hkv, D)),
        v=rng.standard_normal((B, S, Hkv, D)),
        q_gamma=1.0 + 0.1 * rng.standard_normal(D),
        k_gamma=1.0 + 0.1 * rng.standard_normal(D),
        positions=np.tile(np.arange(S), (B, 1)) if positions is None else positions,
        dout=rng.standard_normal((B, S, Hq, D)),
        spans=None if spans is None else np.asarray(spans, dtype=np.int64),
    )
    return x


def _grads(x, kind, W, base, interp, **kw):
    return BW.prefill_backward(x["q"], x["k"], x["v"], x["q_gamma"], x["k_gamma"], x["positions"], kind, W, base,
                               interp, x["dout"], x["spans"], **kw)


def _loss(x, kind, W, base, interp):
    return BW.loss(x["q"], x["k"], x["v"], x["q_gamma"], x["k_gamma"], x["positions"], kind, W, base, interp,
                   x["dout"], x["spans"])


GRAD_OF = dict(q="dq", k="dk", v="dv", q_gamma="dq_gamma", k_gamma="dk_gamma")

FD_CASES = [
    # B, S, Hq, Hkv, D, kind, W, base, interp, spans, positions
    (1, 10, 4, 2, 8, LOC, 3, 1e4, 1.0, [[[2, 6]]], None),
    (2, 9, 2, 1, 4, GLB, 9, 1e6, 8.0, [[[0, 3], [5, 9]], [[4, 6], [6, 8]]], None),
    (1, 12, 3, 3, 6, LOC, 5, 1e4, 1.0, None, np.array([[3 * t + 7 for t in range(12)]])),
]


@pytest.mark.parametrize("ci", range(len(FD_CASES)))
def test_backward_matches_finite_differences(ci):
    """Every gradient coordinate of a tiny case against a central difference."""
    B, S, Hq, Hkv, D, kind, W, base, interp, spans, pos = FD_CASES[ci]
    x = _case(B, S, Hq, Hkv, D, seed=ci, spans=spans, positions=pos)
    g = _grads(x, kind, W, base, interp)
    rng = np.random.default_rng(100 + ci)
    h = 1e-5
    for name, gname in GRAD_OF.items():
        arr = x[name]
        flat = arr.reshape(-1)
        idx = rng.choice(flat.size, size=min(flat.size, 60), replace=False)
        for i in idx:
            keep = flat[i]
            flat[i] = keep + h
            lp = _loss(x, kind, W, base, interp)
            flat[i] = keep - h
            lm = _loss(x, kind, W, base, interp)
            flat[i] = keep
            fd = (lp - lm) / (2 * h)
            an = g[gname].reshape(-1)[i]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (name, int(i), fd, an)


def _torch_forward(x, kind, W, base, interp):
    """A separate torch float64 formulation of the forward, for autograd."""
    t = {k: torch.tensor(v, dtype=torch.float64, requires_grad=k in GRAD_OF) for k, v in x.items()
         if k not in ("spans", "positions")}
    q, k, v = t["q"], t["k"], t["v"]
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]

    def norm(a, gm):
        return a * torch.rsqrt(a.pow(2).mean(-1, keepdim=True) + 1e-6) * gm

    def rot(a, pos):
        half = D // 2
        fr = torch.tensor([base ** (-2.0 * i / D) for i in range(half)], dtype=torch.float64)
        ang = (torch.tensor(pos, dtype=torch.float64) / interp)[:, :, None, None] * fr
        a1, a2 = a[..., :half], a[..., half:]
        return torch.cat([a1 * ang.cos() - a2 * ang.sin(), a2 * ang.cos() + a1 * ang.sin()], -1)

    qh = rot(norm(q, t["q_gamma"]), x["positions"])
    kh = rot(norm(k, t["k_gamma"]), x["positions"])
    mask = torch.zeros(B, S, S, dtype=torch.bool)
    for b in range(B):
        img = [-1] * S
        if x["spans"] is not None:
            for n, (s0, s1) in enumerate(x["spans"][b]):
                for j in range(s0, s1):
                    img[j] = n
        for i in range(S):
            for j in range(S):
                near = j <= i and (kind == GLB or i - j < W)
                mask[b, i, j] = near or (img[i] >= 0 and img[i] == img[j])
    rep = Hq // Hkv
    qT = qh.permute(0, 2, 1, 3)
    kT = kh.repeat_interleave(rep, dim=2).permute(0, 2, 1, 3)
    vT = v.repeat_interleave(rep, dim=2).permute(0, 2, 1, 3)
    out = torch.nn.functional.scaled_dot_product_attention(qT, kT, vT, attn_mask=mask[:, None])
    loss = (out.permute(0, 2, 1, 3) * t["dout"]).sum()
    loss.backward()
    return {GRAD_OF[k]: t[k].grad.numpy() for k in GRAD_OF}


@pytest.mark.parametrize("kind,W,base,interp,spans", [
    (LOC, 7, 1e4, 1.0, [[[10, 30], [30, 41]]]),
    (GLB, 80, 1e6, 8.0, [[[50, 70]]]),
])
def test_backward_matches_torch_autograd(kind, W, base, interp, spans):
    x = _case(1, 80, 4, 2, 16, seed=7, spans=spans)
    ref = _torch_forward(x, kind, W, base, interp)
    got = _grads(x, kind, W, base, interp, row_group=32)
    for name in ref:
        np.testing.assert_allclose(got[name], ref[name], rtol=1e-9, atol=1e-10, err_msg=name)


def test_dv_columns_sum_to_dout():
    """Rows of P sum to one, so sum_j dv_j = sum over the group's heads of sum_i dout_i."""
    x = _case(2, 40, 6, 2, 8, seed=3, spans=[[[5, 15]], [[20, 40]]])
    g = _grads(x, LOC, 6, 1e4, 1.0)
    for b in range(2):
        for kvh in range(2):
            want = x["dout"][b][:, 3 * kvh:3 * kvh + 3].sum(axis=(0, 1))
            np.testing.assert_allclose(g["dv"][b, :, kvh].sum(axis=0), want, atol=1e-10)


def test_identical_keys_give_zero_query_gradient():
    """All keys equal (same raw k, same position): softmax weights do not depend on q."""
    x = _case(1, 24, 4, 2, 8, seed=4, spans=[[[3, 9]]])
    x["k"][:] = x["k"][:, :1]
    x["positions"] = np.zeros((1, 24), dtype=np.int64)
    g = _grads(x, GLB, 24, 1e6, 8.0)
    assert np.abs(g["dq"]).max() < 1e-12
    assert np.abs(g["dq_gamma"]).max() < 1e-12
    assert np.abs(g["dk"]).max() > 1e-3  # the keys' own gradient is not trivially zero


def test_window_of_one_passes_gradient_to_v_only():
    """W = 1 and no image: out_i = v_i, so dv = group sum of dout and dq = dk = 0."""
    x = _case(1, 16, 4, 2, 8, seed=5)
    g = _grads(x, LOC, 1, 1e4, 1.0)
    want = x["dout"].reshape(1, 16, 2, 2, 8).sum(axis=3)
    np.testing.assert_allclose(g["dv"], want, atol=1e-12)
    assert np.abs(g["dq"]).max() < 1e-12 and np.abs(g["dk"]).max() < 1e-12


def test_rmsnorm_gradient_is_scale_invariant():
    """y(c x) = y(x) up to eps, so x . dx = 0 up to a relative O(eps / mean(x^2))."""
    rng = np.random.default_rng(6)
    x = rng.standard_normal((50, 3, 16))
    gm = 1.0 + 0.1 * rng.standard_normal(16)
    gup = rng.standard_normal((50, 3, 16))
    dx, _ = BW.rmsnorm_backward(x, gm, gup)
    dot = np.abs(np.sum(x * dx, axis=-1))
    assert (dot <= 1e-5 * np.linalg.norm(x, axis=-1) * np.linalg.norm(dx, axis=-1)).all()


def test_rope_gradient_is_the_inverse_rotation():
    rng = np.random.default_rng(8)
    g = rng.standard_normal((2, 30, 3, 16))
    pos = np.tile(np.arange(30) * 5, (2, 1))
    back = BW.rope_backward(O.rope(g, pos, 1e6, 8.0), pos, 1e6, 8.0)
    np.testing.assert_allclose(back, g, atol=1e-12)
    zero = np.zeros((2, 30))
    np.testing.assert_allclose(BW.rope_backward(g, zero, 1e4), g, atol=0)


def test_kv_head_subset_matches_full():
    x = _case(1, 33, 4, 2, 8, seed=9, spans=[[[1, 20]]])
    full = _grads(x, LOC, 5, 1e4, 1.0)
    part = _grads(x, LOC, 5, 1e4, 1.0, kv_heads=[1])
    np.testing.assert_allclose(part["dq"][:, :, 2:], full["dq"][:, :, 2:], atol=1e-13)
    np.testing.assert_allclose(part["dk"][:, :, 1:], full["dk"][:, :, 1:], atol=1e-13)
    np.testing.assert_allclose(part["dv"][:, :, 1:], full["dv"][:, :, 1:], atol=1e-13)
    assert np.isnan(part["dq"][:, :, :2]).all() and part["dq_gamma"] is None
