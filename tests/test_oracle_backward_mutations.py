"""The backward oracle's pins must catch plausible mistakes.

Each case swaps one function of oracle/backward.py for a copy with a single
planted error and asserts that at least one pin of test_oracle_backward fails.
"""
import math

import numpy as np
import pytest

from oracle import attention as O
from oracle import backward as BW
import test_oracle_backward as P


def _attention_factory(no_delta=False, no_scale_dk=False, gqa_mod=False, dv_uses_ds=False, no_scale_dq=False,
                       dq_uses_p=False, first_head_only=False):
    def attention_backward(qh, kh, v, dout, kind, window, sid, kv_heads=None, row_group=256):
        qh, kh, v, dout = O._f64(qh), O._f64(kh), O._f64(v), O._f64(dout)
        S, Hq, D = qh.shape
        Hkv = kh.shape[1]
        G = Hq // Hkv
        heads = range(Hkv) if kv_heads is None else kv_heads
        dqh = np.full_like(qh, np.nan)
        dkh = np.full_like(kh, np.nan)
        dv = np.full_like(v, np.nan)
        scale = 1.0 / math.sqrt(D)
        keys = np.arange(S)
        for kvh in heads:
            dK = np.zeros((S, D))
            dV = np.zeros((S, D))
            group = [h for h in range(Hq) if h % Hkv == kvh] if gqa_mod else range(kvh * G, (kvh + 1) * G)
            for n_h, h in enumerate(group):
                vis = O.allowed(keys[:, None], keys[None, :], kind, window, sid)
                K, V, Q, dO = kh[:, kvh], v[:, kvh], qh[:, h], dout[:, h]
                s = np.where(vis, Q @ K.T * scale, -np.inf)
                e = np.exp(s - s.max(axis=1, keepdims=True))
                Pm = e / e.sum(axis=1, keepdims=True)
                dP = dO @ V.T
                dS = Pm * dP if no_delta else Pm * (dP - np.sum(Pm * dP, axis=1, keepdims=True))
                dqh[:, h] = (Pm if dq_uses_p else dS) @ K * (1.0 if no_scale_dq else scale)
                if first_head_only and n_h > 0:
                    continue
                dK += dS.T @ Q * (1.0 if no_scale_dk else scale)
                dV += (dS if dv_uses_ds else Pm).T @ dO
            dkh[:, kvh] = dK
            dv[:, kvh] = dV
        return dqh, dkh, dv
    return attention_backward


def _rope_forward_direction(g, pos, base, interp=1.0):
    return O.rope(g, pos, base, interp)


_ROPE_BACKWARD = BW.rope_backward  # the unmutated function, captured before any patching


def _rope_backward_no_interp(g, pos, base, interp=1.0):
    return _ROPE_BACKWARD(g, pos, base, 1.0)


def _norm_factory(no_second_term=False, dgamma_no_r=False):
    def rmsnorm_backward(x, gamma, g, eps=O.EPS):
        x, gm, g = O._f64(x), O._f64(gamma), O._f64(g)
        D = x.shape[-1]
        r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
        dgamma = (g * x * (1.0 if dgamma_no_r else r)).reshape(-1, D).sum(axis=0)
        dx = r * gm * g
        if not no_second_term:
            dx = dx - x * r ** 3 * np.sum(gm * g * x, axis=-1, keepdims=True) / D
        return dx, dgamma
    return rmsnorm_backward


PINS = [
    lambda: [P.test_backward_matches_finite_differences(i) for i in range(len(P.FD_CASES))],
    lambda: P.test_backward_matches_torch_autograd(O.LOCAL, 7, 1e4, 1.0, [[[10, 30], [30, 41]]]),
    P.test_dv_columns_sum_to_dout,
    P.test_identical_keys_give_zero_query_gradient,
    P.test_window_of_one_passes_gradient_to_v_only,
    P.test_rmsnorm_gradient_is_scale_invariant,
    P.test_rope_gradient_is_the_inverse_rotation,
]

MUTANTS = {
    "softmax Jacobian without the row term": ("attention_backward", _attention_factory(no_delta=True)),
    "dk without the 1/sqrt(D) scale": ("attention_backward", _attention_factory(no_scale_dk=True)),
    "GQA head h -> kv head h % Hkv": ("attention_backward", _attention_factory(gqa_mod=True)),
    "dv accumulated from dS instead of P": ("attention_backward", _attention_factory(dv_uses_ds=True)),
    "dq without the 1/sqrt(D) scale": ("attention_backward", _attention_factory(no_scale_dq=True)),
    "dq from P instead of dS": ("attention_backward", _attention_factory(dq_uses_p=True)),
    "kv gradients from the group's first query head only":
        ("attention_backward", _attention_factory(first_head_only=True)),
    "RoPE gradient rotated forward": ("rope_backward", _rope_forward_direction),
    "RoPE gradient ignores position interpolation": ("rope_backward", _rope_backward_no_interp),
    "RMSNorm gradient without the mean term": ("rmsnorm_backward", _norm_factory(no_second_term=True)),
    "gamma gradient without the 1/rms factor": ("rmsnorm_backward", _norm_factory(dgamma_no_r=True)),
}


def test_unmutated_attention_copy_matches():
    rng = np.random.default_rng(0)
    S, Hq, Hkv, D = 20, 4, 2, 8
    qh, kh, v = rng.standard_normal((S, Hq, D)), rng.standard_normal((S, Hkv, D)), rng.standard_normal((S, Hkv, D))
    dout = rng.standard_normal((S, Hq, D))
    sid = O.span_ids(S, np.array([[3, 9]]))
    want = BW.attention_backward(qh, kh, v, dout, O.LOCAL, 6, sid)
    got = _attention_factory()(qh, kh, v, dout, O.LOCAL, 6, sid)
    for a, b in zip(want, got):
        np.testing.assert_allclose(b, a, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("name", list(MUTANTS))
def test_pins_catch_mutant(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(BW, attr, fn)
    failed = 0
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed > 0, f"no pin caught: {name}"
