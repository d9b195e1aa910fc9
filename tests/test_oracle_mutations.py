"""The oracle's pins must catch plausible mistakes.

Each case swaps one oracle function for a copy with a single planted error
(a dropped term, a flipped sign, an off-by-one, a wrong index) on the CPU and
asserts that at least one pin from test_oracle_pins fails.
"""
import math

import numpy as np
import pytest

from oracle import attention as O
import test_oracle_pins as P


def _norm_no_eps(x, gamma, eps=O.EPS):
    x = O._f64(x); g = O._f64(gamma)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True)) * g


def _norm_no_gamma(x, gamma, eps=O.EPS):
    x = O._f64(x)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def _rope_factory(sign=1.0, interleaved=False, exp_scale=2.0, interp_mul=False):
    def rope(x, pos, base, interp=1.0):
        x = O._f64(x)
        p = O._f64(pos) * float(interp) if interp_mul else O._f64(pos) / float(interp)
        D = x.shape[-1]
        h = D // 2
        d = np.arange(h, dtype=np.float64)
        theta = p[..., :, None] * np.power(float(base), -exp_scale * d / D)
        c = np.cos(theta)[..., :, None, :]
        s = sign * np.sin(theta)[..., :, None, :]
        if interleaved:
            x1, x2 = x[..., 0::2], x[..., 1::2]
            out = np.empty_like(x)
            out[..., 0::2] = x1 * c - x2 * s
            out[..., 1::2] = x1 * s + x2 * c
            return out
        x1, x2 = x[..., :h], x[..., h:]
        return np.concatenate([x1 * c - x2 * s, x1 * s + x2 * c], axis=-1)
    return rope


def _allowed_factory(window_le=False, no_spans=False, spans_leak=False, no_causal=False):
    def allowed(i, j, kind, window, sid):
        i = np.asarray(i, dtype=np.int64); j = np.asarray(j, dtype=np.int64)
        causal = (j <= i) if not no_causal else np.ones(np.broadcast(i, j).shape, bool)
        if kind == O.LOCAL:
            causal = causal & (((i - j) <= int(window)) if window_le else ((i - j) < int(window)))
        if no_spans:
            return causal
        if spans_leak:
            return causal | ((sid[i] >= 0) & (sid[j] >= 0))
        return causal | ((sid[i] == sid[j]) & (sid[i] >= 0))
    return allowed


def _attend_factory(gqa_mod=False, no_scale=False):
    def attend(qh_b, kh_hm, v_hm, rows, kind, window, sid, S):
        Hq, D = qh_b.shape[1], qh_b.shape[2]
        Hkv = kh_hm.shape[0]
        rows = np.asarray(rows, dtype=np.int64)
        R = rows.size
        out = np.empty((R, Hq, D)); lse = np.empty((Hq, R))
        for r, i in enumerate(rows):
            vis = O.allowed(np.int64(i), np.arange(S), kind, window, sid)
            for h in range(Hq):
                kv = (h % Hkv) if gqa_mod else (h // (Hq // Hkv))
                s = kh_hm[kv] @ qh_b[i, h]
                if not no_scale:
                    s = s / math.sqrt(D)
                s = np.where(vis, s, -np.inf)
                m = s.max(); p = np.exp(s - m); l = p.sum()
                out[r, h] = p @ v_hm[kv] / l
                lse[h, r] = m + math.log(l)
        return out, lse
    return attend


MUTANTS = {
    "norm_drops_eps": ("qk_rmsnorm", _norm_no_eps),
    "norm_drops_gamma": ("qk_rmsnorm", _norm_no_gamma),
    "rope_reversed_sign": ("rope", _rope_factory(sign=-1.0)),
    "rope_interleaved_pairs": ("rope", _rope_factory(interleaved=True)),
    "rope_wrong_exponent": ("rope", _rope_factory(exp_scale=1.0)),
    "rope_interp_multiplies": ("rope", _rope_factory(interp_mul=True)),
    "window_off_by_one": ("allowed", _allowed_factory(window_le=True)),
    "spans_ignored": ("allowed", _allowed_factory(no_spans=True)),
    "spans_leak_across_images": ("allowed", _allowed_factory(spans_leak=True)),
    "not_causal": ("allowed", _allowed_factory(no_causal=True)),
    "gqa_head_modulo": ("_attend_rows", _attend_factory(gqa_mod=True)),
    "no_softmax_scale": ("_attend_rows", _attend_factory(no_scale=True)),
}


def test_unmutated_attend_matches():
    """The loop-form attend used for mutants agrees with the oracle when unmutated."""
    q, k, v, qg, kg, pos = P._layer(1, 25, 4, 2, 8, 5)
    a, la = O.prefill(q, k, v, qg, kg, pos, O.LOCAL, 6, 1e4, 1.0, np.array([[[3, 9]]]))
    orig = O._attend_rows
    try:
        O._attend_rows = _attend_factory()
        b, lb = O.prefill(q, k, v, qg, kg, pos, O.LOCAL, 6, 1e4, 1.0, np.array([[[3, 9]]]))
    finally:
        O._attend_rows = orig
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(la, lb, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(O, attr, fn)
    caught = []
    for check in P.ALL_CHECKS:
        try:
            check()
        except (AssertionError, ValueError, IndexError):
            caught.append(check.__name__)
    assert caught, f"no pin caught mutant {name}"
