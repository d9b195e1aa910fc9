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
    with np.errstate(invalid="ignore", divide="ignore"):  # a zero row gives NaN: what a pin catches
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


def _decode_factory(pos_shift=0, gqa_mod=False, value_is_key=False, no_scale=False):
    """Copy of the oracle's decode step with one planted mistake."""
    def decode(q, k_new, v_new, q_gamma, k_gamma, seq_lens, k_hist, v_hist, hist_start,
               kind, window, rope_base, interp):
        qf = O._f64(q)
        B, Hq, D = qf.shape
        L = O._i64(seq_lens)
        out = np.empty((B, Hq, D))
        k_hat = np.empty((B, O._f64(k_new).shape[1], D))
        for b in range(B):
            Lb = int(L[b])
            pos = np.array([Lb - 1 + pos_shift], dtype=np.float64)
            qh = O.rope(O.qk_rmsnorm(qf[b][None], q_gamma), pos, rope_base, interp)[0]
            kn = O.rope(O.qk_rmsnorm(O._f64(k_new)[b][None], k_gamma), pos, rope_base, interp)[0]
            k_hat[b] = kn
            t0 = int(hist_start[b])
            keys = np.concatenate([O._f64(k_hist[b]), kn[None]], axis=0)
            newv = kn if value_is_key else O._f64(v_new)[b]
            vals = np.concatenate([O._f64(v_hist[b]), newv[None]], axis=0)
            vis = O.allowed(np.int64(Lb - 1), np.arange(t0, Lb), kind, window, O.span_ids(Lb, None))
            Hkv = keys.shape[1]
            for h in range(Hq):
                kv = (h % Hkv) if gqa_mod else (h // (Hq // Hkv))
                sc = keys[:, kv, :] @ qh[h]
                if not no_scale:
                    sc = sc / math.sqrt(D)
                sc = np.where(vis, sc, -np.inf)
                m = sc.max(); pr = np.exp(sc - m)
                out[b, h] = pr @ vals[:, kv, :] / pr.sum()
        return out, k_hat
    return decode


MUTANTS = {
    "decode_position_off_by_one": ("decode", _decode_factory(pos_shift=1)),
    "decode_gqa_head_modulo": ("decode", _decode_factory(gqa_mod=True)),
    "decode_new_value_is_its_key": ("decode", _decode_factory(value_is_key=True)),
    "decode_no_softmax_scale": ("decode", _decode_factory(no_scale=True)),
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


def test_unmutated_decode_copy_matches():
    """The copy of decode used for mutants agrees with the oracle when unmutated."""
    for kind, W, L in [(O.LOCAL, 7, 20), (O.GLOBAL, 1, 13)]:
        q, k, v, qg, kg, kh, full, base, interp = P._decode_case(kind, W, L, 5)
        args = (q[:, L - 1], k[:, L - 1], v[:, L - 1], qg, kg, [L], [kh[0, :L - 1]], [v[0, :L - 1]], [0],
                kind, W, base, interp)
        a, ka = O.decode(*args)
        b, kb = _decode_factory()(*args)
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(ka, kb, rtol=1e-12, atol=1e-13)


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
