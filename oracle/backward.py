"""Plain float64 gradients of Gemma 3's block attention (test infrastructure).

ORACLE -- test infrastructure, not product code.  Only tests, the smoke check
and the benchmark's CPU-baseline leg may use this module.  It shares no code
with the CUDA library.

The forward computation is the one in `oracle.attention` (QK-norm, RoPE, the
visibility mask, GQA, softmax attention; Gemma 3 Technical Report, section 2
"Model Architecture" and "Long context"; "Gemma explained: what's new in
Gemma 3", the q_norm/k_norm lines and section "Vision encoder and
processing").  The Technical Report trains these layers (section 2.2
"Pre-training": distillation; section 2.3 "Quantization Aware Training"), which
needs the gradient of a loss through every one of those steps.  Given
dout = dLoss/dout, this module applies the chain rule to each forward step in
reverse order:

5'. softmax attention, per query head h and row i over its visible set A(i):
      s_ij = q^_i . k^_j / sqrt(D),  P_ij = exp(s_ij - lse_i)
      dv_j   += sum_i P_ij dout_i
      dP_ij   = dout_i . v_j
      dS_ij   = P_ij (dP_ij - sum_{j'} P_ij' dP_ij')   (Jacobian of softmax)
      dq^_i   = sum_j dS_ij k^_j / sqrt(D)
      dk^_j  += sum_i dS_ij q^_i / sqrt(D)
4'. GQA: a kv head's gradients are the sums over the G query heads reading it.
3'. the mask has no gradient: pairs outside A(i) carry P_ij = 0.
2'. RoPE is a rotation per pair (d, d + D/2), so its gradient rotates back by
    the same angle: (g_d, g_{d+D/2}) -> (g_d cos t + g_{d+D/2} sin t,
    -g_d sin t + g_{d+D/2} cos t).
1'. RMSNorm y = x * r * gamma with r = (mean_d x_d^2 + eps)^(-1/2):
      dgamma_d += g_d x_d r   (summed over every token and head)
      dx_d      = r gamma_d g_d - x_d r^3 / D * sum_e gamma_e g_e x_e

Rows are processed in groups only to batch the library matmuls; the sums
over query rows in dk^ and dv are accumulated group by group (the same sum,
in another rounding order).
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

from .attention import EPS, LOCAL, GLOBAL, _f64, _i64, allowed, inv_frequencies, qk_rmsnorm, rope, span_ids

__all__ = ["rope_backward", "rmsnorm_backward", "attention_backward", "prefill_backward", "LOCAL", "GLOBAL"]


# --------------------------------------------------------------- step 2' --
def rope_backward(g: np.ndarray, pos: np.ndarray, base: float, interp: float = 1.0) -> np.ndarray:
    """Gradient through the rotation: g [..., T, H, D] at positions pos [..., T].

    Step 2' of the module docstring: the inverse of the rotation that
    `oracle.attention.rope` applies (Technical Report, section 2 "Long context").
    """
    g = _f64(g)
    p = _f64(pos) / float(interp)
    D = g.shape[-1]
    h = D // 2
    theta = p[..., :, None] * inv_frequencies(D, base)
    c = np.cos(theta)[..., :, None, :]
    s = np.sin(theta)[..., :, None, :]
    g1 = g[..., :h]
    g2 = g[..., h:]
    return np.concatenate([g1 * c + g2 * s, -g1 * s + g2 * c], axis=-1)


# --------------------------------------------------------------- step 1' --
def rmsnorm_backward(x: np.ndarray, gamma: np.ndarray, g: np.ndarray, eps: float = EPS):
    """Gradient of y = x / sqrt(mean(x^2) + eps) * gamma over the last axis.

    Returns (dx with the shape of x, dgamma [D] summed over all other axes).
    Step 1' of the module docstring: the chain rule through the QK-norm of the
    Technical Report, section 2 "Model Architecture".
    """
    x = _f64(x)
    gm = _f64(gamma)
    g = _f64(g)
    D = x.shape[-1]
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    dgamma = (g * x * r).reshape(-1, D).sum(axis=0)
    inner = np.sum(gm * g * x, axis=-1, keepdims=True)
    dx = r * gm * g - x * (r ** 3) * inner / D
    return dx, dgamma


# --------------------------------------------------------- steps 5', 4' --
def attention_backward(qh, kh, v, dout, kind: int, window: int, sid: np.ndarray,
                       kv_heads: Optional[Sequence[int]] = None, row_group: int = 256):
    """Gradients of one sequence's attention with respect to q^, k^ and v.

    qh [S, Hq, D], kh / v [S, Hkv, D] (normalised and rotated q and k, raw v),
    dout [S, Hq, D].  Only the kv heads in `kv_heads` (all if None) and their
    query heads are computed; the other heads of the results are NaN.
    Returns dqh [S, Hq, D], dkh [S, Hkv, D], dv [S, Hkv, D].  Steps 5', 4' and
    3' of the module docstring, over the forward's visible sets (Technical
    Report, section 2; "Gemma explained", section "Vision encoder and
    processing").
    """
    qh, kh, v, dout = _f64(qh), _f64(kh), _f64(v), _f64(dout)
    S, Hq, D = qh.shape
    Hkv = kh.shape[1]
    G = Hq // Hkv
    heads = range(Hkv) if kv_heads is None else kv_heads
    dqh = np.full_like(qh, np.nan)
    dkh = np.full_like(kh, np.nan)
    dv = np.full_like(v, np.nan)
    scale = 1.0 / math.sqrt(D)
    keys = np.arange(S, dtype=np.int64)
    for kvh in heads:
        K = kh[:, kvh, :]
        V = v[:, kvh, :]
        dK = np.zeros((S, D))
        dV = np.zeros((S, D))
        for h in range(kvh * G, (kvh + 1) * G):
            for r0 in range(0, S, row_group):
                rows = np.arange(r0, min(S, r0 + row_group), dtype=np.int64)
                vis = allowed(rows[:, None], keys[None, :], kind, window, sid)     # [R, S]
                Q = qh[rows, h, :]
                dO = dout[rows, h, :]
                s = np.where(vis, Q @ K.T * scale, -np.inf)
                m = s.max(axis=1, keepdims=True)
                e = np.exp(s - m)
                P = e / e.sum(axis=1, keepdims=True)                            # 0 off the visible set
                dP = dO @ V.T
                dS = P * (dP - np.sum(P * dP, axis=1, keepdims=True))
                dqh[rows, h, :] = dS @ K * scale
                dK += dS.T @ Q * scale
                dV += P.T @ dO
        dkh[:, kvh, :] = dK
        dv[:, kvh, :] = dV
    return dqh, dkh, dv


# ------------------------------------------------------------ whole call --
def prefill_backward(q, k, v, q_gamma, k_gamma, positions, kind, window, rope_base, interp, dout,
                     spans=None, kv_heads: Optional[Sequence[int]] = None, row_group: int = 256):
    """Gradients of sum(out * dout) for one prefill call of the block (steps 5'
    to 1' of the module docstring; the training that needs them: Technical
    Report, sections 2.2 "Pre-training" and 2.3 "Quantization Aware Training").

    q [B,S,Hq,D], k/v [B,S,Hkv,D] raw (pre-norm, pre-RoPE), gammas [D],
    positions [B,S], spans [B,n,2] or None, dout [B,S,Hq,D].
    Returns dict(dq, dk, dv, dq_gamma, dk_gamma) in float64.  With `kv_heads`
    only those kv heads (and their query heads) are computed: the other heads
    are NaN and the gamma gradients (sums over every head) are None.
    """
    qf, kf, vf, dof = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, S, Hq, D = qf.shape
    Hkv = kf.shape[2]
    G = Hq // Hkv
    pos = _f64(positions)
    sp = None if spans is None else _i64(spans)
    dq = np.full_like(qf, np.nan)
    dk = np.full_like(kf, np.nan)
    dv = np.full_like(vf, np.nan)
    heads = list(range(Hkv)) if kv_heads is None else list(kv_heads)
    qsel = [h for kvh in heads for h in range(kvh * G, (kvh + 1) * G)]
    dqg = np.zeros(D)
    dkg = np.zeros(D)
    for b in range(B):
        # Forward steps 1-2 (needed for the activations the gradients use).
        qh = rope(qk_rmsnorm(qf[b], q_gamma), pos[b], rope_base, interp)
        kh = rope(qk_rmsnorm(kf[b], k_gamma), pos[b], rope_base, interp)
        sid = span_ids(S, None if sp is None else sp[b])
        dqh, dkh, dvb = attention_backward(qh, kh, vf[b], dof[b], kind, window, sid, heads, row_group)
        # Step 2' then step 1', for the computed heads only.
        gq = rope_backward(dqh[:, qsel], pos[b], rope_base, interp)
        gk = rope_backward(dkh[:, heads], pos[b], rope_base, interp)
        dqx, dg = rmsnorm_backward(qf[b][:, qsel], q_gamma, gq)
        dqg += dg
        dkx, dg = rmsnorm_backward(kf[b][:, heads], k_gamma, gk)
        dkg += dg
        dq[b][:, qsel] = dqx
        dk[b][:, heads] = dkx
        dv[b][:, heads] = dvb[:, heads]
    full = kv_heads is None
    return dict(dq=dq, dk=dk, dv=dv, dq_gamma=dqg if full else None, dk_gamma=dkg if full else None)


def loss(q, k, v, q_gamma, k_gamma, positions, kind, window, rope_base, interp, dout, spans=None) -> float:
    """sum(out * dout) of the forward oracle: the scalar whose gradient
    `prefill_backward` returns (used by the finite-difference pins)."""
    from .attention import prefill
    out, _ = prefill(q, k, v, q_gamma, k_gamma, positions, kind, window, rope_base, interp, spans)
    return float(np.sum(out * _f64(dout)))
