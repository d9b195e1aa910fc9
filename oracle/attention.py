"""Plain float64 definition of Gemma 3's block attention (test infrastructure).

ORACLE -- test infrastructure, not product code.  Only tests, the smoke check
and the benchmark's CPU-baseline leg may use this module.  It shares no code
with the CUDA library.

What it computes, one attention call of a 5:1 block, step by step, in the
order the sources give:

1. QK-norm.  Per token and head, q and k are RMS-normalised over head_dim
   with eps 1e-6 and multiplied by a learned per-feature gain.  Gemma 3
   Technical Report, section 2 "Model Architecture" (QK-norm replaces Gemma
   2's soft-capping); eps and dim from the q_norm/k_norm lines of the 27B and
   1B printouts on "Gemma explained: what's new in Gemma 3".
2. RoPE.  Pairs (d, d + D/2) rotate by theta_d = (p / s) * base^(-2d/D).
   Local layers use base 10k, global layers base 1M with linear position
   interpolation by s (Technical Report, section 2 "Long context": base raised
   from 10k to 1M, interpolation "similar to Chen et al. (2023)").  The
   pairing layout and the linear form p/s are readings the pages leave open.
3. Mask.  Token j is visible from token i iff
       (j <= i and (global layer or i - j < W))  or  (i and j lie in the same
       image span).
   Window span 1024 for local layers (Technical Report, section 1
   Introduction and section 2 "5:1 interleaving"); image tokens attend
   bidirectionally within their image (Gemma explained, section
   "Vision encoder and processing").
4. GQA.  Query head h reads key/value head floor(h / G), G = Hq / Hkv
   (Technical Report, section 2: grouped-query attention).
5. Softmax attention with scale 1/sqrt(D) over the visible set; lse = m + ln l.

Rows are evaluated in groups only to batch the library matmul; each row's
softmax is taken over its own visible set in one pass (no streaming).
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

EPS = 1e-6
LOCAL = 0
GLOBAL = 1


def _f64(x) -> np.ndarray:
    """Exact float64 copy of a torch tensor (any dtype) or array."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu").to(torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def _i64(x) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu").to(torch.int64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.int64)


# ---------------------------------------------------------------- step 1 --
def qk_rmsnorm(x: np.ndarray, gamma: np.ndarray, eps: float = EPS) -> np.ndarray:
    """x / sqrt(mean_d x_d^2 + eps) * gamma over the last axis (head_dim).

    Gemma 3 Technical Report, section 2 "Model Architecture" (QK-norm); eps and
    the normalised axis from the q_norm/k_norm lines printed on "Gemma
    explained: what's new in Gemma 3".
    """
    x = _f64(x)
    g = _f64(gamma)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * g


# ---------------------------------------------------------------- step 2 --
def inv_frequencies(D: int, base: float) -> np.ndarray:
    """base^(-2d/D) for d = 0 .. D/2-1 (Technical Report, section 2 "Long context":
    base 10k on local layers, 1M on global layers)."""
    d = np.arange(D // 2, dtype=np.float64)
    return np.power(float(base), -2.0 * d / D)


def rope(x: np.ndarray, pos: np.ndarray, base: float, interp: float = 1.0) -> np.ndarray:
    """Rotate x [..., T, H, D] at token positions pos [..., T].

    Pair (x_d, x_{d+D/2}) becomes (x_d cos t - x_{d+D/2} sin t,
    x_d sin t + x_{d+D/2} cos t) with t = (pos / interp) * base^(-2d/D).
    Technical Report, section 2 "Long context" (bases; linear interpolation
    "similar to Chen et al. (2023)"); the half-split pairing is a reading.
    """
    x = _f64(x)
    p = _f64(pos) / float(interp)
    D = x.shape[-1]
    h = D // 2
    theta = p[..., :, None] * inv_frequencies(D, base)          # [..., T, D/2]
    c = np.cos(theta)[..., :, None, :]                          # [..., T, 1, D/2]
    s = np.sin(theta)[..., :, None, :]
    x1 = x[..., :h]
    x2 = x[..., h:]
    return np.concatenate([x1 * c - x2 * s, x1 * s + x2 * c], axis=-1)


# ---------------------------------------------------------------- step 3 --
def span_ids(S: int, spans_b: Optional[np.ndarray]) -> np.ndarray:
    """Per token: index of the image span [start, end) holding it, else -1
    ("Gemma explained", section "Vision encoder and processing": 256 soft
    tokens per image)."""
    sid = np.full(S, -1, dtype=np.int64)
    if spans_b is None:
        return sid
    for k, (st, en) in enumerate(_i64(spans_b)):
        sid[int(st):int(en)] = k
    return sid


def allowed(i, j, kind: int, window: int, sid: np.ndarray) -> np.ndarray:
    """The visibility predicate, vectorised over broadcastable i and j.

    Causal window of W keys on local layers, all earlier keys on global ones
    (Technical Report, section 1 Introduction and section 2 "5:1 interleaving
    of local/global layers"), joined with bidirectional attention inside one
    image ("Gemma explained", section "Vision encoder and processing").
    """
    i = np.asarray(i, dtype=np.int64)
    j = np.asarray(j, dtype=np.int64)
    causal = j <= i
    if kind == LOCAL:
        causal = causal & ((i - j) < int(window))
    same_image = (sid[i] == sid[j]) & (sid[i] >= 0)
    return causal | same_image


def allowed_row(i: int, S: int, kind: int, window: int, sid: np.ndarray) -> np.ndarray:
    """Visibility of every key j < S from query i (`allowed` on one row)."""
    return allowed(np.int64(i), np.arange(S, dtype=np.int64), kind, window, sid)


def unmasked_pairs(S: int, kind: int, window: int, spans_b=None) -> int:
    """Number of visible (i, j) pairs of one sequence, by enumeration of
    `allowed` (the predicate of step 3 above)."""
    sid = span_ids(S, spans_b)
    total = 0
    for i in range(S):
        total += int(np.count_nonzero(allowed_row(i, S, kind, window, sid)))
    return total


# --------------------------------------------------------------- step 4/5 --
def _prepare(q, k, v, q_gamma, k_gamma, positions, rope_base, interp):
    """Normalised and rotated q, k (float64) and v (float64), all [B,S,H,D]."""
    qh = rope(qk_rmsnorm(q, q_gamma), _f64(positions), rope_base, interp)
    kh = rope(qk_rmsnorm(k, k_gamma), _f64(positions), rope_base, interp)
    return qh, kh, _f64(v)


def _attend_rows(qh_b, kh_hm, v_hm, rows, kind, window, sid, S):
    """Attention of query rows `rows` of one sequence.

    qh_b [S, Hq, D]; kh_hm, v_hm head-major [Hkv, S, D].
    Returns out [len(rows), Hq, D] and lse [Hq, len(rows)].
    """
    Hq, D = qh_b.shape[1], qh_b.shape[2]
    Hkv = kh_hm.shape[0]
    G = Hq // Hkv
    rows = np.asarray(rows, dtype=np.int64)
    R = rows.size
    vis = allowed(rows[:, None], np.arange(S, dtype=np.int64)[None, :], kind, window, sid)  # [R, S]
    cols = np.nonzero(vis.any(axis=0))[0]
    j0, j1 = int(cols[0]), int(cols[-1]) + 1
    vis = vis[:, j0:j1]                                            # [R, n]
    q = qh_b[rows].reshape(R, Hkv, G, D).transpose(1, 2, 0, 3)     # [Hkv, G, R, D]
    q = q.reshape(Hkv, G * R, D)
    kt = kh_hm[:, j0:j1, :].transpose(0, 2, 1)                     # [Hkv, D, n]
    s = np.matmul(q, kt) / math.sqrt(D)                            # [Hkv, G*R, n]
    s = s.reshape(Hkv, G, R, j1 - j0)
    s = np.where(vis[None, None], s, -np.inf)
    m = s.max(axis=-1, keepdims=True)
    p = np.exp(s - m)                                              # 0 where masked
    l = p.sum(axis=-1, keepdims=True)
    o = np.matmul(p.reshape(Hkv, G * R, j1 - j0), v_hm[:, j0:j1, :])  # [Hkv, G*R, D]
    o = o.reshape(Hkv, G, R, D) / l
    lse = (m + np.log(l))[..., 0]                                  # [Hkv, G, R]
    out = o.transpose(2, 0, 1, 3).reshape(R, Hq, D)
    return out, lse.reshape(Hq, R)


def prefill_rows(q, k, v, q_gamma, k_gamma, positions, kind, window, rope_base, interp,
                 spans=None, rows: Optional[Sequence] = None, row_group: int = 64):
    """Attention output for selected query rows of every sequence.

    q [B,S,Hq,D], k/v [B,S,Hkv,D] raw (pre-norm, pre-RoPE); positions [B,S];
    spans [B,n,2] half-open or None; rows: 1-D list of row indices (all rows
    if None), the same for every sequence.
    Returns (out [B, R, Hq, D], lse [B, Hq, R]) in float64.  Steps 1-5 of the
    module docstring: GQA head mapping from the Technical Report, section 2;
    softmax with scale 1/sqrt(D) over each row's visible set.
    """
    B, S, Hq, D = q.shape
    rows = np.arange(S) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.empty((B, rows.size, Hq, D))
    lse = np.empty((B, Hq, rows.size))
    sp = None if spans is None else _i64(spans)
    pos = _f64(positions)
    for b in range(B):
        # Steps 1-2 for the keys of this sequence and for the requested query
        # rows only (a query row's result needs no other query row).
        kh = rope(qk_rmsnorm(k[b], k_gamma), pos[b], rope_base, interp)
        qsel = rope(qk_rmsnorm(q[b][rows], q_gamma), pos[b][rows], rope_base, interp)
        qh = np.zeros((S, Hq, D))
        qh[rows] = qsel
        sid = span_ids(S, None if sp is None else sp[b])
        kh_hm = np.ascontiguousarray(kh.transpose(1, 0, 2))
        v_hm = np.ascontiguousarray(_f64(v[b]).transpose(1, 0, 2))
        del kh
        for g0 in range(0, rows.size, row_group):
            sel = rows[g0:g0 + row_group]
            o, ls = _attend_rows(qh, kh_hm, v_hm, sel, kind, window, sid, S)
            out[b, g0:g0 + sel.size] = o
            lse[b, :, g0:g0 + sel.size] = ls
    return out, lse


def prefill(q, k, v, q_gamma, k_gamma, positions, kind, window, rope_base, interp, spans=None):
    """All rows: out [B,S,Hq,D] and lse [B,Hq,S] (float64); steps 1-5 of the
    module docstring (Technical Report, section 2; "Gemma explained")."""
    return prefill_rows(q, k, v, q_gamma, k_gamma, positions, kind, window, rope_base,
                        interp, spans, rows=None)


def prefill_bruteforce(q, k, v, q_gamma, k_gamma, positions, kind, window, rope_base, interp,
                       spans=None):
    """Second formulation: the full S x S score matrix per head, masked.

    Loops over every (batch, query head) and builds the whole mask with the
    predicate; meant for tiny inputs only.  Same definition and sources as
    `prefill`.
    """
    qh, kh, vf = _prepare(q, k, v, q_gamma, k_gamma, positions, rope_base, interp)
    B, S, Hq, D = qh.shape
    Hkv = kh.shape[2]
    G = Hq // Hkv
    out = np.empty_like(qh)
    lse = np.empty((B, Hq, S))
    ii, jj = np.meshgrid(np.arange(S), np.arange(S), indexing="ij")
    sp = None if spans is None else _i64(spans)
    for b in range(B):
        sid = span_ids(S, None if sp is None else sp[b])
        mask = allowed(ii, jj, kind, window, sid)
        for h in range(Hq):
            kv = h // G
            sc = qh[b, :, h, :] @ kh[b, :, kv, :].T / math.sqrt(D)
            sc = np.where(mask, sc, -np.inf)
            m = sc.max(axis=1, keepdims=True)
            p = np.exp(sc - m)
            l = p.sum(axis=1, keepdims=True)
            out[b, :, h, :] = (p / l) @ vf[b, :, kv, :]
            lse[b, h, :] = (m + np.log(l))[:, 0]
    return out, lse


# ----------------------------------------------------------------- decode --
def decode(q, k_new, v_new, q_gamma, k_gamma, seq_lens, k_hist, v_hist, hist_start,
           kind, window, rope_base, interp):
    """One decode step per sequence: row L-1 of the block attention.

    q [B,Hq,D], k_new/v_new [B,Hkv,D] raw; seq_lens [B] count the new token,
    whose position and index are L-1.  k_hist/v_hist: per sequence b a
    token-major [n_b, Hkv, D] array of the cached (already normalised and
    rotated) keys and values of tokens hist_start[b] .. L-2.  Every token
    older than hist_start[b] must be invisible from row L-1.

    Returns out [B,Hq,D] and the new token's rotated key k_hat [B,Hkv,D].
    The 1024-slot ring of local layers follows from the window (Technical
    Report, section 2 "5:1 interleaving": only global layers keep the long
    context's KV cache).
    """
    qf = _f64(q)
    B, Hq, D = qf.shape
    L = _i64(seq_lens)
    out = np.empty((B, Hq, D))
    k_hat = np.empty((B, _f64(k_new).shape[1], D))
    for b in range(B):
        Lb = int(L[b])
        pos = np.array([Lb - 1], dtype=np.float64)
        qh = rope(qk_rmsnorm(qf[b][None], q_gamma), pos, rope_base, interp)[0]        # [Hq, D]
        kn = rope(qk_rmsnorm(_f64(k_new)[b][None], k_gamma), pos, rope_base, interp)[0]
        k_hat[b] = kn
        t0 = int(hist_start[b])
        keys = np.concatenate([_f64(k_hist[b]), kn[None]], axis=0)                   # tokens t0..L-1
        vals = np.concatenate([_f64(v_hist[b]), _f64(v_new)[b][None]], axis=0)
        assert keys.shape[0] == Lb - t0
        sid = span_ids(Lb, None)
        if t0 > 0:
            assert not allowed(np.int64(Lb - 1), np.arange(t0), kind, window, sid).any()
        vis = allowed(np.int64(Lb - 1), np.arange(t0, Lb), kind, window, sid)
        Hkv = keys.shape[1]
        G = Hq // Hkv
        for h in range(Hq):
            kv = h // G
            s = keys[:, kv, :] @ qh[h] / math.sqrt(D)
            s = np.where(vis, s, -np.inf)
            m = s.max()
            p = np.exp(s - m)
            out[b, h] = p @ vals[:, kv, :] / p.sum()
    return out, k_hat
