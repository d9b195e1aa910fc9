"""Work accounting for the benchmark: unmasked FLOPs and algorithmic bytes.

The visible keys of query row i form one interval [lo_i, hi_i] (the causal
window and the row's image span both contain i), so a sequence's visible
pairs are sum_i (hi_i - lo_i + 1).  FLOPs count only those pairs:
QK^T and PV each take 2*D multiply-adds per (query head, pair), i.e.
4 * D * Hq * pairs per layer.
"""
from __future__ import annotations

from typing import Optional, Sequence

import numpy as np

LOCAL = 0
GLOBAL = 1


def row_intervals(S: int, kind: int, window: int, spans_b: Optional[Sequence] = None):
    i = np.arange(S, dtype=np.int64)
    lo = np.zeros(S, dtype=np.int64) if kind == GLOBAL else np.maximum(0, i - int(window) + 1)
    hi = i.copy()
    if spans_b is not None:
        for st, en in np.asarray(spans_b, dtype=np.int64).reshape(-1, 2):
            lo[st:en] = np.minimum(lo[st:en], st)
            hi[st:en] = np.maximum(hi[st:en], en - 1)
    return lo, hi


def visible_pairs(S: int, kind: int, window: int, spans_b=None) -> int:
    lo, hi = row_intervals(S, kind, window, spans_b)
    return int(np.sum(hi - lo + 1))


def layer_flops(B: int, S: int, Hq: int, D: int, kind: int, window: int, spans=None) -> float:
    total = 0
    for b in range(B):
        sb = None if spans is None else np.asarray(spans[b])
        total += visible_pairs(S, kind, window, sb)
    return 4.0 * D * Hq * total


def block_flops(B, S, Hq, D, layers, spans=None) -> float:
    """Sum over the layers of a block; `layers` items have .kind and .window."""
    return sum(layer_flops(B, S, Hq, D, l.kind, l.window, spans) for l in layers)


def decode_kv_bytes(seq_lens, Hkv: int, D: int, kind: int, window: int) -> int:
    """Cached K and V bytes one decode call must read (bf16)."""
    L = np.asarray(seq_lens, dtype=np.int64)
    n = L if kind == GLOBAL else np.minimum(L, int(window))
    return int(np.sum(n) * Hkv * D * 2 * 2)
