"""Assignment of independent attention units to ranks (one process per GPU).

The attention of one (sequence, kv head) pair reads only that sequence's keys
and values of that kv head and writes only the outputs of the kv head's query
heads (grouped-query attention, Gemma 3 Technical Report, section 2), in
prefill and in decode alike.  Ranks therefore split the units into contiguous
ranges and run with no exchange between them:

  * a batch of sequences (the 64-sequence decode) is split by sequence;
  * one long sequence (the 128K block) is split by kv head, each rank taking
    its kv heads together with their G query heads.

Ranges are balanced: the first `n % world` ranks take one unit more.  A rank
whose range is empty has no work.
"""
from __future__ import annotations

from typing import List, Tuple


def split(n: int, world: int, rank: int) -> Tuple[int, int]:
    """Half-open range [start, end) of the n units that `rank` of `world` takes."""
    if n < 0 or world < 1 or not 0 <= rank < world:
        raise ValueError(f"bad split: n={n} world={world} rank={rank}")
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def sequence_shard(B: int, world: int, rank: int) -> Tuple[int, int]:
    """Sequences [b0, b1) of a batch of B that this rank serves."""
    return split(B, world, rank)


def kv_head_shard(Hkv: int, G: int, world: int, rank: int) -> dict:
    """kv heads [kv0, kv1) of this rank and their query heads [q0, q1) (head
    h of the query reads kv head h // G)."""
    kv0, kv1 = split(Hkv, world, rank)
    return {"kv": (kv0, kv1), "q": (kv0 * G, kv1 * G)}


def rank_units(B: int, Hkv: int, world: int, rank: int, by: str) -> List[Tuple[int, int]]:
    """The (sequence, kv head) units of this rank when splitting by "sequence"
    or by "kv_head"."""
    if by == "sequence":
        b0, b1 = sequence_shard(B, world, rank)
        return [(b, h) for b in range(b0, b1) for h in range(Hkv)]
    if by == "kv_head":
        kv0, kv1 = split(Hkv, world, rank)
        return [(b, h) for b in range(B) for h in range(kv0, kv1)]
    raise ValueError(f"unknown split {by!r}")
