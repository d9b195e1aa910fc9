"""Seeded synthetic inputs for the Gemma 3 5:1 attention block.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests.  It holds workload shapes and random-number recipes only: no
normalisation, rotation, masking or softmax arithmetic lives here.

Shapes follow the 27B module printout on "Gemma explained: what's new in
Gemma 3" (section "Gemma 3 27B": q_proj 5376->4096, k/v_proj 5376->2048,
q_norm/k_norm over 128 features, hence 32 query heads, 16 key/value heads,
head_dim 128).  The block layout (five sliding-window layers of span 1024,
RoPE base 10k, then one global layer, RoPE base 1M) follows the Gemma 3
Technical Report, section 2 "5:1 interleaving of local/global layers" and
"Long context".  Image soft-token spans hold 256 tokens (Technical Report,
section 1 Introduction).

Recipe (fixed, documented):
  * every tensor draws from its own CPU torch.Generator seeded with
    seed_for(seed, layer, tensor_id) = 1_000_003*seed + 101*layer + tensor_id
    (tensor ids: q=0, k=1, v=2, q_gamma=3, k_gamma=4, spans=5, lens=6,
    k_cache=7, v_cache=8, dout=9);
  * q, k, v ~ N(0, 1) drawn in fp32 and rounded to bf16;
  * gamma = 1 + 0.1 * N(0, 1), fp32;
  * positions = 0 .. S-1 for every sequence;
  * image spans: per sequence, draw n integers uniformly in [0, S - n*256],
    sort them (g_k) and place span k at g_k + 256*k, so spans are disjoint and
    may touch;
  * decode context lengths: uniform integers in [lo, hi], inclusive.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional

import torch

LOCAL = 0
GLOBAL = 1

T_Q, T_K, T_V, T_QG, T_KG, T_SPANS, T_LENS, T_KC, T_VC, T_DOUT = range(10)

IMAGE_SPAN_TOKENS = 256


def seed_for(seed: int, layer: int, tensor_id: int) -> int:
    return 1_000_003 * int(seed) + 101 * int(layer) + int(tensor_id)


def _gen(seed: int, layer: int, tensor_id: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed_for(seed, layer, tensor_id))
    return g


@dataclass(frozen=True)
class LayerSpec:
    kind: int            # LOCAL or GLOBAL
    window: int          # used only when kind == LOCAL
    rope_base: float
    interp: float        # positions are divided by this factor before RoPE


def gemma3_block(global_interp: float = 8.0, window: int = 1024) -> List[LayerSpec]:
    """Five local layers then one global layer (local layer first)."""
    local = LayerSpec(LOCAL, window, 10_000.0, 1.0)
    glob = LayerSpec(GLOBAL, window, 1_000_000.0, float(global_interp))
    return [local] * 5 + [glob]


@dataclass(frozen=True)
class PrefillConfig:
    name: str
    B: int
    S: int
    Hq: int
    Hkv: int
    D: int
    n_spans: int = 0
    global_interp: float = 8.0
    seed: int = 0

    def block(self) -> List[LayerSpec]:
        return gemma3_block(self.global_interp)


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    len_lo: int
    len_hi: int
    global_capacity: int
    window: int = 1024
    global_interp: float = 8.0
    seed: int = 0

    def block(self) -> List[LayerSpec]:
        return gemma3_block(self.global_interp, self.window)


# The five synthetic workloads (tiny block, 27B-shaped 8K block, mixed
# text+image 32K block, 128K block, batched decode).
TINY_BLOCK = PrefillConfig("tiny_block_s2048_h4x2_d64", 1, 2048, 4, 2, 64, 0, global_interp=1.0)
BLOCK_8K = PrefillConfig("gemma3_27b_block_s8192", 1, 8192, 32, 16, 128, 0, global_interp=8.0)
MIXED_32K = PrefillConfig("gemma3_27b_mixed_b2_s32768_8img", 2, 32768, 32, 16, 128, 8, global_interp=1.0)
LONG_128K = PrefillConfig("gemma3_27b_block_s131072", 1, 131072, 32, 16, 128, 0, global_interp=8.0)
DECODE_B64 = DecodeConfig("gemma3_27b_decode_b64_l4k_128k", 64, 32, 16, 128, 4096, 131072, 131072)

PREFILL_CONFIGS = {c.name: c for c in (TINY_BLOCK, BLOCK_8K, MIXED_32K, LONG_128K)}


def randn_bf16(shape, seed: int, layer: int, tensor_id: int) -> torch.Tensor:
    g = _gen(seed, layer, tensor_id)
    return torch.randn(*shape, generator=g, dtype=torch.float32).to(torch.bfloat16)


def gamma(D: int, seed: int, layer: int, tensor_id: int) -> torch.Tensor:
    g = _gen(seed, layer, tensor_id)
    return (1.0 + 0.1 * torch.randn(D, generator=g, dtype=torch.float32)).contiguous()


def image_spans(B: int, S: int, n: int, seed: int, layer: int = 0,
                span_len: int = IMAGE_SPAN_TOKENS) -> Optional[torch.Tensor]:
    """[B, n, 2] int32 half-open [start, end) spans, sorted and disjoint."""
    if n == 0:
        return None
    free = S - n * span_len
    if free < 0:
        raise ValueError("spans do not fit in the sequence")
    g = _gen(seed, layer, T_SPANS)
    out = torch.empty(B, n, 2, dtype=torch.int32)
    for b in range(B):
        gaps = torch.randint(0, free + 1, (n,), generator=g, dtype=torch.int64)
        gaps, _ = torch.sort(gaps)
        starts = gaps + span_len * torch.arange(n, dtype=torch.int64)
        out[b, :, 0] = starts.to(torch.int32)
        out[b, :, 1] = (starts + span_len).to(torch.int32)
    return out


def positions(B: int, S: int, offset: int = 0) -> torch.Tensor:
    return (torch.arange(S, dtype=torch.int32) + offset).unsqueeze(0).repeat(B, 1).contiguous()


def prefill_layer_inputs(B: int, S: int, Hq: int, Hkv: int, D: int, *, seed: int = 0,
                         layer: int = 0, n_spans: int = 0) -> dict:
    """Raw (pre-norm, pre-RoPE) bf16 q/k/v in [B, S, H, D] token-major layout."""
    return dict(
        q=randn_bf16((B, S, Hq, D), seed, layer, T_Q),
        k=randn_bf16((B, S, Hkv, D), seed, layer, T_K),
        v=randn_bf16((B, S, Hkv, D), seed, layer, T_V),
        q_gamma=gamma(D, seed, layer, T_QG),
        k_gamma=gamma(D, seed, layer, T_KG),
        positions=positions(B, S),
        spans=image_spans(B, S, n_spans, seed, layer),
    )


def prefill_backward_inputs(B: int, S: int, Hq: int, Hkv: int, D: int, *, seed: int = 0,
                            layer: int = 0, n_spans: int = 0) -> dict:
    """A layer's prefill inputs plus the output gradient dout [B, S, Hq, D] (bf16, N(0, 1))."""
    x = prefill_layer_inputs(B, S, Hq, Hkv, D, seed=seed, layer=layer, n_spans=n_spans)
    x["dout"] = randn_bf16((B, S, Hq, D), seed, layer, T_DOUT)
    return x


def config_layer_inputs(cfg: PrefillConfig, layer: int) -> dict:
    return prefill_layer_inputs(cfg.B, cfg.S, cfg.Hq, cfg.Hkv, cfg.D, seed=cfg.seed,
                                layer=layer, n_spans=cfg.n_spans)


def decode_lengths(B: int, lo: int, hi: int, seed: int, layer: int = 0) -> torch.Tensor:
    g = _gen(seed, layer, T_LENS)
    return torch.randint(lo, hi + 1, (B,), generator=g, dtype=torch.int64).to(torch.int32)


def decode_step_inputs(B: int, Hq: int, Hkv: int, D: int, *, seed: int = 0, layer: int = 0) -> dict:
    """Raw bf16 q [B,Hq,D] and the new token's k/v [B,Hkv,D]."""
    return dict(
        q=randn_bf16((B, Hq, D), seed, layer, T_Q),
        k_new=randn_bf16((B, Hkv, D), seed, layer, T_K),
        v_new=randn_bf16((B, Hkv, D), seed, layer, T_V),
        q_gamma=gamma(D, seed, layer, T_QG),
        k_gamma=gamma(D, seed, layer, T_KG),
    )


def cache_history(n_tokens: int, Hkv: int, D: int, *, seed: int, layer: int, batch: int) -> dict:
    """Cached key/value rows of one sequence, token-major [n_tokens, Hkv, D] bf16.

    The key rows stand for already normalised and rotated keys; the recipe
    only needs N(0,1) values of the right shape.  Each (layer, sequence) has
    its own stream so any single sequence can be regenerated on its own.
    """
    kseed = seed_for(seed, layer, T_KC) * 131 + batch
    vseed = seed_for(seed, layer, T_VC) * 131 + batch
    gk = torch.Generator(device="cpu"); gk.manual_seed(kseed)
    gv = torch.Generator(device="cpu"); gv.manual_seed(vseed)
    k = torch.randn(n_tokens, Hkv, D, generator=gk, dtype=torch.float32).to(torch.bfloat16)
    v = torch.randn(n_tokens, Hkv, D, generator=gv, dtype=torch.float32).to(torch.bfloat16)
    return dict(k=k, v=v)


def device_fill_normal_bf16(t: torch.Tensor, seed: int) -> torch.Tensor:
    """Fill a (large) device tensor with N(0,1) bf16 from torch's own generator."""
    g = torch.Generator(device=t.device)
    g.manual_seed(int(seed))
    flat = t.view(-1)
    step = 1 << 28
    for s in range(0, flat.numel(), step):
        e = min(flat.numel(), s + step)
        flat[s:e] = torch.randn(e - s, generator=g, device=t.device, dtype=torch.float32).to(t.dtype)
    return t
