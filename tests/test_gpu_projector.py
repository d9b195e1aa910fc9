"""Soft-token parity: g3attn_soft_tokens against the float64 oracle.

Inputs are bf16 patch features (N(0,1)) and fp32 gains 1 + 0.1 N(0,1); the
output is bf16, so the tolerance is the prefill one: max |err| <= 2e-2,
relative L2 <= 5e-3 (values are O(1) after the norm)."""
import numpy as np
import pytest
import torch

import global_gqa_b200 as g3
from oracle import projector as P
from gpu_helpers import assert_close, dev

pytestmark = pytest.mark.gpu

CASES = [
    # B, grid_h, grid_w, F, pool
    (3, 64, 64, 1152, 4),   # 896x896 images in 14x14 patches -> 256 soft tokens of 1152 features
    (2, 8, 12, 64, 2),
    (1, 4, 4, 8, 1),
    (2, 16, 8, 8192, 4),    # widest row the kernel is built for
    (1, 4, 8, 24, 4),       # F not a multiple of 32
]


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}_{c[1]}x{c[2]}_F{c[3]}_p{c[4]}" for c in CASES])
def test_soft_tokens(case):
    B, gh, gw, F, pool = case
    gen = torch.Generator().manual_seed(1000 + F + gh)
    x = torch.randn(B, gh * gw, F, generator=gen).to(torch.bfloat16)
    g = (1.0 + 0.1 * torch.randn(F, generator=gen)).float()
    out = g3.soft_tokens(x.to(dev()), g.to(dev()), gh, gw, pool)
    ref = P.soft_tokens(x.double().numpy(), g.double().numpy(), gh, gw, pool)
    assert out.shape == (B, (gh // pool) * (gw // pool), F)
    assert_close(out, ref, what="soft tokens")


def test_soft_tokens_refuses_cpu_tensors():
    x = torch.zeros(1, 16, 8, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        g3.soft_tokens(x, torch.ones(8), 4, 4, 4)
