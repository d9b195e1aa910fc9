"""The binding refuses malformed caller buffers before anything is launched."""
import pytest
import torch

import global_gqa_b200 as g3
import inputs

pytestmark = pytest.mark.gpu


def _layer(S=256):
    x = inputs.prefill_layer_inputs(1, S, 4, 2, 64, seed=3)
    return {k: (None if v is None else v.cuda()) for k, v in x.items()}


def test_prefill_rejects_wrong_out_and_workspace():
    x = _layer()
    args = (x["q"], x["k"], x["v"], x["q_gamma"], x["k_gamma"], x["positions"], 0, 1024, 1e4, 1.0)
    with pytest.raises(ValueError, match="out must have shape"):
        g3.prefill(*args, out=torch.empty(1, 128, 4, 64, dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(TypeError, match="out must be"):
        g3.prefill(*args, out=torch.empty(1, 256, 4, 64, dtype=torch.float32, device="cuda"))
    with pytest.raises(ValueError, match="ws must be"):
        g3.prefill(*args, ws=torch.empty(1 << 20, dtype=torch.uint8))
    with pytest.raises(ValueError, match="k_cache must be"):
        g3.prefill(*args, k_cache=torch.empty(1, 1024, 2, 64, dtype=torch.bfloat16, device="cuda"),
                   v_cache=torch.empty(1, 1024, 2, 64, dtype=torch.bfloat16, device="cuda"))
    # A float32 workspace of enough bytes is accepted (sizes are counted in bytes).
    need = g3.prefill_workspace_size(1, 256, 4, 2, 64)
    out = g3.prefill(*args, ws=torch.empty((need + 3) // 4, dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()


def test_decode_rejects_wrong_out():
    B, Hq, Hkv, D, cap = 2, 4, 2, 64, 1024
    q = torch.randn(B, Hq, D, device="cuda").bfloat16()
    kn = torch.randn(B, Hkv, D, device="cuda").bfloat16()
    gam = torch.ones(D, device="cuda")
    kc = torch.zeros(B, Hkv, cap, D, dtype=torch.bfloat16, device="cuda")
    lens = torch.full((B,), 10, dtype=torch.int32, device="cuda")
    with pytest.raises(ValueError, match="out must have shape"):
        g3.decode(q, kn, kn, gam, gam, kc, kc.clone(), lens, 1024, 0, 1024, 1e4, 1.0,
                  out=torch.empty(B, Hq, D // 2, dtype=torch.bfloat16, device="cuda"))
