"""Plain float64 definition of Gemma 3's image soft tokens (test infrastructure).

ORACLE -- test infrastructure, not product code.  Only tests, the smoke check
and the benchmark's CPU-baseline leg may use this module.  It shares no code
with the CUDA library.

"Gemma explained: what's new in Gemma 3" prints the multimodal projector of
the 27B model as two modules, an RMSNorm over the 1152 vision features
(eps 1e-6) and a 4x4 average pool with stride 4, and says an image becomes a
fixed 256 soft tokens.  The vision encoder takes 896x896 images in 14x14
patches (its patch embedding and its 4096-entry position embedding in the same
printout), i.e. a 64x64 grid of patch vectors, which the pool turns into 16x16
= 256 tokens.

Readings of what the page leaves open:
- patches are in raster order of the grid (index = row * grid_w + col), and
  soft tokens likewise (index = row * (grid_w / pool) + col);
- the pool comes first and the norm applies to each pooled (soft) token, as the
  norm's name says (a norm of the soft embeddings);
- the gain multiplies directly (x_hat * gamma), as in the attention's
  QK-norm;
- the projection to the language model's width is a trained parameter the
  printout does not show; it is not part of this op.
"""
from __future__ import annotations

import numpy as np

EPS = 1e-6


def soft_tokens(patches, gamma, grid_h: int, grid_w: int, pool: int = 4):
    """patches [B, grid_h*grid_w, F] -> soft tokens [B, (grid_h/pool)*(grid_w/pool), F], float64.

    Step 1: average each pool x pool block of the patch grid (no padding).
    Step 2: RMS-normalise every pooled vector over its F features (eps 1e-6)
            and multiply by gamma.
    The projector's printed modules and the 256 tokens per image: "Gemma
    explained: what's new in Gemma 3", the 27B model's printout and section
    "Vision encoder and processing".
    """
    x = np.asarray(patches, dtype=np.float64)
    g = np.asarray(gamma, dtype=np.float64)
    B, n, F = x.shape
    assert n == grid_h * grid_w and grid_h % pool == 0 and grid_w % pool == 0
    th, tw = grid_h // pool, grid_w // pool
    grid = x.reshape(B, th, pool, tw, pool, F)
    pooled = grid.mean(axis=(2, 4)).reshape(B, th * tw, F)
    ms = np.mean(pooled * pooled, axis=-1, keepdims=True)
    return pooled / np.sqrt(ms + EPS) * g
