"""Shared helpers of the GPU parity tests (inputs on the device, comparisons)."""
import numpy as np
import torch

import global_gqa_b200 as g3
from oracle import attention as O

ATOL = 2e-2      # max |gpu - oracle| on outputs
REL_L2 = 5e-3    # ||gpu - oracle||_2 / ||oracle||_2 on outputs
LSE_ATOL = 2e-2  # log-sum-exp of scaled scores


def dev():
    return torch.device("cuda", 0)


def to_dev(d: dict) -> dict:
    return {k: (None if v is None else v.to(dev()).contiguous()) for k, v in d.items()}


def assert_close(got, ref, atol=ATOL, rel_l2=REL_L2, what="out"):
    g = got.detach().double().cpu().numpy() if isinstance(got, torch.Tensor) else np.asarray(got, float)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite values"
    d = np.abs(g - r)
    rel = np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30)
    assert d.max() <= atol, f"{what}: max abs err {d.max():.3e} > {atol} at {np.unravel_index(d.argmax(), d.shape)}"
    assert rel <= rel_l2, f"{what}: rel L2 err {rel:.3e} > {rel_l2}"
    return d.max(), rel


def run_prefill(x: dict, kind, window, base, interp, return_lse=True, **kw):
    return g3.prefill(x["q"], x["k"], x["v"], x["q_gamma"], x["k_gamma"], x["positions"], kind, window,
                      base, interp, x.get("spans"), return_lse=return_lse, **kw)


def oracle_rows(xc: dict, kind, window, base, interp, rows=None):
    return O.prefill_rows(xc["q"], xc["k"], xc["v"], xc["q_gamma"], xc["k_gamma"], xc["positions"], kind,
                          window, base, interp, xc.get("spans"), rows=rows)


def sampled_rows(S, window, spans=None, n_random=256, seed=0):
    """Rows for full-size parity: first/last two tiles, edges, spans, random."""
    rng = np.random.default_rng(seed)
    rows = set(range(min(S, 256))) | set(range(max(0, S - 256), S))
    for e in (window - 1, window, window + 1, 127, 128, 129, S // 2):
        for d in range(-8, 9):
            if 0 <= e + d < S:
                rows.add(e + d)
    if spans is not None:
        sp = np.asarray(spans).reshape(-1, 2)
        for k, (st, en) in enumerate(sp):
            for e in (st, en - 1, en):
                for d in range(-8, 9):
                    if 0 <= e + d < S:
                        rows.add(int(e + d))
            if k < 2:
                rows.update(range(int(st), int(en)))
    rows.update(rng.integers(0, S, n_random).tolist())
    return np.array(sorted(rows), dtype=np.int64)
