"""The soft-token oracle's pins must catch plausible mistakes.

Each case replaces the oracle's soft_tokens with a copy holding one planted
error and asserts that at least one pin of test_oracle_projector fails.
"""
import numpy as np
import pytest

from oracle import projector as P
import test_oracle_projector as PINS


def _factory(norm_first=False, column_major=False, no_eps=False, no_gamma=False, sum_not_mean=False):
    def soft_tokens(patches, gamma, grid_h, grid_w, pool=4):
        x = np.asarray(patches, dtype=np.float64)
        g = np.asarray(gamma, dtype=np.float64)
        B, n, F = x.shape
        eps = 0.0 if no_eps else P.EPS

        def norm(y):
            red = np.sum if sum_not_mean else np.mean
            out = y / np.sqrt(red(y * y, axis=-1, keepdims=True) + eps)
            return out if no_gamma else out * g

        if norm_first:
            x = norm(x) / (1.0 if no_gamma else g)
        th, tw = grid_h // pool, grid_w // pool
        if column_major:
            grid = x.reshape(B, grid_w, grid_h, F).transpose(0, 2, 1, 3)
            grid = grid.reshape(B, th, pool, tw, pool, F)
        else:
            grid = x.reshape(B, th, pool, tw, pool, F)
        pooled = grid.mean(axis=(2, 4)).reshape(B, th * tw, F)
        return pooled * g if norm_first and not no_gamma else (pooled if norm_first else norm(pooled))
    return soft_tokens


MUTANTS = {
    "norm_before_pool": _factory(norm_first=True),
    "pool_column_major": _factory(column_major=True),
    "norm_drops_eps": _factory(no_eps=True),
    "norm_drops_gamma": _factory(no_gamma=True),
    "rms_uses_sum": _factory(sum_not_mean=True),
}

PIN_FUNCS = [f for n, f in sorted(vars(PINS).items()) if n.startswith("test_") and callable(f)]


def test_unmutated_copy_matches():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((2, 8 * 12, 6))
    g = 1.0 + 0.1 * rng.standard_normal(6)
    np.testing.assert_allclose(_factory()(x, g, 8, 12, 4), P.soft_tokens(x, g, 8, 12, 4), rtol=1e-13, atol=0)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, monkeypatch):
    monkeypatch.setattr(P, "soft_tokens", MUTANTS[name])
    caught = []
    for pin in PIN_FUNCS:
        try:
            pin()
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin caught mutant {name}"
