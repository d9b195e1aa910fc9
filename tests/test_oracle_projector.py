"""Pins of the soft-token oracle (pool then RMS norm) against facts that do
not come from the oracle itself: brute-force block means, closed forms and the
printed sizes of "Gemma explained: what's new in Gemma 3"."""
import numpy as np

from oracle import projector as P


def _rand(B, gh, gw, F, seed=0):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((B, gh * gw, F)), 1.0 + 0.1 * rng.standard_normal(F)


def test_printed_sizes_give_256_tokens():
    # 896x896 image, 14x14 patches -> 64x64 grid (4096 position embeddings); 4x4 pool -> 256
    grid = 896 // 14
    assert grid * grid == 4096
    x, g = _rand(1, grid, grid, 8)
    assert P.soft_tokens(x, g, grid, grid, 4).shape == (1, 256, 8)


def test_pool_is_block_mean_in_raster_order():
    B, gh, gw, F, k = 2, 8, 12, 5, 4
    x, g = _rand(B, gh, gw, F, 1)
    out = P.soft_tokens(x, np.ones(F), gh, gw, k)
    for b in range(B):
        for ty in range(gh // k):
            for tx in range(gw // k):
                block = [x[b, (ty * k + dy) * gw + tx * k + dx] for dy in range(k) for dx in range(k)]
                m = np.mean(block, axis=0)
                want = m / np.sqrt(np.mean(m * m) + P.EPS)
                np.testing.assert_allclose(out[b, ty * (gw // k) + tx], want, rtol=1e-12, atol=1e-12)


def test_constant_blocks_normalise_to_gamma_sign():
    # every patch of a block equal to c -> token = c / sqrt(c^2 + eps) * gamma per feature
    gh = gw = 8
    F = 4
    c = np.array([2.0, -3.0, 0.5, 1.0])
    x = np.tile(c, (1, gh * gw, 1))
    g = np.array([1.0, 2.0, 3.0, 4.0])
    out = P.soft_tokens(x, g, gh, gw, 4)
    ms = np.mean(c * c)
    np.testing.assert_allclose(out[0, 0], c / np.sqrt(ms + P.EPS) * g, rtol=1e-12)
    np.testing.assert_allclose(out[0], np.tile(out[0, 0], (4, 1)), rtol=0, atol=0)


def test_unit_rms_after_norm():
    x, _ = _rand(3, 16, 16, 64, 2)
    out = P.soft_tokens(x, np.ones(64), 16, 16, 4)
    rms = np.sqrt(np.mean(out * out, axis=-1))
    ms = np.mean(x.reshape(3, 4, 4, 4, 4, 64).mean(axis=(2, 4)).reshape(3, 16, 64) ** 2, axis=-1)
    np.testing.assert_allclose(rms, np.sqrt(ms / (ms + P.EPS)), rtol=1e-12)


def test_pool_one_is_plain_rmsnorm():
    x, g = _rand(1, 4, 4, 16, 3)
    out = P.soft_tokens(x, g, 4, 4, 1)
    want = x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + P.EPS) * g
    np.testing.assert_allclose(out, want, rtol=1e-12)


def test_norm_after_pool_not_before():
    # Normalising patches before pooling gives a different result on unequal norms.
    x = np.zeros((1, 16, 2))
    x[0, :, 0] = np.arange(1, 17)
    x[0, :, 1] = 1.0
    out = P.soft_tokens(x, np.ones(2), 4, 4, 4)[0, 0]
    m = x[0].mean(axis=0)
    np.testing.assert_allclose(out, m / np.sqrt(np.mean(m * m) + P.EPS), rtol=1e-12)
    pre = x[0] / np.sqrt(np.mean(x[0] ** 2, axis=-1, keepdims=True) + P.EPS)
    assert not np.allclose(out, pre.mean(axis=0))
