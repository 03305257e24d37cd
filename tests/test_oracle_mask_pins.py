"""Pins of the target-mask preparation oracle (CPU)."""
import math

import numpy as np
import pytest

import oracle


def test_shot_lengths_from_the_page(golden_rule):
    period = int(golden_rule["shot_length_period"][0])
    offset = int(golden_rule["shot_length_offset"][0])
    assert oracle.shot_length_ok(int(golden_rule["valid_shot_length"][0]))
    for n in range(10):
        assert oracle.shot_length_ok(period * n + offset)
        assert not oracle.shot_length_ok(period * n + offset + 1)
    assert oracle.mask_length_ok(1, 107) and oracle.mask_length_ok(107, 107)
    assert not oracle.mask_length_ok(360, 107)      # a whole-clip mask into a 107-frame shot
    assert not oracle.mask_length_ok(106, 107)
    with pytest.raises(ValueError):
        oracle.prepare_target_mask(np.zeros((360, 8, 8)), 107, 26, 4, 4, 4)


def test_area_weights_partition_unity():
    for n_in, n_out in ((720, 40), (7, 3), (5, 5), (3, 7), (1280, 50)):
        W = oracle.area_weights(n_in, n_out)
        np.testing.assert_allclose(W.sum(1), 1.0, atol=1e-12)
        # every input cell is fully used: column sums * (n_in/n_out) == 1
        np.testing.assert_allclose(W.sum(0) * (n_in / n_out), 1.0, atol=1e-12)


def test_integer_ratio_is_block_mean():
    rng = np.random.Generator(np.random.PCG64(3))
    m = rng.uniform(0, 1, (1, 36, 48))
    out = oracle.prepare_target_mask(m, 5, 1, 4, 6, 8)
    blocks = m[0].reshape(6, 6, 8, 6).mean(axis=(1, 3))
    np.testing.assert_allclose(out[0], blocks, atol=1e-14)


def test_fractional_ratio_equals_supersampled_block_mean():
    # replicate every pixel k x k times so cell boundaries fall on pixel edges, then take plain
    # block means: the exact area average by brute force
    rng = np.random.Generator(np.random.PCG64(4))
    Hp, Wp, Hq, Wq = 7, 10, 3, 4
    m = rng.uniform(0, 1, (1, Hp, Wp))
    out = oracle.prepare_target_mask(m, 5, 1, 4, Hq, Wq)
    ky, kx = Hq, Wq   # Hp*ky divisible by Hq, Wp*kx divisible by Wq
    big = np.repeat(np.repeat(m[0], ky, axis=0), kx, axis=1)
    ref = big.reshape(Hq, Hp * ky // Hq, Wq, Wp * kx // Wq).mean(axis=(1, 3))
    np.testing.assert_allclose(out[0], ref, atol=1e-14)


def test_mass_and_constants():
    rng = np.random.Generator(np.random.PCG64(5))
    m = rng.uniform(0, 1, (22, 45, 61))   # 22 = 17*1 + 5
    out = oracle.prepare_target_mask(m, 22, 6, 4, 9, 13)
    # area-weighted mean over the grid equals the input mean of the frames each span covers
    for f in range(6):
        t0, t1 = 4 * f, min(4 * f + 4, 22)
        assert out[f].mean() == pytest.approx(m[t0:t1].mean(), abs=1e-12)
    c = np.full((1, 30, 40), 0.37)
    assert np.allclose(oracle.prepare_target_mask(c, 107, 26, 4, 7, 9), 0.37, atol=1e-15)


def test_temporal_spans_and_static_mask():
    L, tau, F_lat = 107, 4, 27
    vals = np.arange(L, dtype=np.float64) / L
    m = np.broadcast_to(vals[:, None, None], (L, 8, 8)).copy()
    out = oracle.prepare_target_mask(m, L, F_lat, tau, 2, 2)
    for f in range(F_lat):
        expect = vals[f * tau:min(f * tau + tau, L)].mean()
        assert np.allclose(out[f], expect, atol=1e-15)
    assert F_lat * tau > L               # the last span is short (3 frames): still averaged
    # a one-frame mask applies unchanged to every latent frame (frame 5: not all zeros)
    static = oracle.prepare_target_mask(m[5:6], L, 26, 4, 2, 2)
    assert static.shape == (26, 2, 2) and np.allclose(static, vals[5]) and vals[5] > 0
    with pytest.raises(ValueError):
        oracle.prepare_target_mask(m, L, 28, 4, 2, 2)   # latent frame 27 starts past the shot
