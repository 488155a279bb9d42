"""Pins of the oracle's weighted Lloyd-Max grid fit ("aidendle94/GLM-5.2-
NF4-Lloyd-Experts-GPTQ", "What this is": 8 magnitudes fitted by weighted
Lloyd-Max over the pooled ratios |W / 2^e|, each weighted by (2^e)^2)."""
import numpy as np
import pytest

import oracle


def _bf16_bits(a):
    """Round fp32 values to bf16 (nearest even) and return the bit patterns."""
    u = np.ascontiguousarray(a, np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def _bits_value(b):
    return (b.astype(np.uint32) << 16).view(np.float32)


def test_uniform_data_converge_to_the_uniform_quantiser():
    # |U(-1, 1)| is U(0, 1), whose 8-level Lloyd-Max quantiser has levels
    # (2j + 1) / 16 (cells of width 1/8, each level its cell's midpoint).
    # With gmax = 1 every block's max is above 1/2, so every block has e = 0
    # and equal weights.  Lloyd steps on data this coarse (bf16: 2^-8 apart
    # near 1) stop once no ratio changes cell, which leaves the slowest mode
    # (a tilt of the spacing) a few thousandths from the optimum; starting
    # 0.01 off it in alternating directions, the fit lands within 0.01.
    rng = np.random.default_rng(7)
    w = _bf16_bits(rng.uniform(-1.0, 1.0, 1 << 18).astype(np.float32))
    assert np.all(np.abs(_bits_value(w)).reshape(-1, 32).max(1) > 0.5)
    opt = (2 * np.arange(8) + 1) / 16
    grid0 = (opt + 0.01 * (-1.0) ** np.arange(8)).astype(np.float32)
    grid0[7] = 1.0
    g, it = oracle.lloyd_fit(w, grid0, max_iter=5000, tol=0.0)
    assert it < 5000
    np.testing.assert_allclose(g, opt, atol=1e-2)
    # the same data with gmax = 0.9 put the blocks whose max exceeds 0.9 at
    # e = 1 (ratios halved, weight 4): a different fit, so the block exponent
    # and its weight enter
    g2, _ = oracle.lloyd_fit(w, (grid0 * 0.9).astype(np.float32), max_iter=5000, tol=0.0)
    assert np.abs(g2 - opt).max() > 0.03


def test_one_step_is_the_squared_scale_weighted_mean():
    # Two blocks whose ratios share the top cell: 0.75 at e = 0 (weight 1) and
    # -7/32 = -0.875 * 2^-2 at e = -2 (weight 2^-4).  One step moves the top
    # level to (32 * 0.75 + 32 * 0.875 / 16) / (32 + 32 / 16) = 25.75 / 34; the
    # unweighted mean would be 0.8125.  The empty cells keep their levels.
    w = np.concatenate([np.full(32, 0.75, np.float32), np.full(32, -7.0 / 32.0, np.float32)])
    grid0 = np.array([0.05, 0.1, 0.15, 0.2, 0.25, 0.3, 0.35, 1.0], np.float32)
    g, it = oracle.lloyd_fit(_bf16_bits(w), grid0, max_iter=1)
    assert it == 1
    assert g[7] == np.float32(25.75 / 34.0)
    assert np.array_equal(g[:7], grid0[:7])


def test_decoded_weights_are_a_fixed_point_of_their_own_grid():
    # Weights decoded from codes on a bf16-exact grid, with the top level in
    # every block: the pack rule gives back each block's own exponent, every
    # ratio is exactly a level, so the first step moves nothing.
    grid = np.array([0.125, 0.375, 0.625, 0.875, 1.25, 1.625, 2.0, 2.75], np.float32)
    rng = np.random.default_rng(3)
    N, K = 64, 256
    codes = rng.integers(0, 16, (N, K), dtype=np.uint8)
    codes[:, ::32] = 7 | (rng.integers(0, 2, (N, K // 32), dtype=np.uint8) << 3)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    scales = rng.integers(120, 136, (N, K // 32), dtype=np.uint8)  # sums of the weights stay exact in fp64
    w = oracle.dequant(packed[None], scales[None], grid, np.zeros(1, np.uint8), 1, N, K)
    g, it = oracle.lloyd_fit(w, grid, max_iter=50, tol=0.0)
    assert it == 1
    assert np.array_equal(g, grid)


def test_a_power_of_two_scale_of_all_weights_changes_nothing():
    rng = np.random.default_rng(11)
    w = rng.standard_normal(1 << 14).astype(np.float32) * 0.02
    grid0 = [0.13, 0.39, 0.66, 0.94, 1.26, 1.62, 2.07, 2.73]
    a = oracle.lloyd_fit(_bf16_bits(w), grid0, max_iter=300, tol=1e-13)
    b = oracle.lloyd_fit(_bf16_bits(w * 8.0), grid0, max_iter=300, tol=1e-13)
    assert a[1] == b[1]
    assert np.array_equal(a[0], b[0])


def test_levels_stay_ordered_and_within_the_starting_range():
    rng = np.random.default_rng(5)
    w = _bf16_bits(rng.standard_normal(1 << 14).astype(np.float32))
    grid0 = [0.13, 0.39, 0.66, 0.94, 1.26, 1.62, 2.07, 2.73]
    g, _ = oracle.lloyd_fit(w, grid0, max_iter=500, tol=1e-12)
    assert np.all(np.diff(g) > 0)
    assert g[0] >= 0.0 and g[7] <= np.float32(2.73)


def test_bad_inputs_are_rejected():
    w = np.zeros(64, np.uint16)
    with pytest.raises(oracle.OracleError):
        oracle.lloyd_fit(w, [0.1, 0.3, 0.2, 0.4, 0.5, 0.6, 0.7, 1.0], 3)  # not ascending
    with pytest.raises(oracle.OracleError):
        oracle.lloyd_fit(np.zeros(48, np.uint16), [0.1, 0.2, 0.3, 0.4, 0.5, 0.6, 0.7, 1.0], 3)
    bad = w.copy()
    bad[5] = 0x7FC0  # NaN
    with pytest.raises(oracle.OracleError):
        oracle.lloyd_fit(bad, [0.1, 0.2, 0.3, 0.4, 0.5, 0.6, 0.7, 1.0], 3)
