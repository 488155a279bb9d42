"""Pins for the oracle's pack ("aidendle94/GLM-5.2-NF4-Lloyd-Experts-GPTQ",
"Codes are indices into the per-layer grid -- not E2M1": codes packed against
gmax * 2^e >= amax; "Contents": block 32 along K, low nibble = even K)."""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from bit_codebook_quantized_router_b200 import inputs
from tests import helpers

HAND = np.array([0.125, 0.375, 0.625, 0.875, 1.25, 1.625, 2.0625, 2.75], np.float32)
TABLES = {"E2M1": inputs.E2M1_TABLE, "HAND": HAND}


def test_hand_packed_blocks():
    for name, scale, packed, values in helpers.read_pack_golden():
        bits = helpers.f32_to_bf16_bits(values)
        assert np.array_equal(helpers.bf16_bits_to_f32(bits), values)  # exact in bf16
        w, s = oracle.pack(bits[None, None], TABLES[name][None], np.zeros(1, np.uint8), 1, 1, 32)
        assert int(s[0, 0, 0]) == scale, name
        assert bytes(w[0, 0]) == packed, (name, bytes(w[0, 0]).hex())


def _brute_exponent(amax, gmax):
    # Smallest integer e in [-127, 127] with gmax * 2^e >= amax, by scanning
    # with exact rational arithmetic (clamped to the E8M0 range).
    g, a = Fraction(float(gmax)), Fraction(float(amax))
    for e in range(-127, 128):
        if g * Fraction(2) ** e >= a:
            return e
    return 127


def _random_blocks(rng, n, scale_spread=True):
    base = rng.standard_normal((n, 32)) * 0.02
    if scale_spread:
        base *= 2.0 ** rng.integers(-20, 20, (n, 1))
    base[rng.random((n, 32)) < 0.05] = 0.0
    return helpers.f32_to_bf16_bits(base.astype(np.float32))


@pytest.mark.parametrize("table_name", ["E2M1", "HAND", "LLOYD"])
def test_pack_brute_force_over_exponents_and_signed_levels(table_name):
    table = inputs.lloyd_max_grid(0) if table_name == "LLOYD" else TABLES[table_name]
    rng = np.random.default_rng(11)
    bits = _random_blocks(rng, 300)
    w, s = oracle.pack(bits[None], table[None], np.zeros(1, np.uint8), 1, 300, 32)
    x = helpers.bf16_bits_to_f32(bits).astype(np.float64)
    gmax = float(np.max(table))
    # every signed level value, as exact rationals
    levels = [(c, (-1 if c & 8 else 1) * Fraction(float(table[c & 7]))) for c in range(16)]
    for n in range(300):
        e = _brute_exponent(np.max(np.abs(x[n])), gmax)
        assert int(s[0, n, 0]) == e + 127
        sc = Fraction(2) ** e
        for i in range(32):
            byte = int(w[0, n, i // 2])
            code = byte & 15 if i % 2 == 0 else byte >> 4
            xi = Fraction(float(x[n, i]))
            # nearest signed level by exhaustive search over all 16 codes
            dist = {c: abs(xi - v * sc) for c, v in levels}
            best = min(dist.values())
            assert dist[code] == best, (n, i, code)
            # ties: the lower magnitude index; a zero input keeps the + sign
            tied = sorted(c & 7 for c, d in dist.items() if d == best)
            assert (code & 7) == tied[0]
            if xi > 0:
                assert not code & 8
            elif xi < 0:
                assert code & 8 or table[code & 7] == 0
            else:
                assert not code & 8


def test_block_max_lands_in_top_octave():
    grid = inputs.lloyd_max_grid(0)
    rng = np.random.default_rng(3)
    bits = _random_blocks(rng, 500)
    w, s = oracle.pack(bits[None], grid[None], np.zeros(1, np.uint8), 1, 500, 32)
    x = helpers.bf16_bits_to_f32(bits).astype(np.float64)
    for n in range(500):
        amax = np.max(np.abs(x[n]))
        e = int(s[0, n, 0]) - 127
        if amax == 0:
            assert e == -127
            continue
        if -127 < e < 127:
            assert grid.max() * 2.0 ** (e - 1) < amax <= grid.max() * 2.0 ** e


def test_round_trip_decode_is_nearest_level():
    grid = inputs.lloyd_max_grid(0)
    rng = np.random.default_rng(4)
    bits = _random_blocks(rng, 200, scale_spread=False)
    w, s = oracle.pack(bits[None], grid[None], np.zeros(1, np.uint8), 1, 200, 32)
    dec = oracle.decode_matrix_f64(w[0], s[0], grid, 200, 32)
    x = helpers.bf16_bits_to_f32(bits).astype(np.float64)
    sc = 2.0 ** (s[0, :, 0].astype(np.float64) - 127)
    cand = grid.astype(np.float64)[None, None, :] * sc[:, None, None]
    d = np.abs(np.abs(x)[:, :, None] - cand)
    idx = np.argmin(d, axis=2)  # numpy argmin returns the first (lowest) index on ties
    ref = np.take_along_axis(cand, idx[:, :, None], 2)[:, :, 0] * np.where(x < 0, -1, 1)
    assert np.array_equal(dec, ref)


def test_clamped_exponents():
    # A table whose top level is 0.5 cannot reach a 3e38 block with e <= 127:
    # the exponent clamps to 127 and every weight saturates to the top level.
    small = np.array([0.015625, 0.03125, 0.0625, 0.125, 0.1875, 0.25, 0.375, 0.5], np.float32)
    big = helpers.f32_to_bf16_bits(np.full(32, 3.0e38, np.float32))
    w, s = oracle.pack(big[None, None], small[None], np.zeros(1, np.uint8), 1, 1, 32)
    assert int(s[0, 0, 0]) == 254
    assert all(b == 0x77 for b in w[0, 0])
    # A block of bf16 subnormals needs e < -127: clamps to -127 (scale byte 0).
    grid = inputs.lloyd_max_grid(0)
    tiny = helpers.f32_to_bf16_bits(np.full(32, 1e-39, np.float32))
    w, s = oracle.pack(tiny[None, None], grid[None], np.zeros(1, np.uint8), 1, 1, 32)
    assert int(s[0, 0, 0]) == 0
    assert _brute_exponent(1e-39, grid.max()) == -127


def test_pack_rejects_non_finite_and_bad_shapes():
    grid = inputs.lloyd_max_grid(0)[None]
    bits = helpers.f32_to_bf16_bits(np.ones(32, np.float32))
    bad = bits.copy()
    bad[7] = 0x7FC0  # NaN
    with pytest.raises(oracle.OracleError):
        oracle.pack(bad[None, None], grid, np.zeros(1, np.uint8), 1, 1, 32)
    bad[7] = 0x7F80  # +Inf
    with pytest.raises(oracle.OracleError):
        oracle.pack(bad[None, None], grid, np.zeros(1, np.uint8), 1, 1, 32)
    with pytest.raises(oracle.OracleError):
        oracle.pack(np.zeros((1, 1, 48), np.uint16), grid, np.zeros(1, np.uint8), 1, 1, 48)


def test_gaussian_block_statistics_are_near_the_pages_anchors():
    # Loose anchors, not pins: the page reports a crest factor of 2.366 for its
    # routed-expert weights ("What this is") and relative RMS error 10.80%
    # (Lloyd) vs 12.18% (E2M1) after GPTQ ("Known defect").  RTN on synthetic
    # Gaussian weights lands near those.
    w = inputs.Workload("t", 0, 1, inputs.TINY)
    wt = torch.cat([inputs.expert_weight(w, e, "gate").float() for e in range(8)])
    x = wt.numpy().astype(np.float64)
    blocks = x.reshape(-1, 32)
    crest = np.mean(np.max(np.abs(blocks), 1) / np.sqrt(np.mean(blocks ** 2, 1)))
    assert 2.2 < crest < 2.55
    N, K = x.shape
    errs = {}
    for name, t in (("lloyd", inputs.lloyd_max_grid(0)), ("e2m1", inputs.E2M1_TABLE)):
        c, s = oracle.pack(inputs.bf16_bits(wt.to(torch.bfloat16))[None], t[None], np.zeros(1, np.uint8), 1, N, K)
        d = oracle.decode_matrix_f64(c[0], s[0], t, N, K)
        errs[name] = np.linalg.norm(d - x) / np.linalg.norm(x)
    assert 0.08 < errs["lloyd"] < 0.14
    assert 0.08 < errs["e2m1"] < 0.15
