"""Pins for the oracle's decode ("aidendle94/GLM-5.2-NF4-Lloyd-Experts-GPTQ",
"Codes are indices into the per-layer grid -- not E2M1" and "Contents")."""
import numpy as np
import pytest
import torch

import oracle
from bit_codebook_quantized_router_b200 import inputs
from tests import helpers


def test_hand_decodes_all_codes_and_edge_scales():
    tables, rows, _ = helpers.read_decode_golden()
    n = 0
    for name, scale, pos in rows:
        for code in range(16):
            exp = pos[code & 7] ^ (0x8000 if code & 8 else 0)
            got = oracle.decode_bf16(code, scale, tables[name])
            assert got == exp, (name, scale, code, hex(got), hex(exp))
            n += 1
    assert n >= 16 * 12


def test_hand_nibble_order_through_dequant():
    tables, _, nib = helpers.read_decode_golden()
    for name, scale, row, exp in nib:
        K = 32
        w = np.zeros((1, 1, K // 2), np.uint8)
        w[0, 0, : len(row)] = np.frombuffer(row, np.uint8)
        s = np.full((1, 1, 1), scale, np.uint8)
        out = oracle.dequant(w, s, tables[name][None], np.zeros(1, np.uint8), 1, 1, K)
        assert [int(v) for v in out[0, 0, : len(exp)]] == exp


def test_nibble_order_both_positions_every_code():
    # byte b holds K=2i (low nibble) and K=2i+1 (high nibble): put code c in
    # one half and the "other" code in the other half, decode both positions.
    table = inputs.E2M1_TABLE
    for c in range(16):
        other = (c + 5) & 15
        w = np.zeros((1, 1, 16), np.uint8)
        w[0, 0, 0] = c | (other << 4)     # K0 = c, K1 = other
        w[0, 0, 1] = other | (c << 4)     # K2 = other, K3 = c
        s = np.full((1, 1, 1), 127, np.uint8)
        out = oracle.dequant(w, s, table[None], np.zeros(1, np.uint8), 1, 1, 32)[0, 0]
        ref_c = oracle.decode_bf16(c, 127, table)
        ref_o = oracle.decode_bf16(other, 127, table)
        assert (out[0], out[1], out[2], out[3]) == (ref_c, ref_o, ref_o, ref_c)


def _e2m1_closed_form(code):
    # OCP MX E2M1 bit decode: s = bit 3, e = bits 2..1, m = bit 0;
    # value = (-1)^s * (m / 2 if e == 0 else (1 + m / 2) * 2^(e - 1)).
    s, e, m = (code >> 3) & 1, (code >> 1) & 3, code & 1
    v = m / 2.0 if e == 0 else (1.0 + m / 2.0) * 2.0 ** (e - 1)
    return -v if s else v


def test_e2m1_table_matches_closed_form_for_all_codes_and_scales():
    # The second table must decode exactly like the E2M1 bit layout
    # ("Serving": the nibble bytes are byte-identical to the E2M1 layout).
    table = inputs.E2M1_TABLE
    for scale in list(range(1, 255)):
        for code in range(16):
            bits = oracle.decode_bf16(code, scale, table)
            got = helpers.bf16_bits_to_f32([bits])[0]
            ref = _e2m1_closed_form(code) * 2.0 ** (scale - 127)
            if abs(ref) > 3.3895313892515355e38:  # beyond bf16/fp32 max -> inf
                assert np.isinf(got) and np.sign(got) == np.sign(ref)
            else:
                assert got == ref, (code, scale)
                assert np.signbit(got) == bool(code & 8)


def test_normal_range_equals_rounded_level_times_power_of_two():
    # In the normal range, fp32(level * 2^e) is exact, so the decode must equal
    # the library's RNE cast of the level to bf16, scaled by 2^e.
    grid = inputs.lloyd_max_grid(0)
    lv_bits = helpers.f32_to_bf16_bits(grid)
    lv = helpers.bf16_bits_to_f32(lv_bits).astype(np.float64)
    for scale in range(3, 253):
        for code in range(16):
            got = helpers.bf16_bits_to_f32([oracle.decode_bf16(code, scale, grid)])[0]
            ref = lv[code & 7] * 2.0 ** (scale - 127) * (-1 if code & 8 else 1)
            assert got == ref


def test_decode_matrix_f64_is_exact_level_times_scale():
    rng = np.random.default_rng(5)
    grid = inputs.lloyd_max_grid(0)
    N, K = 4, 64
    w = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    s = rng.integers(100, 140, (N, K // 32), dtype=np.uint8)
    out = oracle.decode_matrix_f64(w, s, grid, N, K)
    for n in range(N):
        for k in range(K):
            byte = int(w[n, k // 2])
            c = byte & 15 if k % 2 == 0 else byte >> 4
            ref = float(grid[c & 7]) * 2.0 ** (int(s[n, k // 32]) - 127)
            assert out[n, k] == (-ref if c & 8 else ref)


def test_dequant_rejects_bad_arguments():
    grid = inputs.lloyd_max_grid(0)[None]
    w = np.zeros((1, 1, 16), np.uint8)
    s = np.zeros((1, 1, 1), np.uint8)
    with pytest.raises(oracle.OracleError):
        oracle.dequant(w, s, grid, np.array([1], np.uint8), 1, 1, 32)  # table id out of range
    bad = grid.copy()
    bad[0, 3] = np.nan
    with pytest.raises(oracle.OracleError):
        oracle.dequant(w, s, bad, np.zeros(1, np.uint8), 1, 1, 32)
    neg = grid.copy()
    neg[0, 0] = -0.5
    with pytest.raises(oracle.OracleError):
        oracle.dequant(w, s, neg, np.zeros(1, np.uint8), 1, 1, 32)
    negz = grid.copy()
    negz[0, 0] = -0.0
    with pytest.raises(oracle.OracleError):
        oracle.dequant(w, s, negz, np.zeros(1, np.uint8), 1, 1, 32)


def test_wrong_table_decode_is_large_error():
    # "Known defect": E2M1-packed bytes decoded against the Lloyd grid give a
    # real weight error (the page measured 10.5% on its grid).  With this
    # synthetic grid the error must be large and detectable.
    w = inputs.Workload("t", 0, 1, inputs.TINY)
    wt = inputs.expert_weight(w, 0, "gate")
    N, K = wt.shape
    e2m1 = inputs.E2M1_TABLE[None]
    grid = inputs.lloyd_max_grid(0)[None]
    codes, scales = oracle.pack(inputs.bf16_bits(wt)[None], e2m1, np.zeros(1, np.uint8), 1, N, K)
    right = oracle.decode_matrix_f64(codes[0], scales[0], e2m1[0], N, K)
    wrong = oracle.decode_matrix_f64(codes[0], scales[0], grid[0], N, K)
    ref = wt.float().numpy().astype(np.float64)
    rel_right = np.linalg.norm(right - ref) / np.linalg.norm(ref)
    rel_wrong = np.linalg.norm(wrong - ref) / np.linalg.norm(ref)
    assert rel_right < 0.16
    assert rel_wrong > 0.25
