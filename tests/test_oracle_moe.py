"""Pins for the oracle's MoE layer: library matmuls on the tiny workload,
reductions to a dense SwiGLU FFN, zero input, and the intermediate-channel
permutation invariant ("Round 7 -- Rewrite the GLM-5.2 routed-expert
encoder", "Owner-locked decisions" item 7: permutations of the intermediate
channels applied consistently to gate-N, up-N and down-K are exact at serve)."""
import numpy as np
import pytest
import scipy.special

import oracle
from bit_codebook_quantized_router_b200 import inputs
from tests import helpers

TINY = inputs.WORKLOADS["tiny"]


def _dense_ffn(Wg, Wu, Wd, x):
    g = Wg @ x
    u = Wu @ x
    h = g * scipy.special.expit(g) * u
    return Wd @ h


def _expert_mats(L, e):
    t = L.tables[L.table_id[e]]
    H, I = L.H, L.I
    return (oracle.decode_matrix_f64(L.gate_w[e], L.gate_s[e], t, I, H),
            oracle.decode_matrix_f64(L.up_w[e], L.up_s[e], t, I, H),
            oracle.decode_matrix_f64(L.down_w[e], L.down_s[e], t, H, I))


@pytest.fixture(scope="module")
def tiny_layer():
    L, packed, raw = helpers.build_layer_host(TINY)
    return L, packed


def test_tiny_against_library_matmul_and_sort(tiny_layer):
    L, _ = tiny_layer
    x = inputs.bf16_bits(inputs.activations(TINY))
    lg = inputs.router_logits(TINY).numpy()
    out = oracle.moe_tokens(L, x, lg, TINY.shape.k)
    xf = helpers.bf16_bits_to_f32(x).astype(np.float64)
    mats = {e: _expert_mats(L, e) for e in range(TINY.shape.E)}
    for t in range(TINY.T):
        order = np.lexsort((np.arange(TINY.shape.E), -lg[t].astype(np.float64)))[: TINY.shape.k]
        w = scipy.special.softmax(lg[t, order].astype(np.float64))
        ref = sum(w[j] * _dense_ffn(*mats[e], xf[t]) for j, e in enumerate(order))
        np.testing.assert_allclose(out[t], ref, rtol=1e-12, atol=1e-14 * np.abs(ref).max())


def test_top1_reduces_to_dense_ffn(tiny_layer):
    L, _ = tiny_layer
    rng = np.random.default_rng(9)
    xf = rng.standard_normal((6, L.H)).astype(np.float32)
    x = helpers.f32_to_bf16_bits(xf)
    lg = rng.standard_normal((6, L.E)).astype(np.float32)
    out, ids, w = oracle.moe_tokens(L, x, lg, 1, return_routing=True)
    assert np.all(w == 1.0)
    xd = helpers.bf16_bits_to_f32(x).astype(np.float64)
    for t in range(6):
        ref = _dense_ffn(*_expert_mats(L, ids[t, 0]), xd[t])
        np.testing.assert_allclose(out[t], ref, rtol=1e-12, atol=1e-14 * np.abs(ref).max())


def test_identical_experts_equal_dense_ffn_for_any_routing():
    L, _, _ = helpers.build_layer_host(TINY, identical_to=3)
    rng = np.random.default_rng(10)
    x = helpers.f32_to_bf16_bits(rng.standard_normal((5, L.H)).astype(np.float32))
    lg = rng.standard_normal((5, L.E)).astype(np.float32)
    xd = helpers.bf16_bits_to_f32(x).astype(np.float64)
    mats = _expert_mats(L, 3)
    for k in (1, 2, 5, 8):
        out = oracle.moe_tokens(L, x, lg, k)
        for t in range(5):
            ref = _dense_ffn(*mats, xd[t])
            np.testing.assert_allclose(out[t], ref, rtol=1e-12, atol=1e-13 * np.abs(ref).max())


def test_zero_activations_give_zero_output(tiny_layer):
    L, _ = tiny_layer
    x = np.zeros((3, L.H), np.uint16)
    lg = np.random.default_rng(1).standard_normal((3, L.E)).astype(np.float32)
    assert np.all(oracle.moe_tokens(L, x, lg, 2) == 0.0)


def _unpack(codes_bytes):
    lo = codes_bytes & 0x0F
    hi = codes_bytes >> 4
    out = np.empty(codes_bytes.shape[:-1] + (codes_bytes.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = lo  # low nibble = even K
    out[..., 1::2] = hi
    return out


def _repack(codes):
    return (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)


def test_intermediate_permutation_invariant(tiny_layer):
    L, packed = tiny_layer
    I, H = L.I, L.H
    rng = np.random.default_rng(12)
    nb = I // 32
    sigma = rng.permutation(nb)
    taus = [rng.permutation(32) for _ in range(nb)]
    # pi(32 b' + q') = 32 sigma(b') + tau_b'(q'): whole 32-blocks move with their
    # scale byte, codes move inside a block, so nothing is re-quantised.
    pi = np.concatenate([32 * sigma[b] + taus[b] for b in range(nb)])
    blk = sigma
    L2 = oracle.Layer(L.E, H, I, L.tables, L.table_id)
    for e, p in packed.items():
        gw, gs = p["gate"]
        uw, us = p["up"]
        dw, ds = p["down"]
        dcodes = _unpack(dw)[:, pi]
        L2.set_expert(e, gw[pi], gs[pi], uw[pi], us[pi], _repack(dcodes), ds[:, blk])
    x = inputs.bf16_bits(inputs.activations(TINY))
    lg = inputs.router_logits(TINY).numpy()
    a = oracle.moe_tokens(L, x, lg, 2)
    b = oracle.moe_tokens(L2, x, lg, 2)
    np.testing.assert_allclose(b, a, rtol=1e-12, atol=1e-13 * np.abs(a).max())
    # and a permutation that breaks a block (moves single codes between blocks
    # without moving their scales) must change the output: the invariant is
    # sensitive to the scale indexing.
    bad = pi.copy()
    bad[[0, 40]] = bad[[40, 0]]
    L3 = oracle.Layer(L.E, H, I, L.tables, L.table_id)
    for e, p in packed.items():
        gw, gs = p["gate"]
        uw, us = p["up"]
        dw, ds = p["down"]
        L3.set_expert(e, gw[bad], gs[bad], uw[bad], us[bad], _repack(_unpack(dw)[:, bad]), ds[:, blk])
    c = oracle.moe_tokens(L3, x, lg, 2)
    assert np.abs(c - a).max() > 1e-6 * np.abs(a).max()


def test_per_expert_table_id_selects_the_table():
    w = inputs.Workload("mixed", 0, 4, inputs.TINY, mixed_tables=True)
    tables, tid = inputs.layer_tables(w)
    tid = tid.copy()
    tid[5] = 1  # expert 5 decodes with E2M1
    L = oracle.Layer(8, w.shape.H, w.shape.I, tables, tid)
    for e in range(8):
        p = {}
        for proj in inputs.PROJECTIONS:
            N, K = inputs.proj_shape(w.shape, proj)
            wt = inputs.expert_weight(w, e, proj)
            c, s = oracle.pack(inputs.bf16_bits(wt)[None], tables, tid[e:e + 1], 1, N, K)
            p[proj] = (c[0], s[0])
        L.set_expert(e, *p["gate"], *p["up"], *p["down"])
    lg = np.full((1, 8), -5.0, np.float32)
    lg[0, 5] = 5.0
    x = inputs.bf16_bits(inputs.activations(w, T=1))
    out = oracle.moe_tokens(L, x, lg, 1)
    xd = helpers.bf16_bits_to_f32(x).astype(np.float64)[0]
    ref = _dense_ffn(*_expert_mats(L, 5), xd)
    np.testing.assert_allclose(out[0], ref, rtol=1e-12, atol=1e-14 * np.abs(ref).max())
    # decoding the same bytes with the Lloyd grid gives something else
    L.table_id[5] = 0
    wrong = _dense_ffn(*_expert_mats(L, 5), xd)
    assert np.linalg.norm(wrong - ref) > 0.1 * np.linalg.norm(ref)


def test_missing_expert_is_an_error(tiny_layer):
    L, packed = tiny_layer
    L2 = oracle.Layer(L.E, L.H, L.I, L.tables, L.table_id)
    p = packed[0]
    L2.set_expert(0, *p["gate"], *p["up"], *p["down"])
    lg = np.zeros((1, L.E), np.float32)
    lg[0, 1] = 1.0
    with pytest.raises(oracle.OracleError):
        oracle.moe_tokens(L2, np.zeros((1, L.H), np.uint16), lg, 1)


def test_expert_partials_sum_to_the_layer(tiny_layer):
    # Partials over a partition of the intermediate channels, weighted by the
    # routing weights, reproduce the layer output.
    L, _ = tiny_layer
    x = inputs.bf16_bits(inputs.activations(TINY))
    lg = inputs.router_logits(TINY).numpy()
    out, ids, w = oracle.moe_tokens(L, x, lg, 2, return_routing=True)
    for t in range(TINY.T):
        acc = np.zeros(L.H)
        for j in range(2):
            for i0, i1 in ((0, 40), (40, 41), (41, 128)):
                acc += w[t, j] * oracle.expert_partial(L, int(ids[t, j]), x[t], i0, i1)
        np.testing.assert_allclose(acc, out[t], rtol=1e-12, atol=1e-14 * np.abs(out[t]).max())
