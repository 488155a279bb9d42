"""GPU parity: moe_q4_pack and moe_q4_dequant against the oracle, bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import bit_codebook_quantized_router_b200 as q4
from bit_codebook_quantized_router_b200 import inputs
from tests import gpu_support, helpers

pytestmark = pytest.mark.gpu

HAND = np.array([0.125, 0.375, 0.625, 0.875, 1.25, 1.625, 2.0625, 2.75], np.float32)
RNE = np.array([1.00390625, 1.01171875, 1.0039063692092896, 255.5, 0.1, 3.0, 0.0, 1.0], np.float32)
TINY_LEVELS = np.array([1e-45, 3e-39, 1e-38, 0.5, 1.0, 2.0, 3.0e38, 0.0], np.float32)


def _tables():
    return np.stack([inputs.lloyd_max_grid(0), inputs.E2M1_TABLE, HAND, RNE, TINY_LEVELS])


def _rand_bf16(rng, E, N, K, spread=20):
    x = rng.standard_normal((E, N, K)) * 0.02
    x *= 2.0 ** rng.integers(-spread, spread, (E, N, K // 32, 1)).repeat(32, -1).reshape(E, N, K)
    x[rng.random(x.shape) < 0.03] = 0.0
    bits = helpers.f32_to_bf16_bits(x.astype(np.float32))
    bits[rng.random(bits.shape) < 0.01] = 0x8000  # -0.0
    return bits


@pytest.mark.parametrize("E,N,K", [(1, 1, 32), (3, 5, 64), (5, 17, 96), (2, 64, 2048)])
def test_pack_bit_exact(E, N, K):
    rng = np.random.default_rng(E * 100 + N)
    tables = _tables()[:4]
    tid = rng.integers(0, tables.shape[0], E).astype(np.uint8)
    bits = _rand_bf16(rng, E, N, K)
    ref_w, ref_s = oracle.pack(bits, tables, tid, E, N, K)
    wt = inputs.bits_to_bf16(bits).cuda()
    codes, scales = q4.pack(wt, tables, tid)
    assert np.array_equal(scales.cpu().numpy(), ref_s)
    assert np.array_equal(codes.cpu().numpy(), ref_w)


def test_pack_hand_blocks():
    for name, scale, packed, values in helpers.read_pack_golden():
        t = {"E2M1": inputs.E2M1_TABLE, "HAND": HAND}[name]
        bits = helpers.f32_to_bf16_bits(values)
        codes, scales = q4.pack(inputs.bits_to_bf16(bits).reshape(1, 1, 32).cuda(), t[None], [0])
        assert int(scales.item()) == scale
        assert bytes(codes.cpu().numpy().reshape(-1)) == packed


def test_pack_flags_non_finite():
    bits = np.full((1, 2, 32), 0x3F80, np.uint16)
    bits[0, 1, 5] = 0x7FC0
    with pytest.raises(q4.MoeQ4Error) as ei:
        q4.pack(inputs.bits_to_bf16(bits).cuda(), inputs.lloyd_max_grid(0)[None], [0])
    assert ei.value.status == q4._lib.EDEVICE


@pytest.mark.parametrize("table_index", range(5))
def test_dequant_bit_exact_every_scale_byte(table_index):
    rng = np.random.default_rng(7 + table_index)
    E, N, K = 2, 256, 64
    tables = _tables()
    tid = np.full(E, table_index, np.uint8)
    codes = rng.integers(0, 256, (E, N, K // 2), dtype=np.uint8)
    scales = np.empty((E, N, K // 32), np.uint8)
    scales.reshape(-1)[:] = np.arange(scales.size) % 256  # every scale byte, 0..255
    ref = oracle.dequant(codes, scales, tables, tid, E, N, K)
    out = gpu_support.Guarded((E, N, K), torch.bfloat16)  # canary bands around the output
    got = q4.dequant(torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda(), tables, tid, out=out.view)
    torch.cuda.synchronize()
    out.check("dequant output")
    got_bits = inputs.bf16_bits(got)
    bad = np.nonzero(got_bits != ref)
    assert bad[0].size == 0, (bad[0][:5], got_bits[bad][:5], ref[bad][:5])


def test_dequant_hand_nibbles():
    tables, _, nib = helpers.read_decode_golden()
    for name, scale, row, exp in nib:
        w = np.zeros((1, 1, 16), np.uint8)
        w[0, 0, : len(row)] = np.frombuffer(row, np.uint8)
        s = np.full((1, 1, 1), scale, np.uint8)
        got = q4.dequant(torch.from_numpy(w).cuda(), torch.from_numpy(s).cuda(), tables[name][None], [0])
        assert [int(v) for v in inputs.bf16_bits(got)[0, 0, : len(exp)]] == exp


def test_glm_layer_pack_and_dequant_sampled_experts():
    # Full GLM-shaped layer with the mixed tables: GPU pack of every expert;
    # bit-exact against the oracle on a seeded sample of experts that includes
    # an E2M1 expert; dequant of those experts bit-exact too.
    w = inputs.WORKLOADS["prefill_t8192"]
    dev = gpu_support.device_layer(w)
    sample = [0, 15, 101, 255]
    oracle_L = gpu_support.oracle_layer(w, sample, dev)  # asserts pack bytes equal
    tables, tid = inputs.layer_tables(w)
    for e in sample:
        for proj, (cw, cs) in (("gate", (dev.gate_w, dev.gate_s)), ("down", (dev.down_w, dev.down_s))):
            N, K = inputs.proj_shape(w.shape, proj)
            got = q4.dequant(cw[e:e + 1], cs[e:e + 1], tables, tid[e:e + 1])
            ow = getattr(oracle_L, proj + "_w")[e]
            os_ = getattr(oracle_L, proj + "_s")[e]
            ref = oracle.dequant(ow[None], os_[None], tables, tid[e:e + 1], 1, N, K)
            assert np.array_equal(inputs.bf16_bits(got), ref)
