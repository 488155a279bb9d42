"""Pins of the oracle's shared expert (oq_shared_ffn): the BF16 shared-expert
MLP with gate and up merged into one [2 I][H] payload ("GLM-5.2 EXL3 TR3 v4"
README, "Checkpoint layout update"; HF discussion #2).

- a shared expert whose BF16 weights are a routed expert's decoded weights
  gives exactly that expert's output under the routed oracle with top-1
  routing (weight 1), which the routed oracle's own pins hold;
- permuting the intermediate channels consistently in the gate half, the up
  half and the down columns changes nothing ("Round 7", "Owner-locked
  decisions" item 7);
- the merged layout's order matters: swapping the gate and up halves changes
  the output (silu is not symmetric);
- zero activations give zero."""
import numpy as np
import pytest

import oracle
from bit_codebook_quantized_router_b200 import inputs
from tests import helpers

# a grid of bf16-exact levels: decoded weights are exact in bf16, so the
# routed oracle (exact fp64 weights) and the shared expert (bf16 weights) see
# the same numbers
BF16_EXACT = np.array([0.125, 0.375, 0.625, 0.875, 1.25, 1.625, 2.0, 2.75], np.float32)


def _layer(seed=21, E=4, H=128, I=64):
    w = inputs.Workload("shared_pin", seed, 6, inputs.Shape(H=H, I=I, E=E, k=1))
    L = oracle.Layer(E, H, I, BF16_EXACT[None], np.zeros(E, np.uint8))
    for e in range(E):
        parts = []
        for proj in inputs.PROJECTIONS:
            N, K = inputs.proj_shape(w.shape, proj)
            c, s = oracle.pack(inputs.bf16_bits(inputs.expert_weight(w, e, proj))[None], BF16_EXACT[None],
                               np.zeros(1, np.uint8), 1, N, K)
            parts += [c[0], s[0]]
        L.set_expert(e, *parts)
    return w, L


def _decoded_bits(L, e, proj, N, K):
    c, s = {"gate": (L.gate_w, L.gate_s), "up": (L.up_w, L.up_s), "down": (L.down_w, L.down_s)}[proj]
    return oracle.dequant(c[e][None], s[e][None], BF16_EXACT[None], np.zeros(1, np.uint8), 1, N, K)[0]


def test_equals_a_routed_expert_with_top1_routing():
    w, L = _layer()
    H, I, E = L.H, L.I, L.E
    e = 2
    wgu = np.concatenate([_decoded_bits(L, e, "gate", I, H), _decoded_bits(L, e, "up", I, H)])
    wd = _decoded_bits(L, e, "down", H, I)
    x = inputs.bf16_bits(inputs.activations(w))
    lg = np.zeros((w.T, E), np.float32)
    lg[:, e] = 5.0  # every token's top-1 is expert e, weight 1
    routed = oracle.moe_tokens(L, x, lg, 1)
    shared = oracle.shared_ffn(x, wgu, wd)
    np.testing.assert_allclose(shared, routed, rtol=1e-12, atol=1e-13 * np.abs(routed).max())


def _random_shared(rng, H, I):
    def bits(shape, s):
        return helpers.f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32) * s)
    return bits((2 * I, H), 0.05), bits((H, I), 0.05)


def test_intermediate_permutation_changes_nothing():
    rng = np.random.default_rng(4)
    H, I = 96, 64
    wgu, wd = _random_shared(rng, H, I)
    x = helpers.f32_to_bf16_bits(rng.standard_normal((5, H)).astype(np.float32))
    p = rng.permutation(I)
    wgu_p = np.concatenate([wgu[:I][p], wgu[I:][p]])
    wd_p = wd[:, p]
    a = oracle.shared_ffn(x, wgu, wd)
    b = oracle.shared_ffn(x, wgu_p, wd_p)
    np.testing.assert_allclose(b, a, rtol=1e-12, atol=1e-13 * np.abs(a).max())


def test_gate_half_comes_first():
    rng = np.random.default_rng(5)
    H, I = 64, 32
    wgu, wd = _random_shared(rng, H, I)
    x = helpers.f32_to_bf16_bits(rng.standard_normal((3, H)).astype(np.float32) * 4)
    a = oracle.shared_ffn(x, wgu, wd)
    b = oracle.shared_ffn(x, np.concatenate([wgu[I:], wgu[:I]]), wd)
    assert np.abs(a - b).max() > 1e-2 * np.abs(a).max()


def test_zero_activations_give_zero():
    rng = np.random.default_rng(6)
    wgu, wd = _random_shared(rng, 64, 32)
    out = oracle.shared_ffn(np.zeros((2, 64), np.uint16), wgu, wd)
    assert np.all(out == 0.0)


def test_shapes_are_checked():
    rng = np.random.default_rng(7)
    wgu, wd = _random_shared(rng, 64, 32)
    with pytest.raises(oracle.OracleError):
        oracle.shared_ffn(np.zeros((2, 64), np.uint16), wgu[:-1], wd)
