"""Pins of the oracle's router logits (logits[t][e] = sum_h x[t][h] w[e][h]
in fp64 over bf16 inputs), checked against values the mathematics fixes:
exact integer dot products done in Python integers, one-hot hidden states
that select one gate column, and exact power-of-two scaling."""
import numpy as np
import torch

import oracle
from bit_codebook_quantized_router_b200 import inputs


def _bf16(a):
    """bf16 bit patterns (round to nearest even) of the float array a."""
    return inputs.bf16_bits(torch.tensor(np.asarray(a, np.float32)).to(torch.bfloat16))


def _f32(bits):
    return inputs.bits_to_bf16(bits).float().numpy()


def test_integer_inputs_match_python_integer_dot_products():
    rng = np.random.default_rng(11)
    T, H, E = 5, 96, 7
    xi = rng.integers(-16, 17, (T, H))
    wi = rng.integers(-16, 17, (E, H))
    logits, absdot = oracle.router_logits(_bf16(xi), _bf16(wi))
    for t in range(T):
        for e in range(E):
            exact = sum(int(xi[t, h]) * int(wi[e, h]) for h in range(H))
            mag = sum(abs(int(xi[t, h]) * int(wi[e, h])) for h in range(H))
            assert logits[t, e] == exact, (t, e)
            assert absdot[t, e] == mag, (t, e)


def test_one_hot_hidden_state_selects_a_gate_column():
    rng = np.random.default_rng(12)
    H, E = 64, 9
    w = _bf16(rng.normal(0.0, 0.02, (E, H)))
    for h in (0, 17, H - 1):
        x = np.zeros((1, H), np.float32)
        x[0, h] = 1.0
        logits, _ = oracle.router_logits(_bf16(x), w)
        col = _f32(w[:, h]).astype(np.float64)
        assert np.array_equal(logits[0], col)


def test_power_of_two_scaling_is_exact():
    rng = np.random.default_rng(13)
    x = _bf16(rng.normal(0.0, 1.0, (3, 128)))
    w = _bf16(rng.normal(0.0, 0.02, (4, 128)))
    base, _ = oracle.router_logits(x, w)
    x4 = _bf16(_f32(x) * 4.0)
    scaled, _ = oracle.router_logits(x4, w)
    assert np.array_equal(scaled, 4.0 * base)
