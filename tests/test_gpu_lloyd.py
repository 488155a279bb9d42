"""GPU parity of the weighted Lloyd-Max grid fit (moe_q4_lloyd_hist +
moe_q4_lloyd_solve through the C ABI) against the fp64 oracle oq_lloyd_fit
("aidendle94/GLM-5.2-NF4-Lloyd-Experts-GPTQ", "What this is").

The fitted levels are compared bit for bit after rounding to fp32, and the
step counts must be equal: both sides take every nearest-level decision in
fp64 on the same exact ratios, and their per-level sums differ at most in the
last bits of fp64 (the sums of powers of four are exact; the weighted ratio
sums are added in another order), far below fp32's rounding."""
import numpy as np
import pytest
import torch

import oracle
import bit_codebook_quantized_router_b200 as q4
from bit_codebook_quantized_router_b200 import _lib, inputs

pytestmark = pytest.mark.gpu

E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], np.float32)


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16)


def _fit_both(w_bf16_list, grid0, max_iter, tol):
    g, it, st = q4.lloyd_fit([w.cuda() for w in w_bf16_list], grid0, max_iter=max_iter, tol=tol)
    torch.cuda.synchronize()
    assert st == _lib.OK, q4.status_string(st)
    bits = np.concatenate([inputs.bf16_bits(w).reshape(-1) for w in w_bf16_list])
    rg, rit = oracle.lloyd_fit(bits, np.asarray(grid0, np.float32), max_iter=max_iter, tol=tol)
    return g.cpu().numpy(), int(it.item()), rg, rit


def _assert_same(g, it, rg, rit):
    assert it == rit, (it, rit)
    assert np.array_equal(g.view(np.uint32), rg.view(np.uint32)), (g, rg)


def test_uniform_data_to_convergence():
    rng = np.random.default_rng(7)
    w = _bf16(rng.uniform(-1.0, 1.0, 1 << 18))
    opt = (2 * np.arange(8) + 1) / 16
    grid0 = (opt + 0.01 * (-1.0) ** np.arange(8)).astype(np.float32)
    grid0[7] = 1.0
    _assert_same(*_fit_both([w], grid0, 5000, 0.0))


def test_one_step_of_two_blocks():
    w = _bf16(np.concatenate([np.full(32, 0.75), np.full(32, -7.0 / 32.0)]))
    grid0 = np.array([0.05, 0.1, 0.15, 0.2, 0.25, 0.3, 0.35, 1.0], np.float32)
    g, it, rg, rit = _fit_both([w], grid0, 1, 0.0)
    _assert_same(g, it, rg, rit)
    assert g[7] == np.float32(25.75 / 34.0)


@pytest.mark.parametrize("table", ["lloyd", "e2m1"])
def test_gaussian_weights(table):
    rng = np.random.default_rng(5)
    w = _bf16(rng.standard_normal(1 << 20) * 0.02)
    grid0 = inputs.lloyd_max_grid() if table == "lloyd" else E2M1
    _assert_same(*_fit_both([w], grid0, 300, 1e-12))


def test_pooled_arrays_equal_their_concatenation():
    rng = np.random.default_rng(9)
    parts = [_bf16(rng.standard_normal(n) * s) for n, s in ((32 * 1000, 0.02), (32 * 37, 0.5), (32 * 4096, 0.003))]
    _assert_same(*_fit_both(parts, inputs.lloyd_max_grid(), 200, 1e-12))


def test_glm_expert_projection():
    # one expert's gate projection of the GLM-shaped layer ([2048, 6144] bf16)
    w = inputs.WORKLOADS["decode_t1"]
    x = inputs.expert_weight(w, 3, "gate", device="cuda").cpu()
    _assert_same(*_fit_both([x], inputs.lloyd_max_grid(), 20, 0.0))


def test_no_blocks_keep_the_starting_grid():
    grid0 = inputs.lloyd_max_grid()
    g, it, st = q4.lloyd_fit(torch.empty(0, dtype=torch.bfloat16, device="cuda"), grid0, max_iter=10)
    assert st == _lib.OK
    rg, rit = oracle.lloyd_fit(np.zeros(0, np.uint16), grid0, max_iter=10)
    _assert_same(g.cpu().numpy(), int(it.item()), rg, rit)
    assert np.array_equal(g.cpu().numpy(), np.asarray(grid0, np.float32))


def test_repeat_is_bit_identical():
    rng = np.random.default_rng(13)
    w = _bf16(rng.standard_normal(1 << 19) * 0.05).cuda()
    a = q4.lloyd_fit(w, inputs.lloyd_max_grid(), max_iter=100)
    b = q4.lloyd_fit(w, inputs.lloyd_max_grid(), max_iter=100)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_non_finite_weight_reports_device_status():
    w = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    w[5] = float("nan")
    _, _, st = q4.lloyd_fit(w, inputs.lloyd_max_grid(), max_iter=3)
    assert st == _lib.EDEVICE
