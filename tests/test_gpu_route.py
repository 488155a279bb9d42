"""GPU parity: routing (top-k ids bit-exact, softmax weights to 1e-6) and
expert grouping (counts, offsets, row order, inverse map: bit-exact)."""
import numpy as np
import pytest
import torch

import oracle
import bit_codebook_quantized_router_b200 as q4
from bit_codebook_quantized_router_b200 import inputs

pytestmark = pytest.mark.gpu


def _check(lg, k):
    T, E = lg.shape
    ids, w, counts, offsets, row_token, inv, st = q4.route(torch.from_numpy(lg).cuda(), k)
    assert st == 0
    rids, rw = oracle.route(lg, k)
    rc, ro, rrt, rinv = oracle.group(rids, E)
    assert np.array_equal(ids.cpu().numpy(), rids)
    np.testing.assert_allclose(w.cpu().numpy(), rw, rtol=1e-6, atol=1e-7)
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(row_token.cpu().numpy(), rrt)
    assert np.array_equal(inv.cpu().numpy(), rinv)


@pytest.mark.parametrize("T", [1, 4, 8, 64, 255, 256, 257, 1000, 1025, 2048, 8192])
def test_route_glm_shapes(T):
    rng = np.random.default_rng(T)
    _check(rng.standard_normal((T, 256)).astype(np.float32), 8)


@pytest.mark.parametrize("E,k", [(8, 1), (8, 2), (3, 3), (512, 16), (33, 5), (1, 1)])
def test_route_other_shapes(E, k):
    rng = np.random.default_rng(E * 7 + k)
    for T in (1, 37, 300, 1500):
        _check(rng.standard_normal((T, E)).astype(np.float32), k)


@pytest.mark.parametrize("T,E,k", [(65536, 256, 8), (40001, 512, 16)])
def test_route_many_chunks(T, E, k):
    # hundreds of 256-token chunks (the last one ragged) in the large-batch
    # grouping, with a skew so that some experts hold rows in every chunk
    rng = np.random.default_rng(T + E)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    lg[:, : E // 16] += 1.5
    _check(lg, k)


def test_route_ties_and_signed_zeros():
    rng = np.random.default_rng(3)
    lg = (np.round(rng.standard_normal((500, 64)) * 2) / 2).astype(np.float32)  # many exact ties
    lg[0, :] = 0.0
    lg[0, ::3] = -0.0
    _check(lg, 8)


def test_route_zipf_workloads():
    for name in ("prefill_t2048", "prefill_t8192"):
        w = inputs.WORKLOADS[name]
        _check(inputs.router_logits(w).numpy(), 8)


def test_route_all_tokens_on_one_expert():
    lg = np.random.default_rng(4).standard_normal((300, 16)).astype(np.float32)
    lg[:, 5] += 100.0
    _check(lg, 2)


@pytest.mark.parametrize("T", [5, 600])
def test_route_non_finite_logit_sets_status(T):
    lg = np.zeros((T, 16), np.float32)
    lg[T - 1, 3] = np.nan
    *_, st = q4.route(torch.from_numpy(lg).cuda(), 2)
    assert st == q4._lib.EDEVICE
    # and a clean call afterwards reports OK again
    *_, st = q4.route(torch.zeros((T, 16), device="cuda"), 2)
    assert st == 0
