"""Pins for the oracle's routing and grouping: library sorts and softmax on the
same logits, and the invariants a grouping must satisfy."""
import numpy as np
import pytest
import scipy.special

import oracle
from bit_codebook_quantized_router_b200 import inputs


def _library_topk(logits, k):
    # numpy lexsort: primary key -logit, secondary key expert id (ties -> lower id)
    T, E = logits.shape
    ids = np.empty((T, k), np.int32)
    for t in range(T):
        order = np.lexsort((np.arange(E), -logits[t].astype(np.float64)))
        ids[t] = order[:k]
    return ids


@pytest.mark.parametrize("T,E,k,quant", [(64, 256, 8, None), (200, 8, 2, None), (300, 16, 4, 0.5),
                                         (50, 256, 8, 1.0), (7, 3, 3, None), (5, 1, 1, None)])
def test_topk_and_softmax_match_library(T, E, k, quant):
    rng = np.random.default_rng(T * 31 + E)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    if quant:  # force many exact ties
        lg = (np.round(lg / quant) * quant).astype(np.float32)
    lg[0, : min(E, 3)] = -0.0
    ids, w = oracle.route(lg, k)
    assert np.array_equal(ids, _library_topk(lg, k))
    sel = np.take_along_axis(lg.astype(np.float64), ids, 1)
    assert np.allclose(w, scipy.special.softmax(sel, axis=1), rtol=1e-14, atol=0)
    assert np.allclose(w.sum(1), 1.0, rtol=1e-14)
    assert np.all(np.diff(w, axis=1) <= 0)  # descending logit -> non-increasing weight


def test_negative_and_positive_zero_tie_to_lower_id():
    lg = np.array([[0.0, -0.0, 0.0, -1.0]], np.float32)
    lg[0, 0] = -0.0
    ids, _ = oracle.route(lg, 3)
    assert list(ids[0]) == [0, 1, 2]


def test_route_rejects_non_finite():
    for bad in (np.nan, np.inf, -np.inf):
        lg = np.zeros((2, 8), np.float32)
        lg[1, 5] = bad
        with pytest.raises(oracle.OracleError):
            oracle.route(lg, 2)
    with pytest.raises(oracle.OracleError):
        oracle.route(np.zeros((2, 8), np.float32), 9)


@pytest.mark.parametrize("T,E,k", [(1, 256, 8), (64, 256, 8), (500, 8, 2), (0, 8, 2), (33, 4, 4)])
def test_grouping_matches_stable_library_sort(T, E, k):
    rng = np.random.default_rng(T + E)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    ids, _ = oracle.route(lg, k) if T else (np.zeros((0, k), np.int32), None)
    counts, offsets, row_token, inv = oracle.group(ids, E)
    flat = ids.reshape(-1)
    # numpy stable argsort by expert id over the token-major (t, j) order
    order = np.argsort(flat, kind="stable")
    assert np.array_equal(row_token, order // k)
    assert np.array_equal(counts, np.bincount(flat, minlength=E))
    assert offsets[0] == 0 and np.array_equal(np.diff(offsets), counts)
    assert offsets[-1] == T * k
    # inverse maps
    rows = inv.reshape(-1)
    assert np.array_equal(np.sort(rows), np.arange(T * k))
    for t in range(T):
        for j in range(k):
            r = inv[t, j]
            assert row_token[r] == t
            e = ids[t, j]
            assert offsets[e] <= r < offsets[e + 1]
    # token order ascending inside every expert segment
    for e in range(E):
        seg = row_token[offsets[e]:offsets[e + 1]]
        assert np.all(np.diff(seg) > 0)


def test_zipf_workload_is_skewed():
    # The skewed workloads must have experts above 200 rows and experts at 0.
    w = inputs.WORKLOADS["prefill_t2048"]
    lg = inputs.router_logits(w).numpy()
    ids, _ = oracle.route(lg, 8)
    counts, *_ = oracle.group(ids, 256)
    assert counts.max() > 200 and (counts > 200).sum() >= 5
    assert (counts == 0).sum() >= 20
    assert counts.sum() == 2048 * 8
