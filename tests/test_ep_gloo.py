"""Expert parallelism on CPU: the dispatch plan, and two or three gloo ranks running
the expert-parallel layer (whole experts per rank, "Round 7", "Owner-locked
decisions" item 11) with the fp64 oracle as every rank's expert computation;
the result must equal the single-process oracle layer over all tokens."""
import os
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from bit_codebook_quantized_router_b200 import ep, inputs
from tests import helpers


def test_expert_ranges_cover_every_expert_once():
    for E, W in ((8, 2), (256, 8), (10, 4), (3, 3), (5, 1)):
        r = ep.expert_ranges(E, W)
        assert r[0][0] == 0 and r[-1][1] == E
        assert all(a <= b for a, b in r) and all(r[i][1] == r[i + 1][0] for i in range(W - 1))
        sizes = [b - a for a, b in r]
        assert max(sizes) - min(sizes) <= 1


def test_plan_orders_rows_by_owner_then_expert_then_token():
    rng = np.random.default_rng(0)
    E, W, T, k = 16, 4, 11, 3
    ids = torch.from_numpy(np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32))
    p = ep.plan_dispatch(ids, E, W)
    flat = ids.reshape(-1).numpy()
    order = p.order.numpy()
    assert sorted(order.tolist()) == list(range(T * k))
    own = ep.owner_of(E, W).numpy()
    keys = [(own[flat[i]], flat[i], i // k, i % k) for i in order]
    assert keys == sorted(keys)
    assert p.send_counts == np.bincount(own[flat], minlength=W).tolist()
    first = np.array([a for a, _ in ep.expert_ranges(E, W)])
    assert np.array_equal(p.local_ids.numpy(), flat[order] - first[own[flat[order]]])


TINY = inputs.WORKLOADS["tiny"]


def _global_inputs(tokens):
    T = sum(tokens)
    x = inputs.bf16_bits(inputs.activations(TINY, T=T, variant=2))
    lg = inputs.router_logits(TINY, T=T, variant=2).numpy()
    return x, lg


def _rank(rank, world, tokens, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        L, _, _ = helpers.build_layer_host(TINY)
        E, k = TINY.shape.E, TINY.shape.k
        x, lg = _global_inputs(tokens)
        t0 = sum(tokens[:rank])
        xr, lgr = x[t0:t0 + tokens[rank]], lg[t0:t0 + tokens[rank]]
        ids, w = oracle.route(lgr, k)
        a, b = ep.expert_ranges(E, world)[rank]
        shard = oracle.Layer(b - a, L.H, L.I, L.tables, L.table_id[a:b])
        for e in range(a, b):
            shard.set_expert(e - a, L.gate_w[e], L.gate_s[e], L.up_w[e], L.up_s[e], L.down_w[e], L.down_s[e])

        def compute(x_rows, local_ids):
            xb = x_rows.view(torch.int16).numpy().view(np.uint16)
            onehot = np.full((x_rows.shape[0], b - a), -30000.0, np.float32)
            onehot[np.arange(x_rows.shape[0]), local_ids.numpy()] = 0.0
            return torch.from_numpy(oracle.moe_tokens(shard, xb, onehot, 1))

        def combine(y, wts):
            yv = y.numpy().reshape(-1, k, L.H)
            out = np.zeros((yv.shape[0], L.H))
            for j in range(k):
                out += wts[:, j:j + 1] * yv[:, j]
            return out

        x_t = torch.from_numpy(xr.view(np.int16).copy()).view(torch.bfloat16)
        out = ep.ep_moe(x_t, torch.from_numpy(ids), w, E, compute, combine, world=world, out_dtype=torch.float64)
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


# tokens held by each rank: two ranks with 4 experts each; three ranks with
# 3, 3 and 2 experts, one of them holding no tokens
@pytest.mark.parametrize("tokens", [(5, 3), (4, 0, 6)])
def test_gloo_ranks_equal_the_single_process_layer(tokens):
    world = len(tokens)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29600 + (os.getpid() + 7 * world) % 300
    procs = [ctx.Process(target=_rank, args=(r, world, tokens, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    L, _, _ = helpers.build_layer_host(TINY)
    x, lg = _global_inputs(tokens)
    ref = oracle.moe_tokens(L, x, lg, TINY.shape.k)
    got = np.concatenate([res[r] for r in range(world)])
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-14 * np.abs(ref).max())
