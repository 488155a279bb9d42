"""The expert-parallel path on one GPU: the weighted combine alone
(moe_q4_combine) and the expert-parallel layer with a single rank (the
dispatch plan, the library's forward as the experts' computation, the
combine) against the fp64 oracle.  (Several ranks are covered on CPU with
gloo in tests/test_ep_gloo.py.)"""
import numpy as np
import pytest
import torch

import oracle
import bit_codebook_quantized_router_b200 as q4
from bit_codebook_quantized_router_b200 import ep, inputs
from tests import gpu_support
from tests.test_gpu_forward import _small_device_layer

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T", [37, 300])
@pytest.mark.parametrize("k", [1, 5, 8, 11, 16])
@pytest.mark.parametrize("with_inv", [False, True])
def test_combine_alone(with_inv, k, T):
    # up to 64 tokens the kernel takes the slots eight at a time: k below, at,
    # between and at twice that round; above 64 tokens one slot at a time
    g = torch.Generator(device="cuda").manual_seed(3 + k + T)
    H = 384
    y = torch.randn((T * k, H), generator=g, device="cuda")
    w = torch.rand((T, k), generator=g, device="cuda")
    inv = None
    yy = y
    if with_inv:
        perm = torch.randperm(T * k, generator=g, device="cuda")
        inv = perm.to(torch.int32).reshape(T, k)
        yy = torch.empty_like(y)
        yy[perm] = y  # row (t, j) sits at inv[t][j]
    out32 = torch.empty((T, H), dtype=torch.float32, device="cuda")
    out = q4.combine(yy, w, inv=inv, out_f32=out32)
    torch.cuda.synchronize()
    ref = torch.zeros((T, H), dtype=torch.float64, device="cuda")
    for j in range(k):
        ref += w[:, j:j + 1].double() * y.view(T, k, H)[:, j].double()
    assert torch.allclose(out32.double(), ref, rtol=1e-6, atol=1e-6)
    assert torch.equal(out, out32.to(torch.bfloat16))


def _ep(dev, x, lg, k):
    ids, w, *_ = q4.route(lg, k)
    out32 = torch.empty((x.shape[0], dev.H), dtype=torch.float32, device="cuda")

    def combine(y, wt):
        q4.combine(y, wt, out_f32=out32)
        return out32
    return ep.ep_moe(x, ids, w, dev.E, ep.gpu_compute(dev), combine, world=1)


def test_single_rank_expert_parallel_layer_small():
    w = inputs.Workload("ep1", 18, 24, inputs.TINY)
    L, dev = _small_device_layer(w)
    x, lg = inputs.activations(w), inputs.router_logits(w)
    out = _ep(dev, x.cuda(), lg.cuda(), 2)
    torch.cuda.synchronize()
    ref = oracle.moe_tokens(L, inputs.bf16_bits(x), lg.numpy(), 2)
    gpu_support.check_out(out, ref, "single-rank EP, small layer")


def test_single_rank_expert_parallel_layer_glm_decode():
    w = inputs.WORKLOADS["decode_t8"]
    dev = gpu_support.device_layer(w)
    x, lg = inputs.activations(w, device="cuda"), inputs.router_logits(w, device="cuda")
    k = w.shape.k
    out = _ep(dev, x, lg, k)
    torch.cuda.synchronize()
    lg_h = lg.cpu().numpy()
    rids, _ = oracle.route(lg_h, k)
    L = gpu_support.oracle_layer(w, np.unique(rids), dev)
    ref = gpu_support.oracle_tokens(L, inputs.bf16_bits(x), lg_h, k, range(w.T))
    gpu_support.check_out(out, ref, "single-rank EP, GLM decode T=8")


def test_shard_layer_views_the_experts_of_a_rank():
    w = inputs.Workload("ep_shard", 19, 4, inputs.TINY)
    _, dev = _small_device_layer(w)
    for rank in range(3):
        s = ep.shard_layer(dev, rank, 3)
        a, b = ep.expert_ranges(dev.E, 3)[rank]
        assert s.E == b - a
        assert s.gate_w.data_ptr() == dev.gate_w[a].data_ptr()
        assert np.array_equal(s.table_id, dev.table_id[a:b])
