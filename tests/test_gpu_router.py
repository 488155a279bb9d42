"""GPU parity of moe_q4_router (router logits) against the fp64 oracle.

Each bf16 product is exact in fp32, so the only error is the fp32 summation
of H terms (plus the fixed-order sum of the K-split partials).  The bound
checked is (H + 64) * 2^-22 * sum_h |x[t][h] w[e][h]| per logit: the
classical n-term summation bound with twice the unit roundoff of
round-to-nearest, so that it also covers an accumulator that truncates."""
import numpy as np
import pytest
import torch

import oracle
import bit_codebook_quantized_router_b200 as q4
from bit_codebook_quantized_router_b200 import inputs
from tests import gpu_support

pytestmark = pytest.mark.gpu


def _case(T, H, E, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((T, H), generator=g).to(torch.bfloat16)
    w = (torch.randn((E, H), generator=g) * 0.02).to(torch.bfloat16)
    return x, w


def _run_guarded(x, w):
    T, H = x.shape
    E = w.shape[0]
    out = gpu_support.Guarded((T, E), torch.float32)
    need = q4.router_workspace(T, H, E)
    ws = gpu_support.Guarded((max(need, 16),), torch.uint8)
    q4.router(x.cuda(), w.cuda(), out=out.view, ws=ws.view)
    torch.cuda.synchronize()
    out.check("logits")
    ws.check("router workspace")
    return out.view.cpu().numpy().astype(np.float64)


# decode sizes (K split over warps and, up to 32 tokens, over clusters of 1 to
# 8 CTAs, 3, 5, 6 and 7 among them; H = 16384 has warps looping over chunks),
# a ragged token count, prefill-like sizes, E not a multiple of 16 and tiny H
@pytest.mark.parametrize("T,H,E", [(1, 6144, 256), (5, 256, 8), (8, 6144, 256), (32, 6144, 256), (33, 512, 40),
                                   (64, 6144, 256), (300, 256, 24), (1, 32, 1), (2, 128, 17), (3, 1024, 33),
                                   (7, 16384, 64), (4, 1536, 48), (6, 4096, 100),
                                   (2, 2560, 64), (3, 5120, 40), (1, 7168, 160)])
def test_router_logits_within_summation_bound(T, H, E):
    x, w = _case(T, H, E, seed=T * 1000 + H + E)
    got = _run_guarded(x, w)
    ref, absdot = oracle.router_logits(inputs.bf16_bits(x), inputs.bf16_bits(w))
    bound = (H + 64) * 2.0 ** -22 * absdot + 1e-30
    err = np.abs(got - ref)
    assert np.all(err <= bound), (np.max(err / bound), T, H, E)


def test_router_prefill_sampled_tokens():
    T, H, E = 2048, 6144, 256
    x, w = _case(T, H, E, seed=77)
    got = _run_guarded(x, w)
    rows = np.random.default_rng(5).choice(T, 48, replace=False)
    ref, absdot = oracle.router_logits(inputs.bf16_bits(x)[rows], inputs.bf16_bits(w))
    assert np.all(np.abs(got[rows] - ref) <= (H + 64) * 2.0 ** -22 * absdot + 1e-30)


def test_router_is_deterministic():
    x, w = _case(3, 6144, 256, seed=9)
    a = q4.router(x.cuda(), w.cuda())
    b = q4.router(x.cuda(), w.cuda())
    assert torch.equal(a, b)


def test_router_rejects_bad_arguments():
    x, w = _case(2, 48, 8, seed=1)  # H % 32 != 0
    with pytest.raises(q4.MoeQ4Error):
        q4.router(x.cuda(), w.cuda())
    assert q4.router_workspace(1, 6144, 256) == 0  # decode sizes: one kernel, no workspace
    x, w = _case(64, 6144, 256, seed=2)
    assert q4.router_workspace(64, 6144, 256) > 0
    with pytest.raises(q4.MoeQ4Error):
        q4.router(x.cuda(), w.cuda(), ws=torch.empty(16, dtype=torch.uint8, device="cuda"))


def test_router_feeds_forward_like_given_logits():
    """logits from moe_q4_router drive moe_q4_forward exactly as the same
    logits handed in directly (the router is the first step of the layer)."""
    w = inputs.WORKLOADS["tiny"]
    layer = gpu_support.device_layer(w)
    x = inputs.activations(w).cuda()
    gate = inputs.router_weight(w).cuda()
    lg = q4.router(x, gate)
    out_a = q4.forward(layer, x, lg, w.shape.k)
    out_b = q4.forward(layer, x, lg.clone(), w.shape.k)
    assert torch.equal(out_a, out_b)
    ids, *_ = q4.route(lg, w.shape.k)
    rids, _ = oracle.route(lg.cpu().numpy(), w.shape.k)
    assert np.array_equal(ids.cpu().numpy(), rids)
