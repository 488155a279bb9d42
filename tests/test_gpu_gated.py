"""GPU parity of moe_q4_forward_gated: the layer from the hidden states, the
bf16 router gate in front ("GLM-5.2-EXL3-DENSE6-MTP78", "Quant recipe").

The gated call must give (a) logits bit-identical to moe_q4_router's (the
same sums in the same order) and within the fp32 summation bound of the
fp64 oracle, (b) the oracle's routing of those logits, (c) output, ids,
weights and counts bit-identical to moe_q4_forward on those logits, and
(d) output within the layer tolerance of the fp64 oracle.  Decode sizes
(T <= 32) take the fused router + routing launch; larger T the router
kernels then the routing kernels."""
import numpy as np
import pytest
import torch

import oracle
import bit_codebook_quantized_router_b200 as q4
from bit_codebook_quantized_router_b200 import inputs
from tests import gpu_support
from tests.test_gpu_forward import _small_device_layer

pytestmark = pytest.mark.gpu


def _gated_guarded(dev, shared, gate, x, k):
    T, E = x.shape[0], dev.E
    G = gpu_support.Guarded
    bufs = {"out": G((T, dev.H), torch.bfloat16), "out_f32": G((T, dev.H), torch.float32),
            "logits": G((T, E), torch.float32), "ids": G((T, k), torch.int32), "wts": G((T, k), torch.float32),
            "counts": G((E,), torch.int32), "ws": G((q4.forward_gated_workspace(dev, shared, T, k),), torch.uint8)}
    v = {n: b.view for n, b in bufs.items()}
    q4.forward_gated(dev, shared, gate, x, k, out=v["out"], ws=v["ws"], logits=v["logits"], topk_ids=v["ids"],
                     topk_w=v["wts"], counts=v["counts"], out_f32=v["out_f32"])
    torch.cuda.synchronize()
    assert q4.forward_status(v["ws"]) == 0
    for n, b in bufs.items():
        b.check(n)
    gpu_support.check_bf16_is_rounding(v["out"], v["out_f32"])
    return {n: t.clone() for n, t in v.items() if n != "ws"}


def _check_against_router_and_forward(dev, shared, gate, x, k, g):
    """(a) and (c): the gated results equal the two-call path bit for bit.
    One exception: with T = 1 the logits-input forward's gate/up kernel routes
    the token itself on one CTA fewer (the logits are an input there, not a
    result of the same call), so its K split, hence the rounding of its
    partial sums, differs; there the outputs agree to fp32 reordering."""
    T = x.shape[0]
    lg = q4.router(x, gate)
    assert torch.equal(g["logits"], lg), "gated logits differ from moe_q4_router's"
    out_f32 = torch.empty((T, dev.H), dtype=torch.float32, device="cuda")
    ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
    wts = torch.empty((T, k), dtype=torch.float32, device="cuda")
    counts = torch.empty((dev.E,), dtype=torch.int32, device="cuda")
    if shared is None:
        out = q4.forward(dev, x, lg, k, topk_ids=ids, topk_w=wts, counts=counts, out_f32=out_f32)
    else:
        out = q4.forward_ex(dev, shared, x, lg, k, topk_ids=ids, topk_w=wts, counts=counts, out_f32=out_f32)
    torch.cuda.synchronize()
    for name, a, b in (("ids", g["ids"], ids), ("weights", g["wts"], wts), ("counts", g["counts"], counts)):
        assert torch.equal(a, b), f"gated {name} differs from router + forward"
    if T > 1:
        assert torch.equal(g["out"], out) and torch.equal(g["out_f32"], out_f32), "gated output differs"
    else:
        rms = out_f32.double().pow(2).mean().sqrt().item()
        assert (g["out_f32"].double() - out_f32.double()).abs().max().item() <= 1e-5 * rms


def _check_logits_and_routing(gate, x, k, g):
    """(a) against the oracle and (b)."""
    H = x.shape[1]
    ref, absdot = oracle.router_logits(inputs.bf16_bits(x), inputs.bf16_bits(gate))
    got = g["logits"].cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - ref) <= (H + 64) * 2.0 ** -22 * absdot + 1e-30)
    lg_h = g["logits"].cpu().numpy()
    rids, rw = oracle.route(lg_h, k)
    assert np.array_equal(g["ids"].cpu().numpy(), rids)
    np.testing.assert_allclose(g["wts"].cpu().numpy(), rw, rtol=1e-6)
    rc, *_ = oracle.group(rids, g["counts"].numel())
    assert np.array_equal(g["counts"].cpu().numpy(), rc)
    return lg_h


# small layer (H=256, I=128, E=8): T <= 32 fused (one to four 8-token column
# tiles, an expert above the small-M limit at T=17 and 32), T > 32 through the
# mma.sync router (E % 128 != 0) and the routing kernels
@pytest.mark.parametrize("T,k", [(1, 2), (5, 2), (8, 1), (17, 2), (32, 3), (33, 2), (40, 8)])
def test_small_layer_gated(T, k):
    w = inputs.Workload("gated", 21, T, inputs.TINY)
    L, dev = _small_device_layer(w)
    gate = inputs.router_weight(w, device="cuda")
    x = inputs.activations(w).cuda()
    g = _gated_guarded(dev, None, gate, x, k)
    _check_against_router_and_forward(dev, None, gate, x, k, g)
    lg_h = _check_logits_and_routing(gate, x, k, g)
    ref = oracle.moe_tokens(L, inputs.bf16_bits(x), lg_h, k)
    gpu_support.check_out(g["out_f32"], ref, f"gated T={T} k={k}")


# with a shared expert: at a decode size (fused router + routing) and above it
# (the router kernels, the routing kernels, then the shared expert's launches)
@pytest.mark.parametrize("T", [6, 40])
def test_small_layer_gated_with_shared_expert(T):
    w = inputs.Workload("gated_shared", 22, T, inputs.TINY)
    L, dev = _small_device_layer(w)
    gu, dn = inputs.shared_expert_weights(w, I=128, device="cuda")
    sh = q4.Shared(gu, dn)
    gate = inputs.router_weight(w, device="cuda")
    x = inputs.activations(w).cuda()
    g = _gated_guarded(dev, sh, gate, x, 2)
    _check_against_router_and_forward(dev, sh, gate, x, 2, g)
    lg_h = _check_logits_and_routing(gate, x, 2, g)
    x_bits = inputs.bf16_bits(x)
    ref = oracle.moe_tokens(L, x_bits, lg_h, 2) + oracle.shared_ffn(x_bits, inputs.bf16_bits(gu), inputs.bf16_bits(dn))
    gpu_support.check_out(g["out_f32"], ref, f"gated + shared expert T={T}")


def test_gated_calls_in_a_row_share_one_workspace():
    """The fused kernel's ticket returns to zero after every call: calls of
    different sizes on one workspace (decode sizes, then a larger one, then
    decode again) each match their two-call results."""
    w = inputs.Workload("gated_seq", 23, 40, inputs.TINY)
    _, dev = _small_device_layer(w)
    gate = inputs.router_weight(w, device="cuda")
    ws = q4.alloc_workspace(q4.forward_gated_workspace(dev, None, 40, 2))
    for T in (8, 1, 3, 40, 5, 5):
        x = inputs.activations(w, T=T, variant=T).cuda()
        out = q4.forward_gated(dev, None, gate, x, 2, ws=ws)
        ref = q4.forward(dev, x, q4.router(x, gate), 2)
        torch.cuda.synchronize()
        assert q4.forward_status(ws) == 0
        assert torch.equal(out, ref), f"T={T}"


# GLM-shaped layer: the fused launch at T=1 and T=8, the tcgen05 router at
# T=64; every token of T <= 8 against the oracle, samples at T=64
@pytest.mark.parametrize("name,T,n_sample", [("decode_t1", 1, None), ("decode_t8", 8, None), ("decode_t8", 32, 3),
                                             ("decode_t8", 64, 3)])
def test_glm_layer_gated(name, T, n_sample):
    w = inputs.WORKLOADS[name]
    dev = gpu_support.device_layer(w)
    gate = inputs.router_weight(w, device="cuda")
    x = inputs.activations(w, device="cuda", T=T, variant=3)
    k = w.shape.k
    g = _gated_guarded(dev, None, gate, x, k)
    _check_against_router_and_forward(dev, None, gate, x, k, g)
    lg_h = _check_logits_and_routing(gate, x, k, g)
    tokens = list(range(T)) if n_sample is None else sorted(
        np.random.default_rng(T).choice(T, n_sample, replace=False).tolist())
    rids, _ = oracle.route(lg_h, k)
    L = gpu_support.oracle_layer(w, np.unique(rids[tokens]), dev)
    ref = gpu_support.oracle_tokens(L, inputs.bf16_bits(x), lg_h, k, tokens)
    gpu_support.check_out(g["out_f32"][tokens], ref, f"{name} gated T={T}")


def test_gated_rejects_bad_arguments():
    w = inputs.Workload("gated_bad", 24, 4, inputs.TINY)
    _, dev = _small_device_layer(w)
    gate = inputs.router_weight(w, device="cuda")
    x = inputs.activations(w).cuda()
    E, H = gate.shape
    flat = torch.zeros(E * H + 8, dtype=torch.bfloat16, device="cuda")
    shifted = flat[1:1 + E * H].view(E, H)  # 2 bytes off the 16-byte alignment
    with pytest.raises(q4.MoeQ4Error):
        q4.forward_gated(dev, None, shifted, x, 2)
    ws = q4.alloc_workspace(q4.forward_gated_workspace(dev, None, 4, 2))
    with pytest.raises(q4.MoeQ4Error):
        q4.forward_gated(dev, None, gate, x, 2, ws=ws[:ws.numel() - 256])  # short workspace
    assert q4.forward_gated_workspace(dev, None, 4, 2) > q4.forward_workspace(dev, 4, 2)
