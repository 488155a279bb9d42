"""GPU parity of the layer with a BF16 shared expert (moe_q4_forward_ex
through the C ABI) against the fp64 oracle: the routed layer plus the shared
expert ("GLM-5.2 EXL3 TR3 v4" README, "Checkpoint layout update": gate and up
merged into one BF16 payload), within the layer tolerance (relative Frobenius
5e-3, max-abs 2e-2 * rms) on the fp32 combine result."""
import numpy as np
import pytest
import torch

import oracle
import bit_codebook_quantized_router_b200 as q4
from bit_codebook_quantized_router_b200 import inputs
from tests import gpu_support
from tests.test_gpu_forward import _small_device_layer

pytestmark = pytest.mark.gpu


def _run(dev, shared, x, lg, k):
    T = x.shape[0]
    G = gpu_support.Guarded
    bufs = {"out_f32": G((T, dev.H), torch.float32), "out": G((T, dev.H), torch.bfloat16),
            "ws": G((q4.forward_ex_workspace(dev, shared, T, k),), torch.uint8)}
    out = q4.forward_ex(dev, shared, x, lg, k, out=bufs["out"].view, ws=bufs["ws"].view, out_f32=bufs["out_f32"].view)
    torch.cuda.synchronize()
    assert q4.forward_status(bufs["ws"].view) == 0
    for name, b in bufs.items():
        b.check(name)
    gpu_support.check_bf16_is_rounding(out, bufs["out_f32"].view)
    return bufs["out_f32"].view


def _ref(L, x_bits, lg_h, k, gu, dn, tokens):
    routed = gpu_support.oracle_tokens(L, x_bits, lg_h, k, tokens)
    shared = oracle.shared_ffn(x_bits[list(tokens)], inputs.bf16_bits(gu), inputs.bf16_bits(dn))
    return routed + shared


@pytest.mark.parametrize("T,k", [(1, 2), (4, 2), (16, 2), (17, 1), (300, 3)])
def test_small_layer_with_shared_expert(T, k):
    w = inputs.Workload("shared", 14, T, inputs.TINY)
    L, dev = _small_device_layer(w)
    gu, dn = inputs.shared_expert_weights(w, I=256, device="cuda")
    sh = q4.Shared(gu, dn)
    x = inputs.activations(w)
    lg = inputs.router_logits(w)
    out = _run(dev, sh, x.cuda(), lg.cuda(), k)
    ref = _ref(L, inputs.bf16_bits(x), lg.numpy(), k, gu, dn, range(T))
    gpu_support.check_out(out, ref, f"shared T={T} k={k}")


# At decode sizes the shared expert's GEMMs split K over the SMs.  A layer
# with longer K than the tiny one (H = 1024, shared I = 512) makes its gate/up
# split 16 k-steps in 4 and its down 8 in 2; the split partial sums are added
# in split order by a second kernel, and a repeat gives the same bits.
@pytest.mark.parametrize("T", [1, 3, 16])
def test_shared_expert_with_k_splits(T):
    w = inputs.Workload("shared_split", 17, T, inputs.Shape(H=1024, I=256, E=8, k=2))
    L, dev = _small_device_layer(w)
    gu, dn = inputs.shared_expert_weights(w, I=512, device="cuda")
    sh = q4.Shared(gu, dn)
    x = inputs.activations(w)
    lg = inputs.router_logits(w)
    out = _run(dev, sh, x.cuda(), lg.cuda(), 2)
    ref = _ref(L, inputs.bf16_bits(x), lg.numpy(), 2, gu, dn, range(T))
    gpu_support.check_out(out, ref, f"shared with K splits T={T}")
    again = _run(dev, sh, x.cuda(), lg.cuda(), 2)
    assert torch.equal(out, again)


def test_without_shared_expert_equals_forward():
    w = inputs.Workload("shared0", 15, 6, inputs.TINY)
    _, dev = _small_device_layer(w)
    x, lg = inputs.activations(w).cuda(), inputs.router_logits(w).cuda()
    a = torch.empty((6, dev.H), dtype=torch.float32, device="cuda")
    b = torch.empty_like(a)
    q4.forward(dev, x, lg, 2, out_f32=a)
    q4.forward_ex(dev, None, x, lg, 2, out_f32=b)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_repeat_is_bit_identical():
    w = inputs.Workload("shared_det", 16, 40, inputs.TINY)
    _, dev = _small_device_layer(w)
    gu, dn = inputs.shared_expert_weights(w, I=128, device="cuda")
    sh = q4.Shared(gu, dn)
    x, lg = inputs.activations(w).cuda(), inputs.router_logits(w).cuda()
    a = _run(dev, sh, x, lg, 2).clone()
    b = _run(dev, sh, x, lg, 2)
    assert torch.equal(a, b)


@pytest.mark.parametrize("name,n_sample", [("decode_t1", None), ("decode_t8", None), ("prefill_t2048", 4)])
def test_glm_layer_with_shared_expert(name, n_sample):
    w = inputs.WORKLOADS[name]
    dev = gpu_support.device_layer(w)
    gu, dn = inputs.shared_expert_weights(w, device="cuda")
    sh = q4.Shared(gu, dn)
    x = inputs.activations(w, device="cuda")
    lg = inputs.router_logits(w, device="cuda")
    k = w.shape.k
    out = _run(dev, sh, x, lg, k)
    lg_h = lg.cpu().numpy()
    rids, _ = oracle.route(lg_h, k)
    if n_sample is None:
        tokens = list(range(w.T))
    else:
        rng = np.random.default_rng(99)
        tokens = sorted(rng.choice(w.T, n_sample, replace=False).tolist())
    L = gpu_support.oracle_layer(w, np.unique(rids[tokens]), dev)
    ref = _ref(L, inputs.bf16_bits(x), lg_h, k, gu, dn, tokens)
    gpu_support.check_out(out[tokens], ref, f"{name} + shared expert")
