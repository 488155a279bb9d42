"""Every token of the large GLM-shaped workloads, not only the oracle's samples.

The forward's fp32 combine result is compared with a plain PyTorch fp32
evaluation of the same layer, built from:
- the library's per-expert dequantisation, which the pack/dequant tests hold
  bit-exact against the oracle;
- the forward's own routing, which the forward tests hold bit-exact against
  the oracle.

A (token, slot) row that is dropped, or written twice, anywhere moves that
token's output by the slot's share of it (at least several percent with
top-8 softmax weights), far outside the per-token bound below.  The file runs
after the other GPU tests."""
import numpy as np
import pytest
import torch

import bit_codebook_quantized_router_b200 as q4
from bit_codebook_quantized_router_b200 import inputs
from tests import gpu_support

pytestmark = pytest.mark.gpu

# The two evaluations differ by the bf16 storage of h between the GEMMs
# (about 2^-9 relative per element) and by summation order: about 1e-3 per
# token.  A missing or doubled slot is several percent.
ROW_REL = 1e-2
ALL_REL = gpu_support.REL_FRO


def _reference(layer: q4.Layer, x: torch.Tensor, ids: torch.Tensor, wts: torch.Tensor) -> torch.Tensor:
    """out[t] = sum_j w[t, j] * Wd_e (silu(Wg_e x_t) * (Wu_e x_t)), e = ids[t, j], in fp32."""
    T, H = x.shape
    k = ids.shape[1]
    out = torch.zeros((T, H), dtype=torch.float32, device=x.device)
    xf = x.float()
    flat = ids.reshape(-1).long()
    tok = torch.arange(T, device=x.device).repeat_interleave(k)
    wf = wts.reshape(-1).float()
    for e in torch.unique(flat).tolist():
        sel = (flat == e).nonzero().squeeze(1)
        t_e = tok[sel]
        tid = layer.table_id[e:e + 1]

        def weights(codes, scales):
            return q4.dequant(codes[e:e + 1], scales[e:e + 1], layer.tables, tid)[0].float()

        xs = xf[t_e]
        g = xs @ weights(layer.gate_w, layer.gate_s).T
        u = xs @ weights(layer.up_w, layer.up_s).T
        y = (torch.nn.functional.silu(g) * u) @ weights(layer.down_w, layer.down_s).T
        out.index_add_(0, t_e, y * wf[sel, None])
    return out


@pytest.mark.parametrize("name", ["decode_t64", "prefill_t2048", "prefill_t8192"])
def test_every_token_matches_a_torch_evaluation(name):
    w = inputs.WORKLOADS[name]
    layer = gpu_support.device_layer(w)
    x = inputs.activations(w, device="cuda")
    lg = inputs.router_logits(w, device="cuda")
    T, k = w.T, w.shape.k
    ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
    wts = torch.empty((T, k), dtype=torch.float32, device="cuda")
    out_f32 = torch.empty((T, w.shape.H), dtype=torch.float32, device="cuda")
    ws = q4.alloc_workspace(q4.forward_workspace(layer, T, k))
    q4.forward(layer, x, lg, k, ws=ws, topk_ids=ids, topk_w=wts, out_f32=out_f32)
    torch.cuda.synchronize()
    assert q4.forward_status(ws) == 0
    tf32 = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    try:
        ref = _reference(layer, x, ids, wts)
    finally:
        torch.backends.cuda.matmul.allow_tf32 = tf32
    torch.cuda.synchronize()
    assert bool(torch.isfinite(out_f32).all())
    err = (out_f32.double() - ref.double()).norm(dim=1)
    nrm = ref.double().norm(dim=1)
    row_rel = (err / nrm).cpu().numpy()
    worst = int(np.argmax(row_rel))
    assert row_rel[worst] <= ROW_REL, f"{name}: token {worst} off by {row_rel[worst]:.3e} relative"
    all_rel = float(err.norm() / nrm.norm())
    assert all_rel <= ALL_REL, f"{name}: all tokens off by {all_rel:.3e} relative"
