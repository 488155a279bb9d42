"""GPU parity of the whole layer (moe_q4_forward through the C ABI) against
the fp64 oracle: relative Frobenius error <= 5e-3 and max-abs error <=
2e-2 * rms(oracle output), on the tiny workload in full, on small layers
built for edge cases, and on the GLM-shaped workloads (in full where the
oracle finishes in seconds, else on seeded token samples)."""
import numpy as np
import pytest
import torch

import oracle
import bit_codebook_quantized_router_b200 as q4
from bit_codebook_quantized_router_b200 import inputs
from tests import gpu_support, helpers

pytestmark = pytest.mark.gpu


def _small_device_layer(w, identical_to=None):
    """Small layers: pack on the host with the oracle, upload the bytes (so
    the forward is tested independently of the GPU pack)."""
    L, packed, _ = helpers.build_layer_host(w, identical_to=identical_to)
    sh = w.shape

    def stack(proj, i):
        return torch.from_numpy(np.stack([packed[e][proj][i] for e in range(sh.E)])).cuda()

    dev = q4.Layer(stack("gate", 0), stack("gate", 1), stack("up", 0), stack("up", 1),
                   stack("down", 0), stack("down", 1), L.tables, L.table_id)
    return L, dev


def _run(dev, x, lg, k):
    """One forward with every output and the workspace inside canary bands."""
    T = x.shape[0]
    G = gpu_support.Guarded
    bufs = {"ids": G((T, k), torch.int32), "wts": G((T, k), torch.float32), "counts": G((dev.E,), torch.int32),
            "out_f32": G((T, dev.H), torch.float32), "out": G((T, dev.H), torch.bfloat16),
            "ws": G((q4.forward_workspace(dev, T, k),), torch.uint8)}
    ids, wts, counts = bufs["ids"].view, bufs["wts"].view, bufs["counts"].view
    out_f32, ws = bufs["out_f32"].view, bufs["ws"].view
    out = q4.forward(dev, x, lg, k, out=bufs["out"].view, ws=ws, topk_ids=ids, topk_w=wts, counts=counts,
                     out_f32=out_f32)
    torch.cuda.synchronize()
    assert q4.forward_status(ws) == 0
    for name, b in bufs.items():
        b.check(name)
    gpu_support.check_bf16_is_rounding(out, out_f32)
    return out_f32, ids, wts, counts


def test_tiny_workload_full():
    w = inputs.WORKLOADS["tiny"]
    L, dev = _small_device_layer(w)
    x = inputs.activations(w)
    lg = inputs.router_logits(w)
    out, ids, wts, counts = _run(dev, x.cuda(), lg.cuda(), w.shape.k)
    ref, rids, rw = oracle.moe_tokens(L, inputs.bf16_bits(x), lg.numpy(), w.shape.k, return_routing=True)
    assert np.array_equal(ids.cpu().numpy(), rids)
    np.testing.assert_allclose(wts.cpu().numpy(), rw, rtol=1e-6)
    gpu_support.check_out(out, ref, "tiny")


# Edge cases on a small layer (H=256, I=128, E=8): T=1; an expert with
# exactly the small-M path's limit (16 rows) and one more (17, the tensor-core
# path); exactly one tensor-core token tile (256) and one more (257), a tile
# and a half (384, 385), ragged single tiles (192, 193); experts with 0 rows;
# every token on one expert; k = 1; k = E.
@pytest.mark.parametrize("T,k,bias", [(1, 2, None), (16, 1, 3), (17, 1, 3), (33, 2, None),
                                      (40, 2, 5), (64, 8, None), (192, 1, 3), (193, 1, 3), (200, 2, None),
                                      (256, 1, 3), (257, 1, 3), (300, 3, 0), (384, 1, 3), (385, 1, 3)])
def test_small_layer_edge_counts(T, k, bias):
    w = inputs.Workload("small", 7, T, inputs.TINY)
    L, dev = _small_device_layer(w)
    x = inputs.activations(w)
    lg = inputs.router_logits(w)
    if bias is not None:
        lg[:, bias] += 50.0  # every token picks expert `bias` first
    out, ids, wts, counts = _run(dev, x.cuda(), lg.cuda(), k)
    ref, rids, _ = oracle.moe_tokens(L, inputs.bf16_bits(x), lg.numpy(), k, return_routing=True)
    assert np.array_equal(ids.cpu().numpy(), rids)
    rc = np.bincount(rids.reshape(-1), minlength=8)
    assert np.array_equal(counts.cpu().numpy(), rc)
    gpu_support.check_out(out, ref, f"T={T} k={k}")


# The wide tensor-core tiles (experts with 17 to 128 rows: the tokens as MMA M,
# 256 weight rows as N) on a layer whose I and H are multiples of 256 (H=512,
# I=256, E=8): an expert with exactly the small-M limit (16 rows) and one more
# (17), with the wide limit (128) and one more (129, swap-AB), a mix of wide
# and swap-AB experts, and k = E (every expert wide).  Every token against the
# oracle.
@pytest.mark.parametrize("T,k,bias", [(16, 1, 3), (17, 1, 3), (128, 1, 3), (129, 1, 3), (100, 2, None),
                                      (300, 3, 0), (60, 8, None)])
def test_wide_tensor_core_tiles(T, k, bias):
    w = inputs.Workload("wide", 18, T, inputs.Shape(H=512, I=256, E=8, k=k))
    L, dev = _small_device_layer(w)
    x = inputs.activations(w)
    lg = inputs.router_logits(w)
    if bias is not None:
        lg[:, bias] += 50.0  # every token picks expert `bias` first
    out, ids, wts, counts = _run(dev, x.cuda(), lg.cuda(), k)
    ref, rids, _ = oracle.moe_tokens(L, inputs.bf16_bits(x), lg.numpy(), k, return_routing=True)
    assert np.array_equal(ids.cpu().numpy(), rids)
    gpu_support.check_out(out, ref, f"wide tiles T={T} k={k}")


# K a multiple of 128 but not of 256 (H = I = 384): the small-M path streams
# 128-K stages of 64-byte code rows, several per tile; T <= 8 and T > 8 take
# the two activation tile heights of the down projection.
@pytest.mark.parametrize("T,k", [(1, 2), (5, 2), (9, 1), (24, 3)])
def test_layer_k_not_multiple_of_256(T, k):
    w = inputs.Workload("k384", 9, T, inputs.Shape(H=384, I=384, E=8, k=k))
    L, dev = _small_device_layer(w)
    x = inputs.activations(w)
    lg = inputs.router_logits(w)
    out, ids, _, _ = _run(dev, x.cuda(), lg.cuda(), k)
    ref, rids, _ = oracle.moe_tokens(L, inputs.bf16_bits(x), lg.numpy(), k, return_routing=True)
    assert np.array_equal(ids.cpu().numpy(), rids)
    gpu_support.check_out(out, ref, f"H=I=384 T={T} k={k}")


# One token: the small-M gate/up kernel routes the token itself (the routing
# kernel's warp top-k on the same logits) and starts before the routing kernel
# ends.  Equal logits (lower id first), a tie at the k-th place and top-k ids
# in descending id order must still select and order the oracle's experts.
@pytest.mark.parametrize("case", ["ties", "tie_at_k", "descending_ids"])
def test_one_token_self_routing(case):
    w = inputs.Workload("one", 12, 1, inputs.TINY)
    L, dev = _small_device_layer(w)
    x = inputs.activations(w)
    lg = inputs.router_logits(w)
    k = 3
    if case == "ties":
        lg[0, :] = torch.tensor([2.0, 3.0, 3.0, 1.0, 3.0, 0.5, 3.0, -1.0])
    elif case == "tie_at_k":
        lg[0, :] = torch.tensor([1.0, 4.0, 2.0, 2.0, 0.0, 5.0, 2.0, 2.0])
    else:
        lg[0, :] = torch.arange(8, dtype=torch.float32)
    out, ids, _, _ = _run(dev, x.cuda(), lg.cuda(), k)
    ref, rids, _ = oracle.moe_tokens(L, inputs.bf16_bits(x), lg.numpy(), k, return_routing=True)
    assert np.array_equal(ids.cpu().numpy(), rids)
    gpu_support.check_out(out, ref, f"one token, {case}")


def test_one_token_non_finite_logit_reports_device_status():
    w = inputs.Workload("one_nan", 13, 1, inputs.TINY)
    _, dev = _small_device_layer(w)
    lg = inputs.router_logits(w).cuda()
    lg[0, 3] = float("nan")
    ws = q4.alloc_workspace(q4.forward_workspace(dev, 1, 2))
    q4.forward(dev, inputs.activations(w).cuda(), lg, 2, ws=ws)
    assert q4.forward_status(ws) == q4._lib.EDEVICE


def test_identical_experts_equal_dense_ffn():
    w = inputs.Workload("ident", 8, 24, inputs.TINY)
    L, dev = _small_device_layer(w, identical_to=2)
    x = inputs.activations(w)
    lg = inputs.router_logits(w)
    out, *_ = _run(dev, x.cuda(), lg.cuda(), 3)
    ref = oracle.moe_tokens(L, inputs.bf16_bits(x), lg.numpy(), 1)  # k=1 equals any k here
    gpu_support.check_out(out, ref, "identical experts")


def test_zero_activations_give_zero():
    w = inputs.Workload("zero", 9, 5, inputs.TINY)
    L, dev = _small_device_layer(w)
    x = torch.zeros((5, 256), dtype=torch.bfloat16, device="cuda")
    lg = inputs.router_logits(w).cuda()
    out, *_ = _run(dev, x, lg, 2)
    assert torch.all(out == 0)


def test_mixed_tables_small():
    w = inputs.Workload("mixed", 10, 48, inputs.TINY, mixed_tables=True)
    tables, tid = inputs.layer_tables(w)
    tid = tid.copy()
    tid[[1, 6]] = 1
    sh = w.shape
    L = oracle.Layer(sh.E, sh.H, sh.I, tables, tid)
    parts = {p: ([], []) for p in inputs.PROJECTIONS}
    for e in range(sh.E):
        pe = {}
        for proj in inputs.PROJECTIONS:
            N, K = inputs.proj_shape(sh, proj)
            c, s = oracle.pack(inputs.bf16_bits(inputs.expert_weight(w, e, proj))[None], tables,
                               tid[e:e + 1], 1, N, K)
            pe[proj] = (c[0], s[0])
            parts[proj][0].append(c[0])
            parts[proj][1].append(s[0])
        L.set_expert(e, *pe["gate"], *pe["up"], *pe["down"])
    t = {p: [torch.from_numpy(np.stack(v)).cuda() for v in parts[p]] for p in parts}
    dev = q4.Layer(*t["gate"], *t["up"], *t["down"], tables, tid)
    x = inputs.activations(w)
    lg = inputs.router_logits(w)
    out, *_ = _run(dev, x.cuda(), lg.cuda(), 2)
    ref = oracle.moe_tokens(L, inputs.bf16_bits(x), lg.numpy(), 2)
    gpu_support.check_out(out, ref, "mixed tables")


def test_forward_host_matches_device_forward():
    w = inputs.WORKLOADS["tiny"]
    _, dev = _small_device_layer(w)
    x = inputs.activations(w)
    lg = inputs.router_logits(w)
    out_f, *_ = _run(dev, x.cuda(), lg.cuda(), 2)
    out_d = out_f.to(torch.bfloat16)
    ws = q4.alloc_workspace(q4.forward_host_workspace(dev, 4, 2))
    out_h = torch.empty((4, 256), dtype=torch.bfloat16).pin_memory()
    st = q4.forward_host(dev, x.pin_memory(), lg.pin_memory(), 2, out_h, ws)
    assert st == 0
    assert torch.equal(out_h, out_d.cpu())


def test_forward_host_async_back_to_back_matches_device_forward():
    """Several moe_q4_forward_host_async calls enqueued back to back on one
    stream and workspace (different batches, different pinned outputs), the
    status read once at the end: each output equals the device forward's."""
    w = inputs.Workload("host_async", 20, 6, inputs.TINY)
    _, dev = _small_device_layer(w)
    xs = [inputs.activations(w, variant=v) for v in range(3)]
    lgs = [inputs.router_logits(w, variant=v) for v in range(3)]
    ws = q4.alloc_workspace(q4.forward_host_workspace(dev, 6, 2))
    outs = [torch.empty((6, 256), dtype=torch.bfloat16).pin_memory() for _ in range(3)]
    xp = [x.pin_memory() for x in xs]
    lp = [l.pin_memory() for l in lgs]
    for i in range(3):
        q4.forward_host_async(dev, xp[i], lp[i], 2, outs[i], ws)
    assert q4.forward_status(ws) == 0
    for i in range(3):
        ref = q4.forward(dev, xs[i].cuda(), lgs[i].cuda(), 2)
        torch.cuda.synchronize()
        assert torch.equal(outs[i], ref.cpu()), i


def test_non_finite_logit_reports_device_status():
    w = inputs.WORKLOADS["tiny"]
    _, dev = _small_device_layer(w)
    lg = inputs.router_logits(w).cuda()
    lg[2, 1] = float("inf")
    ws = q4.alloc_workspace(q4.forward_workspace(dev, 4, 2))
    q4.forward(dev, inputs.activations(w).cuda(), lg, 2, ws=ws)
    assert q4.forward_status(ws) == q4._lib.EDEVICE


def test_repeat_calls_are_deterministic():
    w = inputs.Workload("det", 11, 64, inputs.TINY)
    _, dev = _small_device_layer(w)
    x = inputs.activations(w).cuda()
    lg = inputs.router_logits(w).cuda()
    a, *_ = _run(dev, x, lg, 2)
    b, *_ = _run(dev, x, lg, 2)
    assert torch.equal(a, b)


# ---- GLM-shaped workloads -------------------------------------------------

def _glm_case(name, n_sample=None, must_hit=()):
    w = inputs.WORKLOADS[name]
    dev = gpu_support.device_layer(w)
    x = inputs.activations(w, device="cuda")
    lg = inputs.router_logits(w, device="cuda")
    k = w.shape.k
    out, ids, wts, counts = _run(dev, x, lg, k)
    lg_h = lg.cpu().numpy()
    x_bits = inputs.bf16_bits(x)
    ids_h = ids.cpu().numpy()
    rids, _ = oracle.route(lg_h, k)
    assert np.array_equal(ids_h, rids)  # full routing check at every size
    rc, *_ = oracle.group(rids, w.shape.E)
    assert np.array_equal(counts.cpu().numpy(), rc)
    if n_sample is None or n_sample >= w.T:
        tokens = list(range(w.T))
    else:
        rng = np.random.default_rng(1234 + w.index)
        tokens = set(rng.choice(w.T, n_sample, replace=False).tolist())
        for e in must_hit:  # include a token routed to each listed expert
            hit = np.nonzero((rids == e).any(1))[0]
            if hit.size:
                tokens.add(int(hit[0]))
        hottest = int(np.argmax(rc))
        tokens.add(int(np.nonzero((rids == hottest).any(1))[0][0]))
        tokens = sorted(tokens)
    experts = np.unique(rids[tokens])
    L = gpu_support.oracle_layer(w, experts, dev)
    ref = gpu_support.oracle_tokens(L, x_bits, lg_h, k, tokens)
    return gpu_support.check_out(out[tokens], ref, name)


def test_glm_decode_t1_full():
    _glm_case("decode_t1")


def test_glm_decode_t8_full():
    _glm_case("decode_t8")


def test_glm_decode_t64_sampled():
    _glm_case("decode_t64", n_sample=6)


def test_glm_prefill_t2048_sampled():
    _glm_case("prefill_t2048", n_sample=5)


def test_glm_prefill_t8192_mixed_sampled():
    _glm_case("prefill_t8192", n_sample=3, must_hit=inputs.E2M1_EXPERTS)
