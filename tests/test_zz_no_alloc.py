"""moe_q4_forward_noalloc: the layer forward for callers that cannot allocate
device memory (a serving loop that may not call cudaMalloc once running, or
code that only holds device pointers from another framework's allocator).  It
takes no workspace and uses the library's static 8 MiB scratch array instead.

The tests call it through the C ABI:
- twice in a row on different batches of the same size, each result checked
  against moe_q4_forward's on the same batch within the parity tolerance of
  the other layer tests;
- on a sequence of different sizes on one stream (T = 8, then 1, then 3):
  the array keeps the previous call's bytes, laid out for another T, so each
  result is checked against moe_q4_forward and, for T = 1 and T = 3, against
  the fp64 oracle's bounds;
- with T = 0 (the status word is still written) and with a size whose
  workspace exceeds the array (refused before anything runs).
This file is named to be collected last."""
import ctypes

import numpy as np
import pytest
import torch

import bit_codebook_quantized_router_b200 as q4
from bit_codebook_quantized_router_b200 import _lib, inputs
from tests import gpu_support

pytestmark = pytest.mark.gpu


def _noalloc_fn():
    fn = q4.lib().moe_q4_forward_noalloc
    vp, ci = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [ctypes.POINTER(_lib._LayerStruct), vp, vp, ci, ci, vp, vp, vp, vp]
    fn.restype = ci
    return fn


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check_close(got_f32, ref_f32, what):
    g = got_f32.cpu().numpy().astype(np.float64)
    r = ref_f32.cpu().numpy().astype(np.float64)
    rel = np.linalg.norm(g - r) / np.linalg.norm(r)
    mx = np.abs(g - r).max() / np.sqrt(np.mean(r * r))
    assert rel <= gpu_support.REL_FRO and mx <= gpu_support.MAX_ABS_RMS, (what, rel, mx)


def _call(fn, layer_struct, x, lg, T, k, out, out32, status):
    stream = torch.cuda.current_stream()
    rc = fn(ctypes.byref(layer_struct), _ptr(x), _ptr(lg), T, k, _ptr(out), _ptr(out32), _ptr(status),
            ctypes.c_void_p(stream.cuda_stream))
    assert rc == _lib.OK, q4.status_string(rc)


def _outputs(T, H):
    return (torch.empty((T, H), dtype=torch.bfloat16, device="cuda"),
            torch.empty((T, H), dtype=torch.float32, device="cuda"),
            torch.full((1,), -1, dtype=torch.int32, device="cuda"))


def test_noalloc_matches_forward_on_two_calls_in_a_row():
    w = inputs.WORKLOADS["decode_t8"]
    layer = gpu_support.device_layer(w)
    T, k, H = w.T, w.shape.k, w.shape.H
    fn = _noalloc_fn()
    batches = [(inputs.activations(w, device="cuda", variant=v), inputs.router_logits(w, device="cuda", variant=v))
               for v in (3, 4)]
    outs = [_outputs(T, H) for _ in batches]
    st = layer.struct()
    # two calls in a row on one stream; the second must not see the first's leftovers
    for (x, lg), (out, out32, status) in zip(batches, outs):
        _call(fn, st, x, lg, T, k, out, out32, status)
    torch.cuda.synchronize()
    for i, ((x, lg), (out, out32, status)) in enumerate(zip(batches, outs)):
        assert int(status.item()) == _lib.OK
        ref32 = torch.empty((T, H), dtype=torch.float32, device="cuda")
        ref = q4.forward(layer, x, lg, k, out_f32=ref32)
        torch.cuda.synchronize()
        _check_close(out32, ref32, f"call {i}")
        _check_close(out.float(), ref.float(), f"call {i} bf16")
        gpu_support.check_bf16_is_rounding(out, out32)


def test_noalloc_sequence_of_sizes_matches_forward_and_oracle():
    w = inputs.WORKLOADS["decode_t8"]
    layer = gpu_support.device_layer(w)
    k, H = w.shape.k, w.shape.H
    fn = _noalloc_fn()
    st = layer.struct()
    sizes = (8, 1, 3)
    batches = [(inputs.activations(w, device="cuda", T=T, variant=5 + i),
                inputs.router_logits(w, device="cuda", T=T, variant=5 + i)) for i, T in enumerate(sizes)]
    outs = [_outputs(T, H) for T in sizes]
    # all three enqueued back to back on one stream, no host wait between them
    for T, (x, lg), (out, out32, status) in zip(sizes, batches, outs):
        _call(fn, st, x, lg, T, k, out, out32, status)
    torch.cuda.synchronize()
    for T, (x, lg), (out, out32, status) in zip(sizes, batches, outs):
        assert int(status.item()) == _lib.OK, T
        ref32 = torch.empty((T, H), dtype=torch.float32, device="cuda")
        q4.forward(layer, x, lg, k, out_f32=ref32)
        torch.cuda.synchronize()
        _check_close(out32, ref32, f"T={T} vs forward")
        gpu_support.check_bf16_is_rounding(out, out32)
        if T <= 3:
            lg_h = lg.cpu().numpy()
            rids, _ = gpu_support.oracle.route(lg_h, k)
            L = gpu_support.oracle_layer(w, np.unique(rids), layer)
            ref = gpu_support.oracle_tokens(L, inputs.bf16_bits(x), lg_h, k, range(T))
            gpu_support.check_out(out32, ref, f"T={T} vs oracle")


def test_noalloc_zero_tokens_writes_ok_status():
    w = inputs.WORKLOADS["decode_t8"]
    layer = gpu_support.device_layer(w)
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    rc = _noalloc_fn()(ctypes.byref(layer.struct()), None, None, 0, w.shape.k, None, None, _ptr(status),
                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == _lib.OK
    torch.cuda.synchronize()
    assert int(status.item()) == _lib.OK


@pytest.mark.parametrize("T", [10, 24])
def test_noalloc_refuses_sizes_beyond_its_scratch(T):
    w = inputs.WORKLOADS["decode_t8"]
    layer = gpu_support.device_layer(w)
    k, H = w.shape.k, w.shape.H  # the GLM shape admits T <= 9 (T = 10 needs 8.86 MiB, T = 24 16.9 MB)
    x = torch.zeros((T, H), dtype=torch.bfloat16, device="cuda")
    lg = torch.zeros((T, w.shape.E), dtype=torch.float32, device="cuda")
    out = torch.full((T, H), 7.0, dtype=torch.bfloat16, device="cuda")
    st = layer.struct()
    rc = _noalloc_fn()(ctypes.byref(st), _ptr(x), _ptr(lg), T, k, _ptr(out), None, None,
                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == _lib.ENOTSUP
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)
