"""The bounds-checking debug build (libmoe_q4_debug.so, MOE_Q4_DEBUG): the
same forward through its C ABI gives the release build's bits and a clean
status (no device index check fails on valid inputs), on the tiny layer, the
small-M and tensor-core paths of a small layer, the wide tensor-core tiles of
a layer whose I and H are multiples of 256, and the GLM decode layer."""
import ctypes

import pytest
import torch

import bit_codebook_quantized_router_b200 as q4
from bit_codebook_quantized_router_b200 import _lib, build, inputs
from tests import gpu_support
from tests.test_gpu_forward import _small_device_layer

pytestmark = pytest.mark.gpu


def _debug_lib():
    L = ctypes.CDLL(build.LIB_DEBUG)
    vp, ci, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    L.moe_q4_forward.argtypes = [ctypes.POINTER(_lib._LayerStruct), vp, vp, ci, ci, vp, vp, vp, vp, vp, vp, sz, vp]
    L.moe_q4_forward.restype = ci
    L.moe_q4_forward_status.argtypes = [vp, vp]
    L.moe_q4_forward_status.restype = ci
    return L


def _both(dev, x, lg, k):
    T = x.shape[0]
    ref = torch.empty((T, dev.H), dtype=torch.float32, device="cuda")
    q4.forward(dev, x, lg, k, out_f32=ref)
    Ld = _debug_lib()
    ws = q4.alloc_workspace(q4.forward_workspace(dev, T, k))
    out = torch.empty((T, dev.H), dtype=torch.bfloat16, device="cuda")
    got = torch.empty((T, dev.H), dtype=torch.float32, device="cuda")
    st = dev.struct()
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = Ld.moe_q4_forward(ctypes.byref(st), ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(lg.data_ptr()), T, k,
                           ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(got.data_ptr()), None, None, None,
                           ctypes.c_void_p(ws.data_ptr()), ws.numel(), s)
    assert rc == _lib.OK
    assert Ld.moe_q4_forward_status(ctypes.c_void_p(ws.data_ptr()), s) == _lib.OK
    torch.cuda.synchronize()
    return got, ref


@pytest.mark.parametrize("T,k", [(4, 2), (1, 2), (16, 3), (300, 2)])
def test_debug_build_matches_release_on_small_layers(T, k):
    w = inputs.Workload("dbg", 17, T, inputs.TINY)
    _, dev = _small_device_layer(w)
    got, ref = _both(dev, inputs.activations(w).cuda(), inputs.router_logits(w).cuda(), k)
    assert torch.equal(got, ref)


@pytest.mark.parametrize("T,k", [(100, 2), (300, 3)])
def test_debug_build_matches_release_on_wide_tiles(T, k):
    w = inputs.Workload("dbg_wide", 19, T, inputs.Shape(H=512, I=256, E=8, k=k))
    _, dev = _small_device_layer(w)
    got, ref = _both(dev, inputs.activations(w).cuda(), inputs.router_logits(w).cuda(), k)
    assert torch.equal(got, ref)


def test_debug_build_matches_release_on_glm_decode():
    w = inputs.WORKLOADS["decode_t8"]
    dev = gpu_support.device_layer(w)
    got, ref = _both(dev, inputs.activations(w, device="cuda"), inputs.router_logits(w, device="cuda"), w.shape.k)
    assert torch.equal(got, ref)
