"""The C-ABI library (no GPU needed): it loads, exports every symbol the
header declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import numpy as np
import pytest

import bit_codebook_quantized_router_b200 as q4
from bit_codebook_quantized_router_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_q4.h")


@pytest.fixture(scope="module")
def L():
    from bit_codebook_quantized_router_b200 import build
    build.build()
    return _lib.lib()


def declared_symbols():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"MOE_Q4_API\s+[\w\s\*]+?\b(moe_q4_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for s in ("moe_q4_pack", "moe_q4_dequant", "moe_q4_forward", "moe_q4_forward_workspace",
              "moe_q4_abi_version", "moe_q4_status_string", "moe_q4_route", "moe_q4_forward_host"):
        assert s in syms


def test_library_exports_every_declared_symbol(L):
    for s in declared_symbols():
        assert hasattr(L, s), s
    assert L.moe_q4_abi_version() == 1
    for code in range(8):
        assert L.moe_q4_status_string(code)


def _layer(E=8, H=256, I=128, tables=None, table_id=None, null=False):
    t = np.ascontiguousarray(tables if tables is not None else np.linspace(0.1, 2, 8, dtype=np.float32)[None])
    tid = np.ascontiguousarray(table_id if table_id is not None else np.zeros(E, np.uint8))
    fake = 0 if null else 1 << 20  # never dereferenced: validation fails first
    st = _lib._LayerStruct(E, H, I, fake, fake, fake, fake, fake, fake, t.ctypes.data, t.shape[0], tid.ctypes.data)
    return st, (t, tid)


def test_workspace_query_and_shape_validation(L):
    st, keep = _layer()
    assert L.moe_q4_forward_workspace(ctypes.byref(st), 4, 2) > 0
    assert L.moe_q4_forward_workspace(ctypes.byref(st), 4, 9) == 0  # k > E
    assert L.moe_q4_forward_workspace(ctypes.byref(st), -1, 2) == 0
    bad, keep2 = _layer(H=250)
    assert L.moe_q4_forward_workspace(ctypes.byref(bad), 4, 2) == 0  # H % 128
    nul, keep3 = _layer(null=True)
    assert L.moe_q4_forward_workspace(ctypes.byref(nul), 4, 2) == 0


def test_forward_rejects_bad_arguments_before_launch(L):
    st, keep = _layer()
    f = L.moe_q4_forward
    # top_k out of range
    assert f(ctypes.byref(st), 16, 16, 4, 0, 16, None, None, None, None, 256, 1 << 20, None) == _lib.EINVAL
    # null activations
    assert f(ctypes.byref(st), None, 16, 4, 2, 16, None, None, None, None, 256, 1 << 20, None) == _lib.EINVAL
    # workspace too small / misaligned
    assert f(ctypes.byref(st), 16, 16, 4, 2, 16, None, None, None, None, 256, 10, None) == _lib.EWORKSPACE
    assert f(ctypes.byref(st), 16, 16, 4, 2, 16, None, None, None, None, 100, 1 << 30, None) == _lib.EWORKSPACE
    # bad tables: NaN, negative, -0.0, all zero, table id out of range
    for tb in ([np.nan] + [1.0] * 7, [-1.0] + [1.0] * 7, [-0.0] + [1.0] * 7, [0.0] * 8):
        bt, k2 = _layer(tables=np.array([tb], np.float32))
        assert f(ctypes.byref(bt), 16, 16, 4, 2, 16, None, None, None, None, 256, 1 << 30, None) == _lib.EINVAL
    bt, k3 = _layer(table_id=np.full(8, 1, np.uint8))
    assert f(ctypes.byref(bt), 16, 16, 4, 2, 16, None, None, None, None, 256, 1 << 30, None) == _lib.EINVAL


def test_pack_dequant_reject_bad_shapes(L):
    t = np.linspace(0.1, 2, 8, dtype=np.float32)
    tid = np.zeros(2, np.uint8)
    # K % 32 != 0
    assert L.moe_q4_pack(16, 2, 4, 48, t.ctypes.data, 1, tid.ctypes.data, 16, 16, 16, None) == _lib.EINVAL
    assert L.moe_q4_dequant(16, 16, t.ctypes.data, 1, tid.ctypes.data, 2, 4, 48, 16, None) == _lib.EINVAL
    # too many tables
    assert L.moe_q4_dequant(16, 16, t.ctypes.data, 17, tid.ctypes.data, 2, 4, 64, 16, None) == _lib.EINVAL
    # empty is a no-op
    assert L.moe_q4_dequant(None, None, t.ctypes.data, 1, tid.ctypes.data, 0, 4, 64, None, None) == _lib.OK


def test_route_workspace_validation(L):
    assert L.moe_q4_route_workspace(256, 8, 8) > 0
    assert L.moe_q4_route_workspace(256, 8, 17) == 0
    assert L.moe_q4_route_workspace(600, 8, 8) == 0
    # past 256 tokens the grouping keeps each 256-token chunk's row counts and
    # first rows: two int32 [ceil(T/256)][E] arrays, 256-byte aligned
    base = L.moe_q4_route_workspace(256, 256, 8)
    assert L.moe_q4_route_workspace(256, 1, 8) == base
    assert L.moe_q4_route_workspace(256, 257, 8) == base + 2 * (2 * 256 * 4)
    assert L.moe_q4_route_workspace(256, 8192, 8) == base + 2 * (32 * 256 * 4)
    assert L.moe_q4_route_workspace(3, 300, 3) == L.moe_q4_route_workspace(3, 8, 3) + 2 * 256


def test_router_workspace_and_argument_validation(L):
    # decode sizes (T <= 32, H % 128 == 0) run as one kernel: no workspace
    assert L.moe_q4_router_workspace(1, 6144, 256) == 0
    assert L.moe_q4_router_workspace(32, 6144, 256) == 0
    # more tokens, or H not a multiple of 128: K-split partials in the workspace
    assert L.moe_q4_router_workspace(64, 6144, 256) > 0
    assert L.moe_q4_router_workspace(1, 6144 + 32, 256) > 0
    assert L.moe_q4_router_workspace(0, 6144, 256) == 0
    # invalid sizes: no workspace, and the call refuses before any launch
    assert L.moe_q4_router_workspace(1, 48, 8) == 0  # H % 32
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails first
    out = ctypes.c_void_p(1 << 21)
    assert L.moe_q4_router(fake, fake, 1, 48, 8, out, None, 0, None) == _lib.EINVAL
    assert L.moe_q4_router(fake, fake, 1, 64, 0, out, None, 0, None) == _lib.EINVAL
    assert L.moe_q4_router(fake, fake, -1, 64, 8, out, None, 0, None) == _lib.EINVAL
    assert L.moe_q4_router(None, fake, 1, 64, 8, out, None, 0, None) == _lib.EINVAL
    assert L.moe_q4_router(ctypes.c_void_p((1 << 20) + 8), fake, 1, 64, 8, out, None, 0, None) == _lib.EINVAL
    # T = 0 is a valid empty call
    assert L.moe_q4_router(None, None, 0, 64, 8, None, None, 0, None) == _lib.OK
    # a split K needs its workspace
    assert L.moe_q4_router(fake, fake, 64, 6144, 256, out, None, 0, None) == _lib.EWORKSPACE


def test_lloyd_host_checks(L):
    g = np.array([0.13, 0.39, 0.66, 0.94, 1.26, 1.62, 2.08, 2.75], np.float32)
    assert L.moe_q4_lloyd_workspace(g.ctypes.data) > 0
    for bad in (g[::-1].copy(), np.where(np.arange(8) == 2, g[1], g).astype(np.float32),
                np.concatenate([[-0.0], g[1:]]).astype(np.float32), (g * 8).astype(np.float32)):
        assert L.moe_q4_lloyd_workspace(np.ascontiguousarray(bad).ctypes.data) == 0
    assert L.moe_q4_lloyd_workspace(None) == 0
    ws_n = L.moe_q4_lloyd_workspace(g.ctypes.data)
    fake = ctypes.c_void_p(1 << 20)
    # a gmax of 16 or more is beyond the histogram of this build
    big = (g * 8).astype(np.float32)
    assert L.moe_q4_lloyd_hist(fake, 1, big.ctypes.data, 1, fake, ws_n, None) == _lib.ENOTSUP
    assert L.moe_q4_lloyd_hist(fake, -1, g.ctypes.data, 1, fake, ws_n, None) == _lib.EINVAL
    assert L.moe_q4_lloyd_hist(ctypes.c_void_p((1 << 20) + 2), 1, g.ctypes.data, 1, fake, ws_n, None) == _lib.EINVAL
    assert L.moe_q4_lloyd_hist(fake, 1, g.ctypes.data, 1, fake, ws_n - 8, None) == _lib.EWORKSPACE
    assert L.moe_q4_lloyd_hist(fake, 1, g.ctypes.data, 1, None, ws_n, None) == _lib.EWORKSPACE
    out = ctypes.c_void_p(1 << 21)
    assert L.moe_q4_lloyd_solve(g.ctypes.data, -1, 0.0, out, out, fake, ws_n, None) == _lib.EINVAL
    assert L.moe_q4_lloyd_solve(g.ctypes.data, 5, -1.0, out, out, fake, ws_n, None) == _lib.EINVAL
    assert L.moe_q4_lloyd_solve(g.ctypes.data, 5, 0.0, None, out, fake, ws_n, None) == _lib.EINVAL


def test_shared_expert_host_checks(L):
    st, keep = _layer()
    base = L.moe_q4_forward_workspace(ctypes.byref(st), 4, 2)
    assert L.moe_q4_forward_ex_workspace(ctypes.byref(st), None, 4, 2) == base
    ok = _lib._SharedStruct(128, 1 << 20, 1 << 21)
    assert L.moe_q4_forward_ex_workspace(ctypes.byref(st), ctypes.byref(ok), 4, 2) > base
    for bad in (_lib._SharedStruct(96, 1 << 20, 1 << 21), _lib._SharedStruct(128, 0, 1 << 21),
                _lib._SharedStruct(128, (1 << 20) + 8, 1 << 21), _lib._SharedStruct(0, 1 << 20, 1 << 21)):
        assert L.moe_q4_forward_ex_workspace(ctypes.byref(st), ctypes.byref(bad), 4, 2) == 0
        assert L.moe_q4_forward_ex(ctypes.byref(st), ctypes.byref(bad), None, None, 4, 2, None, None, None, None,
                                   None, None, 0, None) == _lib.EINVAL


def test_gated_forward_host_checks(L):
    st, keep = _layer()
    base = L.moe_q4_forward_workspace(ctypes.byref(st), 4, 2)
    gated = L.moe_q4_forward_gated_workspace(ctypes.byref(st), None, 4, 2)
    assert gated > base  # the logits (and any router partial sums) live in the workspace
    assert L.moe_q4_forward_gated_workspace(ctypes.byref(st), None, 4, 0) == 0
    fake = ctypes.c_void_p(1 << 20)
    f = L.moe_q4_forward_gated
    # no router gate, a misaligned gate, a misaligned logits buffer, a short workspace
    assert f(ctypes.byref(st), None, None, fake, 4, 2, fake, None, None, None, None, None, fake, gated,
             None) == _lib.EINVAL
    assert f(ctypes.byref(st), None, ctypes.c_void_p((1 << 20) + 2), fake, 4, 2, fake, None, None, None, None, None,
             fake, gated, None) == _lib.EINVAL
    assert f(ctypes.byref(st), None, fake, fake, 4, 2, fake, None, ctypes.c_void_p((1 << 20) + 2), None, None, None,
             fake, gated, None) == _lib.EINVAL
    assert f(ctypes.byref(st), None, fake, fake, 4, 2, fake, None, None, None, None, None, fake, gated - 256,
             None) == _lib.EWORKSPACE


def test_debug_build_exports_every_declared_symbol(L):
    from bit_codebook_quantized_router_b200 import build
    assert os.path.exists(build.LIB_DEBUG)
    D = ctypes.CDLL(build.LIB_DEBUG)
    for s in declared_symbols():
        assert hasattr(D, s), s
    D.moe_q4_status_string.restype = ctypes.c_char_p
    assert b"debug" in D.moe_q4_status_string(_lib.EBOUNDS)


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    # no CPU fallback: without the built library every entry raises
    from bit_codebook_quantized_router_b200 import _lib as binding
    monkeypatch.setattr(binding, "_lib", None)
    monkeypatch.setattr(binding, "LIB_PATH", str(tmp_path / "libmoe_q4.so"))
    with pytest.raises(ImportError, match="is missing"):
        binding.lib()
