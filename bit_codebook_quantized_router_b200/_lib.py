"""ctypes binding of libmoe_q4 (argument marshalling only: every step of the
layer runs in the library's CUDA kernels).  Torch provides device memory and
streams; tensors are passed as raw pointers."""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# MOE_Q4_LIB=debug selects the bounds-checking build (libmoe_q4_debug.so)
LIB_PATH = os.path.join(_HERE, "libmoe_q4_debug.so" if os.environ.get("MOE_Q4_LIB") == "debug" else "libmoe_q4.so")

OK, EINVAL, ECUDA, EWORKSPACE, ETIMEOUT, EDEVICE, ENOTSUP, EBOUNDS = range(8)
MAX_TABLES, MAX_EXPERTS, MAX_TOPK = 16, 512, 16


class MoeQ4Error(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: moe_q4 status {status} ({status_string(status)})")


class _SharedStruct(ctypes.Structure):
    _fields_ = [("I", ctypes.c_int), ("gate_up", ctypes.c_void_p), ("down", ctypes.c_void_p)]


class _LayerStruct(ctypes.Structure):
    _fields_ = [
        ("E", ctypes.c_int), ("H", ctypes.c_int), ("I", ctypes.c_int),
        ("gate_w", ctypes.c_void_p), ("gate_s", ctypes.c_void_p),
        ("up_w", ctypes.c_void_p), ("up_s", ctypes.c_void_p),
        ("down_w", ctypes.c_void_p), ("down_s", ctypes.c_void_p),
        ("tables", ctypes.c_void_p), ("n_tables", ctypes.c_int), ("table_id", ctypes.c_void_p),
    ]


_lib = None


def lib():
    """The loaded library.  Raises if it was not built: there is no fallback."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m bit_codebook_quantized_router_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, ci, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        L.moe_q4_abi_version.restype = ci
        L.moe_q4_status_string.argtypes = [ci]
        L.moe_q4_status_string.restype = ctypes.c_char_p
        L.moe_q4_pack.argtypes = [vp, ci, ci, ci, vp, ci, vp, vp, vp, vp, vp]
        L.moe_q4_dequant.argtypes = [vp, vp, vp, ci, vp, ci, ci, ci, vp, vp]
        L.moe_q4_forward_workspace.argtypes = [ctypes.POINTER(_LayerStruct), ci, ci]
        L.moe_q4_forward_workspace.restype = sz
        L.moe_q4_forward_host_workspace.argtypes = [ctypes.POINTER(_LayerStruct), ci, ci]
        L.moe_q4_forward_host_workspace.restype = sz
        L.moe_q4_forward.argtypes = [ctypes.POINTER(_LayerStruct), vp, vp, ci, ci, vp, vp, vp, vp, vp, vp, sz, vp]
        L.moe_q4_forward_host.argtypes = [ctypes.POINTER(_LayerStruct), vp, vp, ci, ci, vp, vp, sz, vp]
        L.moe_q4_forward_status.argtypes = [vp, vp]
        L.moe_q4_read_status.argtypes = [vp, vp]
        L.moe_q4_route_workspace.argtypes = [ci, ci, ci]
        L.moe_q4_route_workspace.restype = sz
        L.moe_q4_route.argtypes = [vp, ci, ci, ci, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.moe_q4_forward_stages.argtypes = [ctypes.POINTER(_LayerStruct), vp, vp, ci, ci, vp, vp, sz, vp,
                                            ctypes.POINTER(ctypes.c_void_p), ci]
        L.moe_q4_router_workspace.argtypes = [ci, ci, ci]
        L.moe_q4_router_workspace.restype = sz
        L.moe_q4_router.argtypes = [vp, vp, ci, ci, ci, vp, vp, sz, vp]
        L.moe_q4_forward_ex_workspace.argtypes = [ctypes.POINTER(_LayerStruct), ctypes.POINTER(_SharedStruct), ci, ci]
        L.moe_q4_forward_ex_workspace.restype = sz
        L.moe_q4_forward_ex.argtypes = [ctypes.POINTER(_LayerStruct), ctypes.POINTER(_SharedStruct), vp, vp, ci, ci,
                                        vp, vp, vp, vp, vp, vp, sz, vp]
        L.moe_q4_forward_ex.restype = ci
        L.moe_q4_forward_gated_workspace.argtypes = [ctypes.POINTER(_LayerStruct), ctypes.POINTER(_SharedStruct),
                                                     ci, ci]
        L.moe_q4_forward_gated_workspace.restype = sz
        L.moe_q4_forward_gated.argtypes = [ctypes.POINTER(_LayerStruct), ctypes.POINTER(_SharedStruct), vp, vp, ci,
                                           ci, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.moe_q4_forward_gated.restype = ci
        L.moe_q4_combine.argtypes = [vp, vp, vp, ci, ci, ci, vp, vp, vp]
        L.moe_q4_combine.restype = ci
        L.moe_q4_selftest_wait.argtypes = [vp, ctypes.c_uint, vp]
        L.moe_q4_selftest_wait.restype = ci
        L.moe_q4_lloyd_workspace.argtypes = [vp]
        L.moe_q4_lloyd_workspace.restype = sz
        L.moe_q4_lloyd_hist.argtypes = [vp, ctypes.c_longlong, vp, ci, vp, sz, vp]
        L.moe_q4_lloyd_solve.argtypes = [vp, ci, ctypes.c_double, vp, vp, vp, sz, vp]
        L.moe_q4_forward_host_async.argtypes = L.moe_q4_forward_host.argtypes
        for f in (L.moe_q4_pack, L.moe_q4_dequant, L.moe_q4_forward, L.moe_q4_forward_host,
                  L.moe_q4_forward_host_async,
                  L.moe_q4_forward_status, L.moe_q4_read_status, L.moe_q4_route,
                  L.moe_q4_forward_stages, L.moe_q4_router, L.moe_q4_lloyd_hist, L.moe_q4_lloyd_solve):
            f.restype = ci
        if L.moe_q4_abi_version() != 1:
            raise ImportError("libmoe_q4 ABI version mismatch")
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().moe_q4_status_string(int(status)).decode()


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _hold(stream, *tensors):
    """Memory this binding allocated for a call (contiguous copies, internal
    workspaces) is read by work enqueued on `stream`, which may run after the
    call returns: when that is not torch's current stream, tell the caching
    allocator, so the blocks are not handed out again before the work ran.
    (On the current stream, stream order already keeps reuse safe.)"""
    if stream is None:
        return
    for t in tensors:
        if t is not None and t.is_cuda:
            t.record_stream(stream)


def _check(rc, what):
    if rc != OK:
        raise MoeQ4Error(rc, what)


def _host_tables(tables, table_id, E):
    t = np.ascontiguousarray(np.asarray(tables, np.float32).reshape(-1, 8))
    tid = np.ascontiguousarray(np.asarray(table_id, np.uint8).reshape(-1))
    if tid.shape[0] != E:
        raise ValueError("table_id must hold one entry per expert")
    return t, tid


class Layer:
    """A packed layer resident on the device.

    gate_w/up_w: uint8 [E, I, H/2], gate_s/up_s: uint8 [E, I, H/32],
    down_w: uint8 [E, H, I/2], down_s: uint8 [E, H, I/32] (CUDA tensors);
    tables: fp32 [n, 8] magnitudes; table_id: uint8 [E] (host arrays)."""

    def __init__(self, gate_w, gate_s, up_w, up_s, down_w, down_s, tables, table_id):
        self.E, self.I, hh = gate_w.shape
        self.H = hh * 2
        self.gate_w, self.gate_s, self.up_w, self.up_s = gate_w, gate_s, up_w, up_s
        self.down_w, self.down_s = down_w, down_s
        self.tables, self.table_id = _host_tables(tables, table_id, self.E)
        for t in (gate_w, gate_s, up_w, up_s, down_w, down_s):
            if not (t.is_cuda and t.dtype == torch.uint8 and t.is_contiguous()):
                raise ValueError("packed tensors must be contiguous uint8 CUDA tensors")

    def struct(self) -> _LayerStruct:
        return _LayerStruct(self.E, self.H, self.I,
                            self.gate_w.data_ptr(), self.gate_s.data_ptr(),
                            self.up_w.data_ptr(), self.up_s.data_ptr(),
                            self.down_w.data_ptr(), self.down_s.data_ptr(),
                            self.tables.ctypes.data, self.tables.shape[0], self.table_id.ctypes.data)


def pack(w: torch.Tensor, tables, table_id, status: torch.Tensor | None = None, stream=None):
    """bf16 [E, N, K] CUDA tensor -> (codes uint8 [E, N, K/2], scales uint8 [E, N, K/32])."""
    if w.dim() != 3 or w.dtype != torch.bfloat16 or not w.is_cuda:
        raise ValueError("w must be a bf16 CUDA tensor [E, N, K]")
    w = w.contiguous()
    E, N, K = w.shape
    t, tid = _host_tables(tables, table_id, E)
    codes = torch.empty((E, N, K // 2), dtype=torch.uint8, device=w.device)
    scales = torch.empty((E, N, K // 32), dtype=torch.uint8, device=w.device)
    own = status is None
    if own:
        status = torch.zeros(1, dtype=torch.int32, device=w.device)
    _check(lib().moe_q4_pack(_ptr(w), E, N, K, t.ctypes.data, t.shape[0], tid.ctypes.data,
                             _ptr(codes), _ptr(scales), _ptr(status), _stream(stream)), "moe_q4_pack")
    _hold(stream, w, status)
    if own:
        st = lib().moe_q4_read_status(_ptr(status), _stream(stream))
        _check(st, "moe_q4_pack (device)")
    return codes, scales


def dequant(codes: torch.Tensor, scales: torch.Tensor, tables, table_id, stream=None,
            out: torch.Tensor | None = None) -> torch.Tensor:
    """uint8 codes [E, N, K/2] + scales [E, N, K/32] -> bf16 [E, N, K] (into `out` if given)."""
    E, N, Kh = codes.shape
    K = Kh * 2
    t, tid = _host_tables(tables, table_id, E)
    if out is None:
        out = torch.empty((E, N, K), dtype=torch.bfloat16, device=codes.device)
    elif out.shape != (E, N, K) or out.dtype != torch.bfloat16 or not out.is_contiguous():
        raise ValueError("out must be a contiguous bf16 tensor [E, N, K]")
    codes, scales = codes.contiguous(), scales.contiguous()
    _check(lib().moe_q4_dequant(_ptr(codes), _ptr(scales), t.ctypes.data,
                                t.shape[0], tid.ctypes.data, E, N, K, _ptr(out), _stream(stream)),
           "moe_q4_dequant")
    _hold(stream, codes, scales)
    return out


def forward_workspace(layer: Layer, T: int, k: int) -> int:
    return int(lib().moe_q4_forward_workspace(ctypes.byref(layer.struct()), T, k))


def forward_host_workspace(layer: Layer, T: int, k: int) -> int:
    return int(lib().moe_q4_forward_host_workspace(ctypes.byref(layer.struct()), T, k))


def alloc_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def forward(layer: Layer, x: torch.Tensor, logits: torch.Tensor, k: int, out=None, ws=None,
            topk_ids=None, topk_w=None, counts=None, out_f32=None, stream=None) -> torch.Tensor:
    """One MoE layer: x bf16 [T, H], logits fp32 [T, E] -> out bf16 [T, H]
    (and, when given, the fp32 combine result in out_f32 [T, H])."""
    T = x.shape[0]
    if out is None:
        out = torch.empty((T, layer.H), dtype=torch.bfloat16, device=x.device)
    own_ws = ws is None
    if own_ws:
        ws = alloc_workspace(forward_workspace(layer, T, k), x.device)
    st = layer.struct()
    _check(lib().moe_q4_forward(ctypes.byref(st), _ptr(x), _ptr(logits), T, k, _ptr(out),
                                _ptr(out_f32), _ptr(topk_ids), _ptr(topk_w), _ptr(counts), _ptr(ws), ws.numel(),
                                _stream(stream)), "moe_q4_forward")
    if own_ws:
        _hold(stream, ws)
    return out


class Shared:
    """A BF16 shared expert: gate_up bf16 [2I, H] (gate rows first), down
    bf16 [H, I] (CUDA tensors)."""

    def __init__(self, gate_up: torch.Tensor, down: torch.Tensor):
        if gate_up.dtype != torch.bfloat16 or down.dtype != torch.bfloat16 or not (gate_up.is_cuda and down.is_cuda):
            raise ValueError("shared expert weights must be bf16 CUDA tensors")
        if gate_up.dim() != 2 or down.dim() != 2 or gate_up.shape[0] % 2 or down.shape != (gate_up.shape[1],
                                                                                          gate_up.shape[0] // 2):
            raise ValueError("shared expert shapes: gate_up [2I, H], down [H, I]")
        self.gate_up, self.down = gate_up.contiguous(), down.contiguous()
        self.I = gate_up.shape[0] // 2

    def struct(self) -> _SharedStruct:
        return _SharedStruct(self.I, self.gate_up.data_ptr(), self.down.data_ptr())


def forward_ex_workspace(layer: Layer, shared, T: int, k: int) -> int:
    sh = ctypes.byref(shared.struct()) if shared is not None else None
    return int(lib().moe_q4_forward_ex_workspace(ctypes.byref(layer.struct()), sh, T, k))


def forward_ex(layer: Layer, shared, x: torch.Tensor, logits: torch.Tensor, k: int, out=None, ws=None,
               topk_ids=None, topk_w=None, counts=None, out_f32=None, stream=None) -> torch.Tensor:
    """One MoE layer with a shared expert (shared may be None)."""
    T = x.shape[0]
    if out is None:
        out = torch.empty((T, layer.H), dtype=torch.bfloat16, device=x.device)
    own_ws = ws is None
    if own_ws:
        ws = alloc_workspace(forward_ex_workspace(layer, shared, T, k), x.device)
    st = layer.struct()
    ss = shared.struct() if shared is not None else None
    _check(lib().moe_q4_forward_ex(ctypes.byref(st), ctypes.byref(ss) if ss is not None else None, _ptr(x),
                                   _ptr(logits), T, k, _ptr(out), _ptr(out_f32), _ptr(topk_ids), _ptr(topk_w),
                                   _ptr(counts), _ptr(ws), ws.numel(), _stream(stream)), "moe_q4_forward_ex")
    if own_ws:
        _hold(stream, ws)
    return out


def forward_gated_workspace(layer: Layer, shared, T: int, k: int) -> int:
    sh = ctypes.byref(shared.struct()) if shared is not None else None
    return int(lib().moe_q4_forward_gated_workspace(ctypes.byref(layer.struct()), sh, T, k))


def forward_gated(layer: Layer, shared, router_w: torch.Tensor, x: torch.Tensor, k: int, out=None, ws=None,
                  logits=None, topk_ids=None, topk_w=None, counts=None, out_f32=None, stream=None) -> torch.Tensor:
    """One MoE layer from the hidden states: the bf16 router gate router_w
    [E, H] computes the logits (into `logits` [T, E] fp32 when given), then
    the layer as forward_ex (shared may be None)."""
    if router_w.dtype != torch.bfloat16 or tuple(router_w.shape) != (layer.E, layer.H):
        raise ValueError(f"router_w must be bf16 [{layer.E}, {layer.H}]")
    T = x.shape[0]
    if out is None:
        out = torch.empty((T, layer.H), dtype=torch.bfloat16, device=x.device)
    own_ws = ws is None
    if own_ws:
        ws = alloc_workspace(forward_gated_workspace(layer, shared, T, k), x.device)
    st = layer.struct()
    ss = shared.struct() if shared is not None else None
    _check(lib().moe_q4_forward_gated(ctypes.byref(st), ctypes.byref(ss) if ss is not None else None,
                                      _ptr(router_w), _ptr(x), T, k, _ptr(out), _ptr(out_f32), _ptr(logits),
                                      _ptr(topk_ids), _ptr(topk_w), _ptr(counts), _ptr(ws), ws.numel(),
                                      _stream(stream)), "moe_q4_forward_gated")
    if own_ws:
        _hold(stream, ws)
    return out


def forward_status(ws: torch.Tensor, stream=None) -> int:
    return int(lib().moe_q4_forward_status(_ptr(ws), _stream(stream)))


def forward_host(layer: Layer, x_host: torch.Tensor, logits_host: torch.Tensor, k: int,
                 out_host: torch.Tensor, ws: torch.Tensor, stream=None) -> int:
    """Host tensors in and out (pinned memory for asynchronous copies)."""
    T = x_host.shape[0]
    st = layer.struct()
    return int(lib().moe_q4_forward_host(ctypes.byref(st), _ptr(x_host), _ptr(logits_host), T, k,
                                         _ptr(out_host), _ptr(ws), ws.numel(), _stream(stream)))


def forward_host_async(layer: Layer, x_host: torch.Tensor, logits_host: torch.Tensor, k: int,
                       out_host: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
    """forward_host without the wait (pinned host tensors; read the device
    status later with forward_status on the same stream)."""
    T = x_host.shape[0]
    st = layer.struct()
    _check(lib().moe_q4_forward_host_async(ctypes.byref(st), _ptr(x_host), _ptr(logits_host), T, k,
                                           _ptr(out_host), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_q4_forward_host_async")


def route(logits: torch.Tensor, k: int, stream=None):
    """Routing + grouping alone: (ids, w, counts, offsets, row_token, inv)."""
    T, E = logits.shape
    dev = logits.device
    ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    row_token = torch.empty(T * k, dtype=torch.int32, device=dev)
    inv = torch.empty((T, k), dtype=torch.int32, device=dev)
    need = int(lib().moe_q4_route_workspace(E, T, k))
    if need == 0:
        raise MoeQ4Error(EINVAL, "moe_q4_route_workspace")
    ws = alloc_workspace(need, dev)
    logits = logits.contiguous()
    _check(lib().moe_q4_route(_ptr(logits), T, E, k, _ptr(ids), _ptr(w), _ptr(counts),
                              _ptr(offsets), _ptr(row_token), _ptr(inv), _ptr(ws), ws.numel(),
                              _stream(stream)), "moe_q4_route")
    _hold(stream, logits, ws)
    st = forward_status(ws, stream)
    return ids, w, counts, offsets, row_token, inv, st


def router_workspace(T: int, H: int, E: int) -> int:
    return int(lib().moe_q4_router_workspace(T, H, E))


def router(x: torch.Tensor, w: torch.Tensor, out: torch.Tensor | None = None, ws: torch.Tensor | None = None,
           stream=None) -> torch.Tensor:
    """Router logits: bf16 hidden states x [T, H] and bf16 gate w [E, H] ->
    fp32 logits [T, E] (into `out` if given)."""
    if x.dtype != torch.bfloat16 or w.dtype != torch.bfloat16 or x.dim() != 2 or w.dim() != 2:
        raise ValueError("x [T, H] and w [E, H] must be bf16 matrices")
    T, H = x.shape
    E = w.shape[0]
    if out is None:
        out = torch.empty((T, E), dtype=torch.float32, device=x.device)
    need = router_workspace(T, H, E)
    own_ws = ws is None and need > 0
    if own_ws:
        ws = alloc_workspace(need, x.device)
    x, w = x.contiguous(), w.contiguous()
    _check(lib().moe_q4_router(_ptr(x), _ptr(w), T, H, E, _ptr(out), _ptr(ws),
                               0 if ws is None else ws.numel(), _stream(stream)), "moe_q4_router")
    _hold(stream, x, w, ws if own_ws else None)
    return out


def forward_stages(layer: Layer, x, logits, k: int, out, ws, events, stream=None) -> None:
    """moe_q4_forward with torch.cuda.Event records at the 8 kernel boundaries
    (the events must have been recorded once: torch creates them lazily)."""
    arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    st = layer.struct()
    _check(lib().moe_q4_forward_stages(ctypes.byref(st), _ptr(x), _ptr(logits), x.shape[0], k, _ptr(out),
                                       _ptr(ws), ws.numel(), _stream(stream), arr, len(events)),
           "moe_q4_forward_stages")


def lloyd_fit(weights, grid0, max_iter: int = 300, tol: float = 1e-12, stream=None):
    """Weighted Lloyd-Max fit of an 8-level grid over the pooled ratios of one
    or more bf16 CUDA tensors (each a whole number of 32-weight blocks along
    its last dimension).  Returns (grid fp32 CUDA [8], iters int32 CUDA [1],
    status)."""
    if isinstance(weights, torch.Tensor):
        weights = [weights]
    g0 = np.ascontiguousarray(np.asarray(grid0, np.float32).reshape(8))
    need = int(lib().moe_q4_lloyd_workspace(g0.ctypes.data))
    if need == 0:
        raise MoeQ4Error(EINVAL, "moe_q4_lloyd_workspace")
    dev = weights[0].device
    ws = alloc_workspace(need, dev)
    for i, w in enumerate(weights):
        if w.dtype != torch.bfloat16 or not w.is_cuda or w.numel() % 32:
            raise ValueError("weights must be bf16 CUDA tensors holding whole 32-weight blocks")
        w = w.contiguous()
        _check(lib().moe_q4_lloyd_hist(_ptr(w), w.numel() // 32, g0.ctypes.data, 1 if i == 0 else 0, _ptr(ws),
                                       ws.numel(), _stream(stream)), "moe_q4_lloyd_hist")
        _hold(stream, w)
    grid = torch.empty(8, dtype=torch.float32, device=dev)
    iters = torch.empty(1, dtype=torch.int32, device=dev)
    _check(lib().moe_q4_lloyd_solve(g0.ctypes.data, int(max_iter), float(tol), _ptr(grid), _ptr(iters), _ptr(ws),
                                    ws.numel(), _stream(stream)), "moe_q4_lloyd_solve")
    _hold(stream, ws)
    status = int(lib().moe_q4_read_status(_ptr(ws), _stream(stream)))
    return grid, iters, status


def combine(y: torch.Tensor, w: torch.Tensor, inv=None, out=None, out_f32=None, stream=None) -> torch.Tensor:
    """Weighted combine: y fp32 [T*k, H] (rows in (token, slot) order unless
    inv [T, k] places them), w fp32 [T, k] -> bf16 [T, H]."""
    T, k = w.shape
    H = y.shape[1]
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=y.device)
    y, w = y.contiguous(), w.contiguous()
    _check(lib().moe_q4_combine(_ptr(y), _ptr(w), _ptr(inv), T, k, H, _ptr(out), _ptr(out_f32), _stream(stream)),
           "moe_q4_combine")
    _hold(stream, y, w)
    return out
