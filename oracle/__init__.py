"""moe_q4 oracle -- TEST INFRASTRUCTURE ONLY.

ctypes wrapper around ``moe_q4_oracle.c``: a plain single-threaded fp64 CPU
restatement of the routed-expert MoE over 4-bit codebook weights (decode,
pack, top-k routing, expert grouping, the layer, the router gate and the
weighted Lloyd-Max grid fit).  Only ``tests/``, the
package's ``smoke()`` check and ``bench.py``'s CPU-baseline leg may import
this module.  It shares no code with the CUDA library.

Each function cites the passage it follows in the C source.  The pins that
tie it to the pages and to mathematics live in ``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_q4_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_q4_oracle.so")

OQ_OK = 0
OQ_EINVAL = 1


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
             "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


class _Layer(ctypes.Structure):
    _fields_ = [
        ("E", ctypes.c_int), ("H", ctypes.c_int), ("I", ctypes.c_int),
        ("gate_w", ctypes.POINTER(ctypes.c_void_p)), ("gate_s", ctypes.POINTER(ctypes.c_void_p)),
        ("up_w", ctypes.POINTER(ctypes.c_void_p)), ("up_s", ctypes.POINTER(ctypes.c_void_p)),
        ("down_w", ctypes.POINTER(ctypes.c_void_p)), ("down_s", ctypes.POINTER(ctypes.c_void_p)),
        ("tables", ctypes.c_void_p), ("n_tables", ctypes.c_int), ("table_id", ctypes.c_void_p),
    ]


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        vp, ci = ctypes.c_void_p, ctypes.c_int
        L.oq_abi_version.restype = ci
        L.oq_decode_bf16.argtypes = [ctypes.c_uint8, ctypes.c_uint8, vp]
        L.oq_decode_bf16.restype = ctypes.c_uint16
        L.oq_dequant.argtypes = [vp, vp, vp, ci, vp, ci, ci, ci, vp]
        L.oq_decode_matrix_f64.argtypes = [vp, vp, vp, ci, ci, vp]
        L.oq_pack.argtypes = [vp, ci, ci, ci, vp, ci, vp, vp, vp]
        L.oq_route.argtypes = [vp, ci, ci, ci, vp, vp]
        L.oq_router_logits.argtypes = [vp, vp, ci, ci, ci, vp, vp]
        L.oq_group.argtypes = [vp, ci, ci, ci, vp, vp, vp, vp]
        L.oq_moe_tokens.argtypes = [ctypes.POINTER(_Layer), vp, vp, ci, ci, vp, vp, vp]
        L.oq_expert_partial.argtypes = [ctypes.POINTER(_Layer), ci, vp, ci, ci, vp]
        L.oq_lloyd_fit.argtypes = [vp, ctypes.c_longlong, vp, ci, ctypes.c_double, vp, vp]
        L.oq_shared_ffn.argtypes = [vp, ci, ci, vp, vp, ci, vp]
        for f in (L.oq_dequant, L.oq_decode_matrix_f64, L.oq_pack, L.oq_route, L.oq_group, L.oq_moe_tokens,
                  L.oq_expert_partial, L.oq_router_logits, L.oq_lloyd_fit):
            f.restype = ci
        _lib = L
    return _lib


class OracleError(ValueError):
    pass


def _p(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _check(rc):
    if rc != OQ_OK:
        raise OracleError(f"oracle status {rc}")


def _tables(tables):
    t = _c(tables, np.float32).reshape(-1, 8)
    return t, t.shape[0]


def decode_bf16(code: int, scale: int, table8) -> int:
    """bf16 bit pattern of one weight (fp32 multiply, RNE to bf16, sign flip)."""
    t = _c(table8, np.float32)
    return int(lib().oq_decode_bf16(code, scale, _p(t)))


def dequant(weight, weight_scale, tables, table_id, E, N, K):
    """[E][N][K] bf16 bit patterns (uint16) of packed projections."""
    w, s = _c(weight, np.uint8), _c(weight_scale, np.uint8)
    t, nt = _tables(tables)
    tid = _c(table_id, np.uint8)
    out = np.empty((E, N, K), np.uint16)
    _check(lib().oq_dequant(_p(w), _p(s), _p(t), nt, _p(tid), E, N, K, _p(out)))
    return out


def decode_matrix_f64(weight, weight_scale, table8, N, K):
    """Exact fp64 values of one packed [N][K] projection."""
    w, s, t = _c(weight, np.uint8), _c(weight_scale, np.uint8), _c(table8, np.float32)
    out = np.empty((N, K), np.float64)
    _check(lib().oq_decode_matrix_f64(_p(w), _p(s), _p(t), N, K, _p(out)))
    return out


def pack(src_bf16_bits, tables, table_id, E, N, K):
    """Pack bf16 bit patterns [E][N][K] -> (codes [E][N][K/2], scales [E][N][K/32])."""
    src = _c(src_bf16_bits, np.uint16)
    t, nt = _tables(tables)
    tid = _c(table_id, np.uint8)
    w = np.empty((E, N, K // 2), np.uint8)
    s = np.empty((E, N, K // 32), np.uint8)
    _check(lib().oq_pack(_p(src), E, N, K, _p(t), nt, _p(tid), _p(w), _p(s)))
    return w, s


def lloyd_fit(src_bf16_bits, grid0, max_iter: int, tol: float = 0.0):
    """Weighted Lloyd-Max fit of the 8 grid magnitudes over the ratios
    |w / 2^e| of bf16 weights (any shape, a whole number of 32-blocks along
    the last axis), weighted by (2^e)^2, from the ascending grid0:
    (grid fp32 [8], steps taken)."""
    src = _c(src_bf16_bits, np.uint16).reshape(-1)
    if src.size % 32:
        raise OracleError("weights must be whole 32-blocks")
    g0 = _c(grid0, np.float32)
    out = np.empty(8, np.float32)
    it = np.zeros(1, np.int32)
    _check(lib().oq_lloyd_fit(_p(src), src.size // 32, _p(g0), max_iter, float(tol), _p(out), _p(it)))
    return out, int(it[0])


def router_logits(x_bf16_bits, w_bf16_bits):
    """Router logits of the bf16 hidden states x [T, H] under the bf16 router
    gate w [E, H], in fp64: (logits [T, E], absdot [T, E]) with absdot the sum
    of |x[t][h] w[e][h]| (the scale of a finite-precision evaluation's error)."""
    x = _c(x_bf16_bits, np.uint16)
    w = _c(w_bf16_bits, np.uint16)
    T, H = x.shape
    E = w.shape[0]
    if w.shape[1] != H:
        raise OracleError("x and w disagree on H")
    logits = np.zeros((T, E), np.float64)
    absdot = np.zeros((T, E), np.float64)
    _check(lib().oq_router_logits(_p(x), _p(w), T, H, E, _p(logits), _p(absdot)))
    return logits, absdot


def shared_ffn(x_bf16_bits, wgu_bf16_bits, wd_bf16_bits):
    """The shared expert's output for every token, fp64 [T][H]: x [T][H],
    merged gate+up Wgu [2I][H] (gate rows first), down Wd [H][I], all bf16
    bit patterns."""
    x = _c(x_bf16_bits, np.uint16)
    wgu = _c(wgu_bf16_bits, np.uint16)
    wd = _c(wd_bf16_bits, np.uint16)
    T, H = x.shape
    I2, H2 = wgu.shape
    if H2 != H or I2 % 2 or wd.shape != (H, I2 // 2):
        raise OracleError("shared expert shapes disagree")
    out = np.zeros((T, H), np.float64)
    _check(lib().oq_shared_ffn(_p(x), T, H, _p(wgu), _p(wd), I2 // 2, _p(out)))
    return out


def route(logits, k):
    """(ids [T][k] int32, w [T][k] fp64) from fp32 logits [T][E]."""
    lg = _c(logits, np.float32)
    T, E = lg.shape
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    _check(lib().oq_route(_p(lg), T, E, k, _p(ids), _p(w)))
    return ids, w


def group(ids, E):
    """(counts [E], offsets [E+1], row_token [T*k], inv [T][k]) from ids [T][k]."""
    ids = _c(ids, np.int32)
    T, k = ids.shape
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    row_token = np.empty(T * k, np.int32)
    inv = np.empty((T, k), np.int32)
    _check(lib().oq_group(_p(ids), T, E, k, _p(counts), _p(offsets), _p(row_token), _p(inv)))
    return counts, offsets, row_token, inv


class Layer:
    """Host copy of a packed layer, one array per expert (None = not loaded).

    gate_w[e], up_w[e]: [I][H/2] uint8; gate_s[e], up_s[e]: [I][H/32];
    down_w[e]: [H][I/2]; down_s[e]: [H][I/32]; tables [n][8] fp32; table_id [E].
    """

    def __init__(self, E, H, I, tables, table_id):
        self.E, self.H, self.I = E, H, I
        self.tables = _c(tables, np.float32).reshape(-1, 8)
        self.table_id = _c(table_id, np.uint8)
        self.gate_w = [None] * E
        self.gate_s = [None] * E
        self.up_w = [None] * E
        self.up_s = [None] * E
        self.down_w = [None] * E
        self.down_s = [None] * E

    def set_expert(self, e, gate_w, gate_s, up_w, up_s, down_w, down_s):
        H, I = self.H, self.I
        self.gate_w[e] = _c(gate_w, np.uint8).reshape(I, H // 2)
        self.gate_s[e] = _c(gate_s, np.uint8).reshape(I, H // 32)
        self.up_w[e] = _c(up_w, np.uint8).reshape(I, H // 2)
        self.up_s[e] = _c(up_s, np.uint8).reshape(I, H // 32)
        self.down_w[e] = _c(down_w, np.uint8).reshape(H, I // 2)
        self.down_s[e] = _c(down_s, np.uint8).reshape(H, I // 32)

    def _struct(self):
        def arr(lst):
            a = (ctypes.c_void_p * self.E)()
            for i, v in enumerate(lst):
                a[i] = None if v is None else v.ctypes.data
            return a
        keep = [arr(x) for x in (self.gate_w, self.gate_s, self.up_w, self.up_s, self.down_w, self.down_s)]
        st = _Layer(self.E, self.H, self.I,
                    *[ctypes.cast(a, ctypes.POINTER(ctypes.c_void_p)) for a in keep],
                    ctypes.c_void_p(self.tables.ctypes.data), self.tables.shape[0],
                    ctypes.c_void_p(self.table_id.ctypes.data))
        return st, keep


def moe_tokens(layer: Layer, x_bf16_bits, logits, k, return_routing=False):
    """fp64 MoE output [n][H] for n independent tokens (x bf16 bits [n][H],
    logits fp32 [n][E])."""
    x = _c(x_bf16_bits, np.uint16)
    lg = _c(logits, np.float32)
    n = x.shape[0]
    out = np.empty((n, layer.H), np.float64)
    ids = np.empty((n, k), np.int32)
    w = np.empty((n, k), np.float64)
    st, keep = layer._struct()
    _check(lib().oq_moe_tokens(ctypes.byref(st), _p(x), _p(lg), n, k, _p(out), _p(ids), _p(w)))
    del keep
    if return_routing:
        return out, ids, w
    return out


def expert_partial(layer: Layer, e: int, x_bits_row, i0: int, i1: int):
    """fp64 [H]: expert e's output for one token (x bf16 bits [H]) restricted
    to intermediate channels [i0, i1)."""
    x = _c(x_bits_row, np.uint16).reshape(-1)
    y = np.empty(layer.H, np.float64)
    st, keep = layer._struct()
    _check(lib().oq_expert_partial(ctypes.byref(st), e, _p(x), i0, i1, _p(y)))
    del keep
    return y
