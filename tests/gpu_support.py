"""GPU-test support: device layers packed by the CUDA library from the seeded
generators, the matching oracle layers (packed by the oracle from the same
bf16 weights), and the output tolerance check."""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

import oracle
import bit_codebook_quantized_router_b200 as q4
from bit_codebook_quantized_router_b200 import inputs

# MoE output tolerance: relative Frobenius error <= 5e-3 and max-abs error <=
# 2e-2 * rms(reference) against the fp64 oracle, applied to the layer's fp32
# combine result.  (Storing that result as bf16 adds a rounding of up to
# 2^-8 |out| -- 0.018 rms at a 4.5-sigma element -- that the max-abs bound
# cannot absorb; the bf16 output is checked to be the exact round-to-nearest-
# even of the fp32 result instead: check_bf16_is_rounding.)
REL_FRO = 5e-3
MAX_ABS_RMS = 2e-2

# Canary bands: every buffer the library writes in the forward tests sits
# inside a larger allocation whose bytes before and after it hold a fixed
# pattern, checked after the call (catches writes past an output's end).
GUARD_BYTES = 4096  # keeps the view 512-byte aligned, as the workspace needs
GUARD_BYTE = 0xA5


class Guarded:
    """A tensor `view` of `shape` and `dtype` with canary bands around it."""

    def __init__(self, shape, dtype, device="cuda"):
        esize = torch.tensor([], dtype=dtype).element_size()
        self.n = int(np.prod(shape)) * esize
        self.buf = torch.full((self.n + 2 * GUARD_BYTES,), GUARD_BYTE, dtype=torch.uint8, device=device)
        self.view = self.buf[GUARD_BYTES:GUARD_BYTES + self.n].view(dtype).view(shape)

    def check(self, what=""):
        head = self.buf[:GUARD_BYTES]
        tail = self.buf[GUARD_BYTES + self.n:]
        assert bool((head == GUARD_BYTE).all()) and bool((tail == GUARD_BYTE).all()), \
            f"{what}: bytes written outside the buffer"


_POOL = None


def pool():
    global _POOL
    if _POOL is None:
        _POOL = ThreadPoolExecutor(max_workers=max(1, os.cpu_count() or 1))
    return _POOL


def check_out(gpu_rows: torch.Tensor, ref_rows: np.ndarray, what=""):
    """Assert the GPU rows (the fp32 combine result) match the fp64 oracle
    rows within tolerance."""
    g = gpu_rows.float().cpu().numpy().astype(np.float64)
    r = np.asarray(ref_rows, np.float64)
    assert g.shape == r.shape
    assert np.all(np.isfinite(g)), what
    nr = np.linalg.norm(r)
    rel = np.linalg.norm(g - r) / nr if nr > 0 else np.linalg.norm(g)
    rms = np.sqrt(np.mean(r * r))
    mx = np.max(np.abs(g - r)) if g.size else 0.0
    assert rel <= REL_FRO, f"{what}: rel Frobenius {rel:.3e} > {REL_FRO}"
    assert mx <= MAX_ABS_RMS * rms + 1e-30, f"{what}: max abs {mx:.3e} > {MAX_ABS_RMS}*rms {rms:.3e}"
    return rel, mx / rms if rms > 0 else 0.0


_DEV_LAYERS = {}


def device_layer(w: inputs.Workload, keep: int = 2) -> q4.Layer:
    """All experts of workload w, generated on the GPU and packed by
    moe_q4_pack (cached per workload; at most `keep` layers resident)."""
    key = (w.index, w.shape, w.mixed_tables)
    if key in _DEV_LAYERS:
        return _DEV_LAYERS[key]
    while len(_DEV_LAYERS) >= keep:
        _DEV_LAYERS.pop(next(iter(_DEV_LAYERS)))
        torch.cuda.empty_cache()
    sh = w.shape
    tables, tid = inputs.layer_tables(w)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    packed = {}
    for proj in inputs.PROJECTIONS:
        N, K = inputs.proj_shape(sh, proj)
        big = torch.empty((sh.E, N, K), dtype=torch.bfloat16, device="cuda")
        for e in range(sh.E):
            big[e] = inputs.expert_weight(w, e, proj, device="cuda")
        packed[proj] = q4.pack(big, tables, tid, status=status)
        del big
    st = q4.lib().moe_q4_read_status(q4._lib._ptr(status), q4._lib._stream())
    assert st == 0, f"pack status {st}"
    L = q4.Layer(*packed["gate"], *packed["up"], *packed["down"], tables, tid)
    _DEV_LAYERS[key] = L
    return L


def oracle_layer(w: inputs.Workload, experts, dev: q4.Layer | None = None) -> oracle.Layer:
    """Oracle layer holding `experts`, packed by the oracle from the same bf16
    weights the device layer was packed from.  When `dev` is given, the GPU
    bytes of those experts must equal the oracle's bit for bit."""
    sh = w.shape
    tables, tid = inputs.layer_tables(w)
    L = oracle.Layer(sh.E, sh.H, sh.I, tables, tid)
    experts = sorted(set(int(e) for e in experts))
    dev_name = "cuda" if dev is not None else "cpu"

    def pack_job(job):
        e, blobs = job
        res = {}
        for proj in inputs.PROJECTIONS:
            N, K = inputs.proj_shape(sh, proj)
            c, s = oracle.pack(blobs[proj][None], tables, tid[e:e + 1], 1, N, K)
            res[proj] = (c[0], s[0])
        return e, res

    # weights are drawn on the main thread (torch), packing runs in threads,
    # a chunk of experts at a time to bound host memory
    chunk = max(4, os.cpu_count() or 1)
    for i in range(0, len(experts), chunk):
        jobs = []
        for e in experts[i:i + chunk]:
            blobs = {proj: inputs.bf16_bits(inputs.expert_weight(w, e, proj, device=dev_name))
                     for proj in inputs.PROJECTIONS}
            jobs.append((e, blobs))
        for e, res in pool().map(pack_job, jobs):
            if dev is not None:
                for proj, (dw, ds) in (("gate", (dev.gate_w, dev.gate_s)), ("up", (dev.up_w, dev.up_s)),
                                       ("down", (dev.down_w, dev.down_s))):
                    assert np.array_equal(dw[e].cpu().numpy(), res[proj][0]), f"codes differ e={e} {proj}"
                    assert np.array_equal(ds[e].cpu().numpy(), res[proj][1]), f"scales differ e={e} {proj}"
            L.set_expert(e, *res["gate"], *res["up"], *res["down"])
    return L


def oracle_tokens(L: oracle.Layer, x_bits: np.ndarray, logits: np.ndarray, k: int, tokens):
    """fp64 oracle rows for the listed tokens, one token per thread."""
    tokens = list(tokens)

    def one(t):
        return oracle.moe_tokens(L, x_bits[t:t + 1], logits[t:t + 1], k)[0]

    return np.stack(list(pool().map(one, tokens))) if tokens else np.zeros((0, L.H))


def check_bf16_is_rounding(out_bf16: torch.Tensor, out_f32: torch.Tensor):
    """The bf16 output must be the round-to-nearest-even of the fp32 result."""
    assert torch.equal(out_bf16, out_f32.to(torch.bfloat16))
