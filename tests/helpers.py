"""Shared test helpers: golden-file readers and small packed layers built by
the oracle from the seeded input generators."""
from __future__ import annotations

import os

import numpy as np
import torch

import oracle
from bit_codebook_quantized_router_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read_decode_golden():
    tables, rows, nibbles = {}, [], []
    with open(os.path.join(GOLDEN, "decode_hand.txt")) as f:
        for line in f:
            p = line.split()
            if not p or p[0].startswith("#"):
                continue
            if p[0] == "table":
                tables[p[1]] = np.array([float(v) for v in p[2:10]], np.float32)
            elif p[0] == "row":
                rows.append((p[1], int(p[2]), [int(v, 16) for v in p[3:11]]))
            elif p[0] == "nibbles":
                nibbles.append((p[1], int(p[2]), bytes.fromhex(p[3]), [int(v, 16) for v in p[4:]]))
    return tables, rows, nibbles


def read_pack_golden():
    blocks = []
    with open(os.path.join(GOLDEN, "pack_hand.txt")) as f:
        cur = None
        for line in f:
            p = line.split()
            if not p or p[0].startswith("#"):
                continue
            if p[0] == "block":
                cur = (p[1], int(p[2]), bytes.fromhex("".join(p[3:])))
            elif p[0] == "values":
                blocks.append(cur + (np.array([float(v) for v in p[1:]], np.float32),))
    return blocks


def f32_to_bf16_bits(a):
    """bf16 bits of fp32 values that are exact in bf16 (torch's RNE cast)."""
    return inputs.bf16_bits(torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16))


def bf16_bits_to_f32(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


def build_layer_host(w: inputs.Workload, experts=None, device="cpu", identical_to=None):
    """Generate bf16 weights for `experts` (default all) and pack them with the
    oracle.  Returns (oracle.Layer, dict e -> {proj: (codes, scales)}, dict e ->
    {proj: bf16 tensor})."""
    sh = w.shape
    tables, tid = inputs.layer_tables(w)
    L = oracle.Layer(sh.E, sh.H, sh.I, tables, tid)
    experts = range(sh.E) if experts is None else experts
    packed, raw = {}, {}
    for e in experts:
        src_e = e if identical_to is None else identical_to
        packed[e], raw[e] = {}, {}
        for proj in inputs.PROJECTIONS:
            N, K = inputs.proj_shape(sh, proj)
            wt = inputs.expert_weight(w, src_e, proj, device=device)
            raw[e][proj] = wt
            codes, scales = oracle.pack(inputs.bf16_bits(wt)[None], tables, tid[e:e + 1], 1, N, K)
            packed[e][proj] = (codes[0], scales[0])
        L.set_expert(e, *packed[e]["gate"], *packed[e]["up"], *packed[e]["down"])
    return L, packed, raw
