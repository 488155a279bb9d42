"""Seeded synthetic inputs for the routed-expert MoE over 4-bit codebook weights.

This module is shared by the tests, the benchmark and the oracle's callers.
It holds no step of the layer's arithmetic: only random draws, the two value
tables the layer is given, and the fixed shapes of the workloads.

Workloads (all synthetic; the pages ship no data):
  * tiny:  T=4, hidden 256, intermediate 128, 8 experts, top-2;
  * GLM-5.2-shaped layer: hidden 6144, intermediate 2048, 256 routed experts,
    top-8 ("Round 7 -- Rewrite the GLM-5.2 routed-expert encoder",
    "Ground truth and corrections": model geometry), at T = 1, 8, 64
    (uniform routing) and T = 2048, 8192 (Zipf-skewed routing).
Value distributions: expert weights N(0, 0.02) as bf16; activations bf16
N(0, 1); router logits fp32 N(0, 1), plus for the skewed workloads a
per-expert bias -s * ln(rank_e), rank a seeded permutation of 1..E, s = 1.1.
Seeds: workload c uses seed c for weights, c+100 for activations, c+200 for
logits, c+300 for the Zipf ranks.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

# E2M1 (MXFP4) value table: the power-of-two grid {0, .5, 1, 1.5, 2, 3, 4, 6}
# ("aidendle94/GLM-5.2-NF4-Lloyd-Experts-GPTQ", "What this is").
E2M1_TABLE = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float32)

# Experts that the pages' defect list names as written with E2M1 nibbles
# ("aidendle94/GLM-5.2-NF4-Lloyd-Experts-GPTQ", "Known defect: 5 experts are
# packed on the wrong grid"); the mixed-table workload flags these ids.
E2M1_EXPERTS = (15, 30, 86, 139, 164)

WEIGHT_STD = 0.02


@dataclasses.dataclass(frozen=True)
class Shape:
    H: int
    I: int
    E: int
    k: int


TINY = Shape(H=256, I=128, E=8, k=2)
GLM = Shape(H=6144, I=2048, E=256, k=8)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int
    T: int
    shape: Shape
    zipf: bool = False
    mixed_tables: bool = False

    @property
    def seed_weights(self):
        return self.index

    @property
    def seed_x(self):
        return self.index + 100

    @property
    def seed_logits(self):
        return self.index + 200

    @property
    def seed_zipf(self):
        return self.index + 300


WORKLOADS = {
    "tiny": Workload("tiny", 0, 4, TINY),
    "decode_t1": Workload("decode_t1", 1, 1, GLM),
    "decode_t8": Workload("decode_t8", 2, 8, GLM),
    "decode_t64": Workload("decode_t64", 2, 64, GLM),
    "prefill_t2048": Workload("prefill_t2048", 3, 2048, GLM, zipf=True),
    "prefill_t8192": Workload("prefill_t8192", 4, 8192, GLM, zipf=True, mixed_tables=True),
}


def lloyd_max_grid(seed: int = 0, n_samples: int = 100_000, levels: int = 8,
                   tol: float = 1e-12, max_iter: int = 100_000) -> np.ndarray:
    """Lloyd-Max magnitude grid fitted to |N(0,1)| draws.

    Unweighted Lloyd iteration in fp64 (the pages fit a weighted variant to
    real weights: "aidendle94/GLM-5.2-NF4-Lloyd-Experts-GPTQ", "What this
    is"; the synthetic workload has no real weights to weight by).  Start at
    the sample quantiles (i + 0.5) / levels; alternate cell boundaries at
    midpoints and levels at cell means until no level moves by more than tol.
    Returned ascending as fp32 (the grid files store JSON floats).
    """
    rng = np.random.default_rng(seed)
    a = np.sort(np.abs(rng.standard_normal(n_samples)))
    c = np.quantile(a, (np.arange(levels) + 0.5) / levels)
    for _ in range(max_iter):
        edges = (c[1:] + c[:-1]) / 2
        cell = np.searchsorted(edges, a)
        sums = np.bincount(cell, weights=a, minlength=levels)
        cnt = np.bincount(cell, minlength=levels)
        new = np.where(cnt > 0, sums / np.maximum(cnt, 1), c)
        done = np.max(np.abs(new - c)) < tol
        c = new
        if done:
            break
    return np.sort(c).astype(np.float32)


def layer_tables(w: Workload, lloyd_seed: int = 0):
    """(tables [n][8] fp32, table_id [E] uint8): table 0 is the Lloyd grid,
    table 1 (mixed workload only) is E2M1 for the flagged experts."""
    grid = lloyd_max_grid(lloyd_seed)
    if w.mixed_tables:
        tables = np.stack([grid, E2M1_TABLE])
        tid = np.zeros(w.shape.E, np.uint8)
        for e in E2M1_EXPERTS:
            if e < w.shape.E:
                tid[e] = 1
        return tables, tid
    return grid[None, :].copy(), np.zeros(w.shape.E, np.uint8)


PROJECTIONS = ("gate", "up", "down")


def proj_shape(shape: Shape, proj: str):
    """[N, K] of a projection: gate/up map hidden -> intermediate, down maps
    intermediate -> hidden."""
    return (shape.I, shape.H) if proj in ("gate", "up") else (shape.H, shape.I)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & ((1 << 63) - 1))
    return g


def expert_weight(w: Workload, e: int, proj: str, device="cpu") -> torch.Tensor:
    """bf16 [N, K] weights of one projection of expert e, N(0, 0.02).

    Each (workload seed, expert, projection) has its own generator, so any
    subset of experts can be regenerated alone.  Draws on ``device``; the same
    seed gives different values on CPU and CUDA, so both sides of a
    comparison must take the same tensor.
    """
    N, K = proj_shape(w.shape, proj)
    seed = (int(w.seed_weights) * 1_000_003 + int(e) * 17 + PROJECTIONS.index(proj)) * 2_654_435_761
    g = _gen(seed, device)
    t = torch.randn((N, K), generator=g, device=device, dtype=torch.float32)
    return (t * WEIGHT_STD).to(torch.bfloat16)


def shared_expert_weights(w: Workload, I: int | None = None, device="cpu"):
    """BF16 shared expert of the workload's layer: (gate_up [2I, H], down
    [H, I]), N(0, 0.02), gate rows first; I defaults to the routed experts'
    intermediate size (the GLM-5.2 shared expert's, 75.5 MB of BF16 per
    layer at H = 6144)."""
    I = w.shape.I if I is None else I
    H = w.shape.H
    g = _gen(w.seed_weights * 7919 + 11, device)
    gu = torch.randn((2 * I, H), generator=g, device=device, dtype=torch.float32) * WEIGHT_STD
    dn = torch.randn((H, I), generator=g, device=device, dtype=torch.float32) * WEIGHT_STD
    return gu.to(torch.bfloat16).contiguous(), dn.to(torch.bfloat16).contiguous()


def activations(w: Workload, device="cpu", T: int | None = None, variant: int = 0) -> torch.Tensor:
    """bf16 [T, H] activations, N(0, 1); `variant` > 0 draws another batch."""
    T = w.T if T is None else T
    g = _gen(w.seed_x * 7919 + 1 + variant * 1_000_033, device)
    return torch.randn((T, w.shape.H), generator=g, device=device).to(torch.bfloat16)


def zipf_bias(w: Workload, s: float = 1.1) -> np.ndarray:
    """Per-expert logit bias -s * ln(rank), rank a seeded permutation of 1..E."""
    rng = np.random.default_rng(w.seed_zipf)
    rank = rng.permutation(w.shape.E) + 1
    return (-s * np.log(rank.astype(np.float64))).astype(np.float32)


def router_logits(w: Workload, device="cpu", T: int | None = None, variant: int = 0) -> torch.Tensor:
    """fp32 [T, E] router logits: N(0, 1), plus the Zipf bias when skewed;
    `variant` > 0 draws another batch (same bias)."""
    T = w.T if T is None else T
    g = _gen(w.seed_logits * 7919 + 2 + variant * 1_000_033, device)
    lg = torch.randn((T, w.shape.E), generator=g, device=device, dtype=torch.float32)
    if w.zipf:
        lg = lg + torch.from_numpy(zipf_bias(w)).to(device)
    return lg.contiguous()


def router_weight(w: Workload, device="cpu") -> torch.Tensor:
    """bf16 [E, H] router gate (the "mlp.gate" linear the pages hold in
    BF16): N(0, 0.02), seeded from the workload's weight seed."""
    g = _gen(w.seed_weights * 7919 + 5, device)
    return (torch.randn((w.shape.E, w.shape.H), generator=g, device=device, dtype=torch.float32) * 0.02).to(
        torch.bfloat16).contiguous()


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Host uint16 view of a bf16 tensor's bit patterns."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def bits_to_bf16(a: np.ndarray) -> torch.Tensor:
    """bf16 tensor from host uint16 bit patterns."""
    return torch.from_numpy(np.ascontiguousarray(a, np.uint16).view(np.int16)).view(torch.bfloat16)
