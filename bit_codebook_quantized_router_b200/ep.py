"""Expert parallelism: whole experts per rank ("Round 7 -- Rewrite the
GLM-5.2 routed-expert encoder", "Owner-locked decisions" item 11: EP gets
whole experts), one all-to-all of routed token rows to the experts' owners
and one all-to-all of the expert outputs back, then the weighted combine at
the tokens' own rank.

Per rank (every rank holds its own tokens and the experts
[first(r), first(r+1)) of the layer):
  1. route its tokens: ids [T][k], weights [T][k];
  2. order its T*k (token, slot) rows by (owner rank, expert, token, slot)
     and exchange the row counts, then the activation rows and their local
     expert ids (all_to_all_single);
  3. run its experts on the rows it received (`compute`: rows grouped by
     local expert, each row through its expert with weight 1);
  4. send the output rows back (all_to_all_single with the counts swapped),
     put them back in (token, slot) order and add them in slot order
     (moe_q4_combine on the GPU).
Every step is deterministic: the received rows come in source-rank order, each
source's rows in a fixed order, and the combine adds slots in order.

This module is the host-side plumbing (plans and collectives); the expert
GEMMs and the combine run in the library's kernels (`gpu_compute`,
`bit_codebook_quantized_router_b200.combine`).  The same plan code runs with
the gloo backend on CPU, with any `compute`, which is how its bookkeeping is
tested without several GPUs.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

# a logit that never wins against 0 and is finite (non-finite logits are an error)
_LOSER = -30000.0


def expert_ranges(E: int, world: int):
    """[first, last) experts of every rank: contiguous, sizes differ by at most one."""
    base, rem = divmod(E, world)
    out, e0 = [], 0
    for r in range(world):
        n = base + (1 if r < rem else 0)
        out.append((e0, e0 + n))
        e0 += n
    return out


def owner_of(E: int, world: int) -> torch.Tensor:
    """int64 [E]: the rank that owns each expert."""
    own = torch.empty(E, dtype=torch.int64)
    for r, (a, b) in enumerate(expert_ranges(E, world)):
        own[a:b] = r
    return own


@dataclass
class DispatchPlan:
    order: torch.Tensor        # int64 [T*k]: (token, slot) rows in send order
    send_counts: list          # rows to each rank
    local_ids: torch.Tensor    # int32 [T*k]: expert of each sent row, local to its owner


def plan_dispatch(ids: torch.Tensor, E: int, world: int) -> DispatchPlan:
    """Order the (token, slot) rows of ids [T][k] by (owner rank, expert,
    token, slot) -- a stable sort on owner * E + expert of the row-major flat
    rows, on the ids' own device -- and count the rows per destination rank
    (the only values that go to the host: the collective's split sizes)."""
    dev = ids.device
    flat = ids.reshape(-1).to(torch.int64)
    own = owner_of(E, world).to(dev)
    first = torch.tensor([a for a, _ in expert_ranges(E, world)], dtype=torch.int64, device=dev)
    key = own[flat] * E + flat
    order = torch.sort(key, stable=True).indices
    counts = torch.bincount(own[flat], minlength=world).tolist()
    local = (flat[order] - first[own[flat[order]]]).to(torch.int32)
    return DispatchPlan(order, counts, local)


def _exchange_counts(send_counts, group, device):
    import torch.distributed as dist
    world = len(send_counts)
    if group is None and not (dist.is_available() and dist.is_initialized()):
        return list(send_counts)
    s = torch.tensor(send_counts, dtype=torch.int64, device=device)
    r = torch.empty(world, dtype=torch.int64, device=device)
    dist.all_to_all_single(r, s, group=group)
    return r.tolist()


def _a2a(x: torch.Tensor, send_counts, recv_counts, group):
    """all_to_all_single of the rows of x (any trailing shape)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return x.clone()
    out = torch.empty((sum(recv_counts),) + tuple(x.shape[1:]), dtype=x.dtype, device=x.device)
    # (bf16 rows travel as int32 pairs: every backend moves 32-bit words)
    xs = x.contiguous().view(torch.int32) if x.dtype == torch.bfloat16 else x.contiguous()
    os_ = out.view(torch.int32) if x.dtype == torch.bfloat16 else out
    dist.all_to_all_single(os_, xs, recv_counts, send_counts, group=group)
    return out


def ep_moe(x: torch.Tensor, ids: torch.Tensor, w: torch.Tensor, E: int, compute, combine, world: int = 1,
           group=None, out_dtype=torch.float32) -> torch.Tensor:
    """One expert-parallel MoE layer on this rank's tokens.

    x [T, H] bf16 (this rank's tokens); ids [T, k] int and w [T, k] fp32
    (their routing); compute(x_rows [R, H], local_ids int32 [R]) -> fp32
    [R, H] (each row through this rank's expert local_ids[i], weight 1);
    combine(y [T*k, H] in (token, slot) order, w) -> [T, H]; out_dtype:
    the dtype compute() returns (fp32 on the GPU)."""
    T, k = ids.shape
    H = x.shape[1]
    plan = plan_dispatch(ids.to(x.device), E, world)
    recv_counts = _exchange_counts(plan.send_counts, group, x.device)
    rows = x[plan.order // k]
    recv_x = _a2a(rows, plan.send_counts, recv_counts, group)
    recv_ids = _a2a(plan.local_ids, plan.send_counts, recv_counts, group)
    y_recv = compute(recv_x, recv_ids) if recv_x.shape[0] else torch.zeros((0, H), dtype=out_dtype,
                                                                             device=x.device)
    y_back = _a2a(y_recv.contiguous(), recv_counts, plan.send_counts, group)
    y = torch.empty((T * k, H), dtype=out_dtype, device=x.device)
    y[plan.order] = y_back
    return combine(y, w)


def gpu_compute(shard_layer, stream=None):
    """compute() of ep_moe on the GPU: the rows through this rank's experts
    with the library's forward, each row a token routed (top-1, weight 1) to
    its expert by a one-hot logit row.  shard_layer: a Layer holding the
    rank's experts only."""
    from . import _lib

    def run(x_rows, local_ids):
        R = x_rows.shape[0]
        lg = torch.full((R, shard_layer.E), _LOSER, dtype=torch.float32, device=x_rows.device)
        lg[torch.arange(R, device=x_rows.device), local_ids.to(torch.int64)] = 0.0
        out32 = torch.empty((R, shard_layer.H), dtype=torch.float32, device=x_rows.device)
        _lib.forward(shard_layer, x_rows.contiguous(), lg, 1, out_f32=out32, stream=stream)
        return out32
    return run


def shard_layer(layer, rank: int, world: int):
    """The Layer of rank `rank`'s experts (views into the full layer's arrays)."""
    from . import _lib
    a, b = expert_ranges(layer.E, world)[rank]
    return _lib.Layer(layer.gate_w[a:b], layer.gate_s[a:b], layer.up_w[a:b], layer.up_s[a:b],
                      layer.down_w[a:b], layer.down_s[a:b], layer.tables, layer.table_id[a:b])
