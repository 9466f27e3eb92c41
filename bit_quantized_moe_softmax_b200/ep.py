"""Expert parallelism: the exchange steps of a routed-MoE layer whose experts
are split across ranks (one process per GPU, torch.distributed).

The router and the shared expert are replicated; expert e lives on the rank
whose contiguous range of experts holds it (``expert_owner``).  For the tokens
a rank holds:

* dispatch -- every (token, slot) pair is sent, as the token's row of x and
  the slot's expert id, to the rank that owns that expert; rows leave in
  (destination rank, slot index) order, so every rank receives its rows
  grouped by source rank and, within a source, in slot order;
* the owning ranks run their experts on the rows they received (a function
  the caller passes in: one output row per input row);
* combine -- the results travel back along the reverse route and the home
  rank adds them to its shared-expert output as sum_j w_j y_j, j = 0..k-1 in
  slot order, one multiply-add per slot (the fixed order of the one-GPU
  combine).

The layer is the one the pages describe for ds4 (DeepSeek V4 Flash's routed
experts plus a shared expert); splitting its experts over GPUs is this
project's extension for multi-GPU serving.  The functions take torch tensors
on any device; the collectives are those of the default process group (gloo
on CPU, NCCL on GPUs) or of ``group``.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist

from .dist import shard_range


def expert_owner(E: int, world: int) -> torch.Tensor:
    """[E] int64: the rank holding each expert (contiguous ranges, sizes differ by at most one)."""
    own = torch.empty(E, dtype=torch.int64)
    for r in range(world):
        a, b = shard_range(E, r, world)
        own[a:b] = r
    return own


def local_experts(E: int, rank: int, world: int) -> range:
    a, b = shard_range(E, rank, world)
    return range(a, b)


@dataclass
class DispatchPlan:
    n: int                     # tokens on this rank
    k: int                     # slots per token
    order: torch.Tensor        # [n*k] slot indices (t*k + j) in send order
    send_counts: list          # rows sent to each rank
    recv_counts: list          # rows received from each rank


def _world(group):
    return dist.get_world_size(group) if dist.is_initialized() else 1


def plan(ids: torch.Tensor, E: int, group=None) -> DispatchPlan:
    """Send order and per-rank row counts for this rank's routing ids [n, k].

    Collective: every rank of the group calls it (the counts are exchanged)."""
    n, k = ids.shape
    world = _world(group)
    owner = expert_owner(E, world).to(ids.device)
    dest = owner[ids.reshape(-1).long()]
    order = torch.sort(dest, stable=True).indices          # by destination, slot order within
    send = torch.bincount(dest, minlength=world).to(torch.int64)
    recv = torch.empty_like(send)
    if world > 1:
        dist.all_to_all_single(recv, send, group=group)
    else:
        recv.copy_(send)
    return DispatchPlan(n, k, order, send.tolist(), recv.tolist())


def _exchange(t: torch.Tensor, out_rows: int, send_counts, recv_counts, group):
    out = torch.empty((out_rows,) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
    if _world(group) > 1:
        dist.all_to_all_single(out, t.contiguous(), output_split_sizes=list(recv_counts),
                               input_split_sizes=list(send_counts), group=group)
    else:
        out.copy_(t)
    return out


def dispatch(x: torch.Tensor, ids: torch.Tensor, p: DispatchPlan, group=None):
    """Rows of x and their expert ids, moved to the experts' owners.

    Returns (rows [R, H], row_expert [R] int64), R = sum(p.recv_counts)."""
    rows = x[p.order // p.k]
    eid = ids.reshape(-1)[p.order].to(torch.int64)
    R = int(sum(p.recv_counts))
    return (_exchange(rows, R, p.send_counts, p.recv_counts, group),
            _exchange(eid, R, p.send_counts, p.recv_counts, group))


def combine(y_rows: torch.Tensor, w: torch.Tensor, p: DispatchPlan, base: torch.Tensor, group=None):
    """out[t] = base[t] + sum_j w[t, j] * y[t*k + j], j ascending.

    y_rows: the expert outputs for the rows this rank received, in the order
    dispatch delivered them; w: [n, k] routing weights; base: [n, H] (the
    shared expert's output, or zeros)."""
    back = _exchange(y_rows, p.n * p.k, p.recv_counts, p.send_counts, group)
    ys = torch.empty_like(back)
    ys[p.order] = back                                       # slot order again
    ys = ys.reshape((p.n, p.k) + tuple(back.shape[1:]))
    out = base.clone()
    for j in range(p.k):
        out = torch.addcmul(out, w[:, j:j + 1].to(out.dtype), ys[:, j].to(out.dtype))
    return out


def moe_forward_ep(x: torch.Tensor, ids: torch.Tensor, w: torch.Tensor, E: int, local_fn, base: torch.Tensor,
                   group=None) -> torch.Tensor:
    """One expert-parallel layer step for this rank's tokens: dispatch, the
    rank's own experts (local_fn(rows, row_expert) -> [R, H]), combine."""
    p = plan(ids, E, group)
    rows, eid = dispatch(x, ids, p, group)
    y = local_fn(rows, eid) if rows.shape[0] else rows.new_zeros((0,) + tuple(base.shape[1:]))
    return combine(y, w, p, base, group)


# ------------------------------------------------------------------ GPU halves (one rank's device work)
class GpuExpertShard:
    """This rank's experts on its GPU, as ``local_fn`` of ``moe_forward_ep``.

    A ds4moe handle over the contiguous expert range the rank owns, with top_k
    1 and no shared expert; every received row is one token routed to its
    local expert with weight 1 (ds4moe_forward_routed), so each output row is
    that expert's output for the row, computed by the same kernels as the
    one-GPU layer.  ``layer``: canonical blocks of every expert (gate, up,
    down indexed by global expert id), grid, H, I; rows beyond ``max_rows``
    are processed in chunks (decode plan up to decode_max rows, the tensor-core
    plan above)."""

    def __init__(self, layer: dict, E: int, rank: int, world: int, max_rows: int, device="cuda", expert_bits=0):
        from . import MoELayer

        rng = local_experts(E, rank, world)
        self.first, self.count = rng.start, len(rng)
        self.max_rows = max_rows
        self.H = layer["H"]
        self.lay = MoELayer(layer["H"], layer["I"], self.count, 1, max_rows, has_shared=False, device=device,
                            expert_bits=expert_bits) if self.count else None
        if self.lay is not None:
            sl = slice(self.first, self.first + self.count)
            self.lay.load(dict(H=layer["H"], I=layer["I"], E=self.count, k=1,
                               grid=layer.get("grid") if expert_bits != 4 else None,
                               W_r=torch.zeros(self.count, layer["H"]), b_r=None,
                               gate=layer["gate"][sl], up=layer["up"][sl], down=layer["down"][sl]))

    def __call__(self, rows: torch.Tensor, row_expert: torch.Tensor) -> torch.Tensor:
        from . import ds4moe_forward_routed

        R = rows.shape[0]
        out = torch.empty(R, self.H, dtype=torch.float32, device=rows.device)
        ids = (row_expert - self.first).to(torch.int32).reshape(R, 1).contiguous()
        ones = torch.ones(R, 1, dtype=torch.float32, device=rows.device)
        for a in range(0, R, self.max_rows):
            b = min(R, a + self.max_rows)
            ds4moe_forward_routed(self.lay.h, rows[a:b].contiguous(), ids[a:b], ones[a:b], out[a:b])
        return out


def combine_gpu(y_rows: torch.Tensor, w: torch.Tensor, p: DispatchPlan, base: torch.Tensor, group=None):
    """``combine`` with the sum on the device: the rows travel back and are put
    in slot order as there, then ds4moe_combine_slots adds base + sum_j w_j
    y_j, j ascending, one fused multiply-add per slot (the one-GPU layer's
    combine order, so a layer split over ranks gives the same bits)."""
    from . import ds4moe_combine_slots

    back = _exchange(y_rows, p.n * p.k, p.recv_counts, p.send_counts, group)
    ys = torch.empty_like(back)
    ys[p.order] = back
    out = torch.empty_like(base)
    ds4moe_combine_slots(ys.contiguous(), w.to(torch.float32).contiguous(), base.contiguous(), out)
    return out
