"""Row placement for expert parallelism across GPUs (host-side planning).

Rowwise expert parallelism ("Ai2 rebuilds Olmo's training stack for
trillion-parameter MoEs", "Routing work stays on the GPU", first bullet;
"Supercharging Olmo-core for Efficient and Scalable MoE Training", Summary):
the E experts are split over W ranks, E / W consecutive experts per rank, and
every rank writes each of its routed token rows straight into the receive
buffer of the rank that holds the row's expert.  The placement has to agree
on every rank without a host round trip: each rank knows its own routing,
and after one exchange of the per-expert counts (W x E integers, e.g. an
all-gather of the counts tensor that stays on the device) every rank can
compute, for every (source rank, expert), where that source's rows start in
the owner's buffer.

Receive buffer of rank r: its local experts back to back in expert order;
inside an expert, rows grouped by source rank in rank order; inside a source,
the source's own dispatch order (ascending token index).  This is exactly the
single-GPU dispatch of the batch formed by concatenating the ranks' batches
in rank order, restricted to rank r's experts -- so the expert GEMMs and the
combine see the same rows as a single GPU would.

A row (t, i) of rank s routed to expert e lands on rank owner(e) at
    send_base[e] + (dest_local[t, i] - offsets_local[e])
where dest_local / offsets_local are rank s's own single-GPU dispatch plan
(moe_permute_rows).  Everything here is integer tensor arithmetic (torch ops on
whatever device the counts live on); the row movement itself is the
dispatch's job.
"""
from __future__ import annotations

import torch


def experts_per_rank(E: int, world: int) -> int:
    if world < 1 or E % world:
        raise ValueError(f"E = {E} experts do not split evenly over {world} ranks")
    return E // world


def owner(expert: torch.Tensor, E: int, world: int) -> torch.Tensor:
    """Rank holding each expert index."""
    return torch.div(expert, experts_per_rank(E, world), rounding_mode="floor")


def exchange_counts(counts: torch.Tensor, group=None) -> torch.Tensor:
    """All ranks' per-expert counts [W, E] from this rank's [E] counts (one
    all-gather on the process group; the result stays on counts' device)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    out = torch.empty(world * counts.numel(), dtype=counts.dtype, device=counts.device)
    dist.all_gather_into_tensor(out, counts.contiguous().view(-1), group=group)
    return out.view(world, counts.numel())


def plan(counts_all: torch.Tensor, rank: int) -> dict:
    """Placement from the exchanged counts ``counts_all`` [W, E] (int).

    Returns, for this rank:
      recv_offsets [E/W + 1]  offsets of its local experts in its receive
                              buffer (exclusive scan; the last entry = rows
                              it receives);
      src_base     [W, E/W]   where source rank s's rows of local expert j
                              start in its receive buffer;
      send_base    [E]        where this rank's rows of expert e start in the
                              receive buffer of owner(e)."""
    W, E = counts_all.shape
    El = experts_per_rank(E, W)
    c = counts_all.to(torch.int64)
    per_rank = c.view(W, W, El)                 # [source, owner, local expert]
    totals = per_rank.sum(dim=0)                # [owner, local expert]
    offs = torch.zeros(W, El + 1, dtype=torch.int64, device=c.device)
    offs[:, 1:] = torch.cumsum(totals, dim=1)   # per owner: offsets of its experts
    before = torch.cumsum(per_rank, dim=0) - per_rank  # rows of earlier sources
    base = offs[:, :El].unsqueeze(0) + before   # [source, owner, local expert]
    return {"recv_offsets": offs[rank].clone(),
            "src_base": base[:, rank, :].clone(),
            "send_base": base[rank].reshape(E).clone()}


def destinations(dest_local: torch.Tensor, idx: torch.Tensor, offsets_local: torch.Tensor,
                 send_base: torch.Tensor, E: int, world: int):
    """(owner rank, position in the owner's receive buffer) of every routed
    row (t, i) of this rank, from its single-GPU dispatch plan."""
    e = idx.to(torch.int64)
    pos = send_base[e] + (dest_local.to(torch.int64) - offsets_local.to(torch.int64)[e])
    return owner(e, E, world), pos
