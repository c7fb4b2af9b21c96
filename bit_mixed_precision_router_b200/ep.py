"""Expert parallelism over the ranks of a process group: every rank routes its tokens
over all E experts, sends each routed row to the rank that owns its expert (rank r owns
experts [r E/G, (r+1) E/G)), the owners run the grouped FFN on what they received, and
the rows return for the combine (after "Every Expert Counts: ExactMoE for
Memory-Efficient W4A16 Inference", abstract: every selected expert is executed).

The layer is split into phases so that the two exchanges are the only collectives:
  prepare  route, gather the rows in sorted-row order, count rows per expert;
  expert   label received rows by local expert, permute, grouped FFN, rows back to
           arrival order;
  finish   combine with the sender's routing.
Every phase runs in the library's kernels; the exchanges are torch.distributed
all-to-alls (NCCL on GPUs)."""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import (Routing, moe_combine, moe_gather_rows, moe_grouped_ffn, moe_ids_from_counts, moe_permute,
               moe_route_topk)


@dataclass
class Sent:
    routing: Routing
    rows: torch.Tensor    # bf16 [T*k][H] in sorted-row order (ascending owner)
    counts: torch.Tensor  # int32 [E] rows per expert


def ep_prepare(x: torch.Tensor, w_router: torch.Tensor, bias: torch.Tensor | None, k: int) -> Sent:
    T, E = x.shape[0], w_router.shape[0]
    r = moe_route_topk(x, w_router, bias, k)
    rows = moe_gather_rows(x, r.sorted_pair, div=k, n=T * k)
    if T == 0:  # nothing was routed (the router writes nothing for an empty batch)
        counts = torch.zeros(E, dtype=torch.int32, device=x.device)
    else:
        counts = torch.diff(r.expert_offsets).to(torch.int32)  # kept on the device
    return Sent(r, rows, counts)


def ep_expert(recv_rows: torch.Tensor, recv_counts: torch.Tensor, experts_local, I: int) -> torch.Tensor:
    """recv_counts int32 [G][El] on the device, rows ordered by source then local expert;
    returns the FFN output rows in arrival order."""
    n = recv_rows.shape[0]
    El = recv_counts.shape[1]
    ids = moe_ids_from_counts(recv_counts, n)
    local = Routing.empty(n, El, 1, recv_rows.device)
    local.topk_ids.copy_(ids[:max(n, 1)])
    moe_permute(local.topk_ids, n, 1, El, out=local)
    y_sorted = moe_grouped_ffn(recv_rows, local, experts_local, I, El, 1)
    return moe_gather_rows(y_sorted, local.pair_to_row, n=n)


def ep_finish(y_back: torch.Tensor, sent: Sent, T: int, k: int, residual: torch.Tensor | None) -> torch.Tensor:
    return moe_combine(y_back, sent.routing, T, k, residual=residual)


def ep_moe_layer(x: torch.Tensor, w_router: torch.Tensor, bias: torch.Tensor | None, experts_local, I: int, k: int,
                 group=None, residual: bool = True) -> torch.Tensor:
    """The layer with experts sharded over the group (each rank passes its own E/G experts)."""
    import torch.distributed as dist
    G = dist.get_world_size(group)
    T, E = x.shape[0], w_router.shape[0]
    if E % G != 0:
        raise ValueError(f"{E} experts do not split evenly over {G} ranks")
    El = E // G
    sent = ep_prepare(x, w_router, bias, k)
    recv_counts = torch.empty_like(sent.counts)
    dist.all_to_all_single(recv_counts, sent.counts, group=group)  # El experts' counts to each owner
    send_splits = sent.counts.view(G, El).sum(1).tolist()
    recv_splits = recv_counts.view(G, El).sum(1).tolist()
    recv_rows = torch.empty((sum(recv_splits), x.shape[1]), dtype=x.dtype, device=x.device)
    dist.all_to_all_single(recv_rows, sent.rows[:T * k], recv_splits, send_splits, group=group)
    y_arrival = ep_expert(recv_rows, recv_counts.view(G, El), experts_local, I)
    y_back = torch.empty((T * k, x.shape[1]), dtype=x.dtype, device=x.device)
    dist.all_to_all_single(y_back, y_arrival[:sum(recv_splits)], send_splits, recv_splits, group=group)
    return ep_finish(y_back, sent, T, k, x if residual else None)
