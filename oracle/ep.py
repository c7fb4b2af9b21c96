"""Expert parallelism over G ranks (test infrastructure, like the rest of ``oracle``):
each rank routes its own tokens over all E experts, sends every routed row to the rank
that owns its expert, the owner runs the grouped FFN on what it received, and the rows
come back for the combine.

The pages state no multi-device scheme ("Every Expert Counts: ExactMoE for
Memory-Efficient W4A16 Inference", abstract: every selected expert is executed, none
pruned or substituted; the layer's result must not depend on where an expert runs).
Readings:

  R35  E is a multiple of G and rank r owns the contiguous experts
       [r E/G, (r+1) E/G);
  R36  a rank sends its routed rows in its sorted-row order (ascending expert, then
       ascending pair): destinations ascend, so each destination's rows are one
       contiguous run; the owner receives the runs in source-rank order and serves them
       as a batch of single-slot "tokens", grouped by local expert (stable in arrival
       order), then returns each row to its sender in the order it arrived;
  R37  the combine runs on the sender with its own routing weights, unchanged.
"""
from __future__ import annotations

import numpy as np

from .ffn import Experts, combine, grouped_ffn
from .routing import permute, router_logits, topk_softmax


def owner(e: int, E: int, G: int) -> int:
    """Rank that owns expert e (R35)."""
    assert E % G == 0
    return e // (E // G)


def dispatch_plan(offsets_by_rank, E: int, G: int):
    """From each rank's routing offsets [E+1] (R36): send_splits [G][G] (rows rank s sends
    to rank d) and recv_counts [G][G][E/G] (rows rank d receives from rank s for its local
    expert j)."""
    El = E // G
    send = np.zeros((G, G), dtype=np.int64)
    recv = np.zeros((G, G, El), dtype=np.int64)
    for s, off in enumerate(offsets_by_rank):
        n_e = np.diff(np.asarray(off, dtype=np.int64))
        for d in range(G):
            send[s, d] = int(n_e[d * El:(d + 1) * El].sum())
            recv[d, s] = n_e[d * El:(d + 1) * El]
    return send, recv


def _slice_experts(ex: Experts, lo: int, hi: int) -> Experts:
    g13 = None if ex.w13_g is None else ex.w13_g[lo:hi]
    g2 = None if ex.w2_g is None else ex.w2_g[lo:hi]
    return Experts(ex.fmt, ex.w13[lo:hi], ex.w13_s[lo:hi], ex.w2[lo:hi], ex.w2_s[lo:hi], g13, g2)


def ep_layer(x_by_rank, wr_bits, bias, experts: Experts, k: int, G: int, residual: bool = True):
    """The layer on G ranks (R35-R37); x_by_rank[r] bf16 bits [T_r][H].  Returns each
    rank's output float64 [T_r][H] (the combine with residual = x when ``residual``)."""
    E = wr_bits.shape[0]
    El = E // G
    routes = []
    for x in x_by_rank:
        ids, w = topk_softmax(router_logits(x, wr_bits, bias), k)
        off, sp, p2r = permute(ids, E)
        routes.append((ids, w, off, sp, p2r))
    # sends: each rank's rows (token rows of its sorted pairs) in sorted-row order
    sent = []
    for x, (ids, w, off, sp, p2r) in zip(x_by_rank, routes):
        sent.append(x[sp // k])
    send, recv = dispatch_plan([r[2] for r in routes], E, G)
    # each owner: received rows in source order, grouped by local expert, one slot each
    y_back = [np.full((len(r[3]), x_by_rank[0].shape[1]), np.nan) for r in routes]
    for d in range(G):
        parts, local_ids, origin = [], [], []
        for s in range(G):
            start = int(send[s, :d].sum())
            n = int(send[s, d])
            parts.append(sent[s][start:start + n])
            for j in range(El):
                local_ids += [j] * int(recv[d, s, j])
            origin += [(s, start + i) for i in range(n)]
        if not origin:
            continue
        xr = np.concatenate(parts, axis=0)
        lids = np.asarray(local_ids, dtype=np.int64).reshape(-1, 1)
        loff, lsp, lp2r = permute(lids, El)
        y_sorted = grouped_ffn(xr, loff, lsp, 1, _slice_experts(experts, d * El, (d + 1) * El))
        y_arrival = y_sorted[lp2r]  # back to arrival order
        for i, (s, row) in enumerate(origin):
            y_back[s][row] = y_arrival[i]
    outs = []
    for x, (ids, w, off, sp, p2r), yb in zip(x_by_rank, routes, y_back):
        outs.append(combine(yb, w, p2r, x if residual else None))
    return outs
