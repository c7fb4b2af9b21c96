"""Router logits, top-k with softmax weights, per-pair bit-width choice and the
stable permutation of (token, slot) pairs by expert.

The router stays in bf16 with an unchanged top-k (ExactMoE abstract: router in
BF16, top-k routing procedure unchanged, nothing pruned or substituted; "MoET in
FP4 MoE Inference": router/gate kept at higher precision).
"""
from __future__ import annotations

import numpy as np

from .numerics import bf16_to_f32

LANES = 32
CHUNK = 8  # consecutive elements per lane per step


def router_logits(x_bits: np.ndarray, wr_bits: np.ndarray, bias: np.ndarray | None = None) -> np.ndarray:
    """fp32 logits l[t][e] = sum_h x[t][h] * Wr[e][h] (+ bias[e]) in one fixed
    summation order (reading R13), so that the routing ids are reproducible bit
    for bit:

    * 32 partial sums ("lanes"); lane L owns h = 256*j + 8*L + i for
      j = 0..H/256-1, i = 0..7, and accumulates them in that (j, i) order,
      starting from +0, each step acc <- fp32(acc + x*w) (a fused multiply-add:
      the bf16*bf16 product is exact in float64 and the float64 sum rounded to
      fp32 equals one fp32 rounding of the exact value);
    * the 32 partials are combined pairwise by lane distance 16, 8, 4, 2, 1
      (partial[L] <- partial[L] + partial[L + d] for L < d), each an fp32 add;
    * then + bias[e] in fp32.

    x [T][H] and Wr [E][H] are bf16 bit patterns; H must be a multiple of 256.
    """
    x = bf16_to_f32(x_bits).astype(np.float64)   # [T][H]
    w = bf16_to_f32(wr_bits).astype(np.float64)  # [E][H]
    T, H = x.shape
    E = w.shape[0]
    assert H % (LANES * CHUNK) == 0
    J = H // (LANES * CHUNK)
    xv = x.reshape(T, J, LANES, CHUNK)
    wv = w.reshape(E, J, LANES, CHUNK)
    acc = np.zeros((T, E, LANES), dtype=np.float32)
    for j in range(J):
        for i in range(CHUNK):
            prod = xv[:, None, j, :, i] * wv[None, :, j, :, i]  # [T][E][32], exact
            acc = (acc.astype(np.float64) + prod).astype(np.float32)
    d = LANES // 2
    while d >= 1:
        acc = (acc[..., :d] + acc[..., d:2 * d]).astype(np.float32)
        d //= 2
    logits = acc[..., 0]
    if bias is not None:
        logits = (logits + np.asarray(bias, dtype=np.float32)[None, :]).astype(np.float32)
    return logits


def router_logits_f64(x_bits: np.ndarray, wr_bits: np.ndarray, bias: np.ndarray | None = None) -> np.ndarray:
    """The same logits in float64 with no prescribed order; used only to find
    near-ties whose fp32 order is decided by rounding."""
    x = bf16_to_f32(x_bits).astype(np.float64)
    w = bf16_to_f32(wr_bits).astype(np.float64)
    l = x @ w.T
    if bias is not None:
        l = l + np.asarray(bias, dtype=np.float64)[None, :]
    return l


def topk_softmax(logits: np.ndarray, k: int):
    """Top-k experts per token and their routing weights (reading R14/R15).

    Order: logit descending, equal logits by ascending expert id; the output slot
    j = 0..k-1 follows that order.  Weights: softmax restricted to the selected k,
    w_j = exp(l_j - l_0) / sum_i exp(l_i - l_0), evaluated in float64 from the
    fp32 logits and rounded to fp32 (equal to the full softmax renormalised over
    the selected experts, so the weights sum to 1).

    Returns ids int32 [T][k], weights float32 [T][k].
    """
    l = np.asarray(logits, dtype=np.float32)
    T, E = l.shape
    assert 1 <= k <= E
    order = np.lexsort((np.broadcast_to(np.arange(E), (T, E)), -l.astype(np.float64)), axis=-1)
    ids = order[:, :k].astype(np.int32)
    sel = np.take_along_axis(l, ids, axis=-1).astype(np.float64)
    ex = np.exp(sel - sel[:, :1])
    w = (ex / ex.sum(axis=-1, keepdims=True)).astype(np.float32)
    return ids, w


BIT_THRESHOLDS = (0.05, 0.15, 0.30)
BIT_CHOICES = (2, 3, 4, 8)


def select_bits(weights: np.ndarray, thresholds=BIT_THRESHOLDS, choices=BIT_CHOICES) -> np.ndarray:
    """Bit-width of each (token, slot) pair from its routing weight (MatMoE
    abstract: precision per expert from routing scores; PagedMoE abstract: prefix
    length chosen from the current routing weights).  Reading R16: with fp32
    thresholds t0 < t1 < t2, b = choices[0] if w < t0, choices[1] if w < t1,
    choices[2] if w < t2, else choices[3]; a weight equal to a threshold takes
    the higher tier.  Returns uint8 [T][k]."""
    w = np.asarray(weights, dtype=np.float32)
    t = [np.float32(v) for v in thresholds]
    tier = (w >= t[0]).astype(np.int64) + (w >= t[1]) + (w >= t[2])
    return np.asarray(choices, dtype=np.uint8)[tier]


def permute(ids: np.ndarray, E: int):
    """Group the T*k (token, slot) pairs by expert, stably (reading R17).

    Pair p = t*k + j has expert ids[t][j].  offsets[e] = number of pairs whose
    expert is below e (offsets[E] = T*k); inside expert e's segment the pairs
    appear in ascending p.  sorted_pair[r] is the pair at sorted row r and
    pair_to_row is its inverse.

    Returns (offsets int32 [E+1], sorted_pair int32 [T*k], pair_to_row int32 [T*k]).
    """
    flat = np.asarray(ids, dtype=np.int64).reshape(-1)
    P = flat.size
    counts = np.bincount(flat, minlength=E)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    sorted_pair = np.argsort(flat, kind="stable")
    pair_to_row = np.empty(P, dtype=np.int64)
    pair_to_row[sorted_pair] = np.arange(P)
    return offsets.astype(np.int32), sorted_pair.astype(np.int32), pair_to_row.astype(np.int32)


def active_experts(offsets: np.ndarray) -> np.ndarray:
    """Ids of the experts that received at least one pair, ascending."""
    o = np.asarray(offsets)
    return np.nonzero(o[1:] > o[:-1])[0].astype(np.int32)
