"""Grouped SwiGLU expert FFN over the permuted pairs, the routing-weighted
combine, the whole layer, the chained decode stack, and a dense brute-force
checker that shares none of the grouping logic.

Numerics: weights are dequantised exactly (every dequantised value is exact in
float64) and every sum is taken in float64 with numpy matmul; the intermediate
h and the per-row outputs stay float64 (reading R18/R19).  This is the
"dequantise, then matmul naively" reference, for tolerance comparison only
(ExactMoE abstract: the low-bit layer is not meant to be numerically identical
to the BF16 one).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from .numerics import bf16_round_bits, bf16_to_f32
from .quant import dequant_bitplane, dequant_nvfp4, dequant_w4g128
from .routing import active_experts, permute, router_logits, select_bits, topk_softmax

FMT_W4G128, FMT_BITPLANE8, FMT_NVFP4 = 0, 1, 2


@dataclass
class Experts:
    """Quantised expert weights as produced by ``oracle.quant`` (numpy arrays).

    fmt FMT_W4G128: w13/w2 packed uint32, w13_s/w2_s bf16 bits.
    fmt FMT_BITPLANE8: w13/w2 planes uint32 [E][8][N][K/32], w13_s/w2_s bf16 bits.
    fmt FMT_NVFP4: w13/w2 uint8 codes, w13_s/w2_s E4M3 uint8, w13_g/w2_g fp32 [E].
    """
    fmt: int
    w13: np.ndarray
    w13_s: np.ndarray
    w2: np.ndarray
    w2_s: np.ndarray
    w13_g: np.ndarray | None = None
    w2_g: np.ndarray | None = None

    def dequant(self, e: int, b: int = 8):
        """(W13 [2I][H], W2 [H][I]) of expert e as float64; b = prefix planes for bitplanes."""
        sl = slice(e, e + 1)
        if self.fmt == FMT_W4G128:
            return dequant_w4g128(self.w13[e], self.w13_s[e]), dequant_w4g128(self.w2[e], self.w2_s[e])
        if self.fmt == FMT_BITPLANE8:
            return (dequant_bitplane(self.w13[sl], self.w13_s[sl], b)[0],
                    dequant_bitplane(self.w2[sl], self.w2_s[sl], b)[0])
        if self.fmt == FMT_NVFP4:
            return (dequant_nvfp4(self.w13[sl], self.w13_s[sl], self.w13_g[sl])[0],
                    dequant_nvfp4(self.w2[sl], self.w2_s[sl], self.w2_g[sl])[0])
        raise ValueError(self.fmt)


def silu(g: np.ndarray) -> np.ndarray:
    """g * sigmoid(g), sigmoid(g) = 1 / (1 + exp(-g))."""
    return g / (1.0 + np.exp(-g))


def swiglu_expert(x_rows: np.ndarray, w13: np.ndarray, w2: np.ndarray) -> np.ndarray:
    """One expert on a block of rows: gate = x W_gate^T, up = x W_up^T (W_gate =
    rows 0..I-1 of w13, W_up = rows I..2I-1), h = silu(gate) * up, y = h W2^T."""
    I = w13.shape[0] // 2
    gu = x_rows @ w13.T
    h = silu(gu[:, :I]) * gu[:, I:]
    return h @ w2.T


def grouped_ffn(x_bits: np.ndarray, offsets: np.ndarray, sorted_pair: np.ndarray, k: int,
                experts: Experts, bits: np.ndarray | None = None, rows: np.ndarray | None = None) -> np.ndarray:
    """Grouped expert FFN over the permuted pairs.

    Sorted row r (expert e with offsets[e] <= r < offsets[e+1]) holds pair
    p = sorted_pair[r] = t*k + j; its output is expert e's SwiGLU FFN applied to
    x[t], with expert e read at bits[t][j] planes for the bitplane format.
    Returns y_rows float64 [T*k][H] (rows in sorted order).  ``rows`` restricts
    the computation to a subset of sorted rows (other rows are NaN).
    """
    x = bf16_to_f32(x_bits).astype(np.float64)
    P = sorted_pair.size
    H = x.shape[1]
    want = np.ones(P, dtype=bool) if rows is None else np.isin(np.arange(P), rows)
    y = np.full((P, H), np.nan)
    flat_bits = None if bits is None else np.asarray(bits).reshape(-1)
    for e in active_experts(offsets):
        r = np.arange(offsets[e], offsets[e + 1])
        r = r[want[r]]
        if r.size == 0:
            continue
        p = sorted_pair[r]
        t = p // k
        if experts.fmt == FMT_BITPLANE8:
            bsel = flat_bits[p].astype(np.int64)
            for b in np.unique(bsel):
                m = bsel == b
                w13, w2 = experts.dequant(int(e), int(b))
                y[r[m]] = swiglu_expert(x[t[m]], w13, w2)
        else:
            w13, w2 = experts.dequant(int(e))
            y[r] = swiglu_expert(x[t], w13, w2)
    return y


def combine(y_rows: np.ndarray, weights: np.ndarray, pair_to_row: np.ndarray,
            residual_bits: np.ndarray | None = None) -> np.ndarray:
    """out[t] = sum_j w[t][j] * y_rows[pair_to_row[t*k + j]] (+ residual[t]),
    float64 [T][H] (ExactMoE abstract: the selected experts' outputs are combined
    by the unchanged routing weights)."""
    T, k = weights.shape
    yr = y_rows[np.asarray(pair_to_row).reshape(T, k)]  # [T][k][H]
    out = np.einsum("tk,tkh->th", np.asarray(weights, dtype=np.float64), yr)
    if residual_bits is not None:
        out = out + bf16_to_f32(residual_bits).astype(np.float64)
    return out


@dataclass
class Routing:
    logits: np.ndarray
    ids: np.ndarray
    weights: np.ndarray
    offsets: np.ndarray
    sorted_pair: np.ndarray
    pair_to_row: np.ndarray
    bits: np.ndarray | None


def route(x_bits, wr_bits, bias, k, E, bit_rule: bool = False) -> Routing:
    logits = router_logits(x_bits, wr_bits, bias)
    ids, w = topk_softmax(logits, k)
    offsets, sorted_pair, pair_to_row = permute(ids, E)
    bits = select_bits(w) if bit_rule else None
    return Routing(logits, ids, w, offsets, sorted_pair, pair_to_row, bits)


def moe_layer(x_bits, wr_bits, bias, experts: Experts, k: int, residual_bits=None, bit_rule=None):
    """The whole layer: route, grouped FFN, combine.  Returns (out float64 [T][H], Routing)."""
    E = wr_bits.shape[0]
    if bit_rule is None:
        bit_rule = experts.fmt == FMT_BITPLANE8
    r = route(x_bits, wr_bits, bias, k, E, bit_rule)
    y = grouped_ffn(x_bits, r.offsets, r.sorted_pair, k, experts, r.bits)
    return combine(y, r.weights, r.pair_to_row, residual_bits), r


def stack_layer_step(x_bits, wr_bits, experts: Experts, k: int):
    """One layer of the chained decode stack (reading R20): no norm and no
    attention; x_next = bf16(x + moe(x)), the residual add being the layer's
    combine with residual = x.  Returns (x_next bf16 bits, Routing)."""
    out, r = moe_layer(x_bits, wr_bits, None, experts, k, residual_bits=x_bits)
    return bf16_round_bits(out.astype(np.float32)), r


def dense_bruteforce(x_bits, weights_full: np.ndarray, ids: np.ndarray, experts: Experts,
                     bits: np.ndarray | None = None) -> np.ndarray:
    """Checker with no permutation: evaluate every expert on every token, then
    out[t] = sum_j w[t][j] * FFN_{ids[t][j]}(x[t]).  Only for tiny shapes."""
    x = bf16_to_f32(x_bits).astype(np.float64)
    T, k = ids.shape
    E = experts.w13.shape[0]
    out = np.zeros_like(x)
    for e in range(E):
        for bb in ([8] if bits is None else sorted(set(int(v) for v in np.asarray(bits).ravel()))):
            w13, w2 = experts.dequant(e, bb)
            ye = swiglu_expert(x, w13, w2)  # all tokens through expert e
            for t in range(T):
                for j in range(k):
                    if ids[t, j] == e and (bits is None or int(bits[t, j]) == bb):
                        out[t] += float(weights_full[t, j]) * ye[t]
    return out
