"""NVFP4 weights with NVFP4 activations (W4A4) for the prefill GEMMs (test
infrastructure, like the rest of ``oracle``).

The "MoET in FP4 MoE Inference" page (Q&A) names NVFP4 for expert weights; quantising
the activations to the same format on the fly and running a block-scaled FP4 product is
this repository's next prefill step, and the page fixes no activation recipe. Readings:

  R32  activations are quantised with the weights' NVFP4 recipe (R9): E2M1 elements, an
       E4M3 scale per 16 consecutive K elements, one fp32 scale per tensor, where the
       tensor is the whole input of one grouped GEMM -- x [T][H] for gate/up, the SwiGLU
       output h [P][I] (all routed rows) for down -- with its amax taken on the fly;
  R33  h is quantised from its float32 value (the kernel's epilogue precision), not from a
       bf16 rounding;
  R34  the product is exact per block pair: sum_k E2M1(a_k) E4M3(sa) E2M1(w_k) E4M3(sw),
       accumulated in float32 by the hardware, float64 here, with the two per-tensor
       scales g_a g_w applied once to the sum.
"""
from __future__ import annotations

import numpy as np

from .ffn import FMT_NVFP4, Experts, silu
from .numerics import bf16_to_f32
from .quant import dequant_nvfp4, quantize_nvfp4_f32
from .routing import active_experts


def quantize_act_nvfp4(a: np.ndarray):
    """One activation tensor [R][C] (float32 values) -> (codes uint8 [R][C/2], block
    scales uint8 E4M3 [R][C/16], g float32 scalar) by the NVFP4 recipe (R32)."""
    codes, sb, g = quantize_nvfp4_f32(np.asarray(a, dtype=np.float32)[None])
    return codes[0], sb[0], np.float32(g[0])


def dequant_act_nvfp4(codes: np.ndarray, sb: np.ndarray, g) -> np.ndarray:
    """The exact values E2M1 * E4M3 * g of a quantised activation tensor, float64 [R][C]."""
    return dequant_nvfp4(codes[None], sb[None], np.array([g], dtype=np.float32))[0]


def w4a4_gemm(a_codes, a_sb, a_g, w_codes, w_sb, w_g) -> np.ndarray:
    """[R][N] float64: sum_k a_k w_k of two NVFP4 operands (R34); the per-tensor scales
    multiply the block-scaled sum once."""
    a = dequant_act_nvfp4(a_codes, a_sb, np.float32(1))
    w = dequant_nvfp4(w_codes[None], w_sb[None], np.array([1], dtype=np.float32))[0]
    return (a @ w.T) * (float(a_g) * float(w_g))


def w4a4_grouped_ffn(x_bits: np.ndarray, offsets: np.ndarray, sorted_pair: np.ndarray, k: int,
                     experts: Experts) -> np.ndarray:
    """Grouped SwiGLU FFN with NVFP4 activations: x is quantised as one tensor; per expert
    g, u = x_hat W13_hat^T, h = silu(g) u; every routed row's h (float32, R33) is quantised
    as one tensor; y = h_hat W2_hat^T.  Returns y_rows float64 [T*k][H] in sorted-row order."""
    assert experts.fmt == FMT_NVFP4
    x = bf16_to_f32(x_bits)
    xc, xsb, xg = quantize_act_nvfp4(x)
    x_hat = dequant_act_nvfp4(xc, xsb, xg)
    P, H = sorted_pair.size, x.shape[1]
    I = experts.w13.shape[1] // 2
    h = np.zeros((P, I), dtype=np.float32)
    for e in active_experts(offsets):
        r = np.arange(offsets[e], offsets[e + 1])
        t = sorted_pair[r] // k
        w13 = experts.dequant(int(e))[0]
        gu = x_hat[t] @ w13.T
        h[r] = (silu(gu[:, :I]) * gu[:, I:]).astype(np.float32)
    hc, hsb, hg = quantize_act_nvfp4(h)
    h_hat = dequant_act_nvfp4(hc, hsb, hg)
    y = np.full((P, H), np.nan)
    for e in active_experts(offsets):
        r = np.arange(offsets[e], offsets[e + 1])
        w2 = experts.dequant(int(e))[1]
        y[r] = h_hat[r] @ w2.T
    return y
