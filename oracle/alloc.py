"""Budgeted per-expert bit allocation for bitplane experts (test infrastructure, like
the rest of ``oracle``).

Follows "DuoRate: Two-Rate Per-Expert Precision Allocation for Mixture-of-Experts
Serving" (AI Radio episode), key concepts "DuoRate Pipeline Stages" and "Routing
Frequency Cancellation": a distortion tensor baked offline, unlabeled profiling of a
workload's prefill, and a selection that solves a Lagrangian rate-distortion
allocation with one dot product per expert and a bisection to a read budget; the
routing frequency drops out of every per-expert decision.  The pages give no
formulas beyond the two rates (resident rate = mean over experts of R(M_e), read
rate = sum_e f_e R(M_e)), so the steps below are the plainest reading (readings
R23-R27):

  R23  distortion tensor: for expert e, prefix length b (planes 0..b-1) and input
       channel k of the gate/up matrix (the one that reads the token),
       delta[e][b][k] = sum_n (s_{n, k/128} * (u'_b[n][k] - u[n][k]))^2, i.e. the
       squared dequantisation error of the b-bit floor-and-compensation prefix
       against the full 8-bit code (b = 8 gives 0);
  R24  profiling: m[k] = mean over the workload's tokens of x[t][k]^2;
  R25  per-expert distortion D[e][b] = sum_k m[k] * delta[e][b][k] (one dot product
       per expert and candidate); rate R(b) = b bits per weight; routing frequency
       f_e = (pairs routed to e) / (T * k);
  R26  at multiplier lam >= 0 every expert takes argmin_b D[e][b] + lam * b over the
       candidate set (f_e > 0 multiplies both terms and cancels); ties go to the
       larger b;
  R27  the read rate sum_e f_e * b_e(lam) does not increase with lam; bisection
       (a fixed number of halvings of [0, lam_hi]) finds the smallest lam whose read
       rate is within the budget, and the allocation at the upper end of the final
       interval is returned.  "Within the budget" is decided exactly: the integer
       sum_e n_e * b_e (n_e pairs routed to e) against the fp64 product budget * sum_e n_e.
       A budget below the smallest candidate returns the smallest candidate
       everywhere; experts with n_e = 0 take the smallest candidate (they are not read).
"""
from __future__ import annotations

import numpy as np

from .quant import GROUP, prefix_reconstruct, unpack_bitplanes
from .numerics import bf16_to_f32

BISECT_STEPS = 100


def bitplane_distortion(planes: np.ndarray, s_bits: np.ndarray) -> np.ndarray:
    """delta [E][8][K] float64 (index b-1 for prefix length b) of bitplane weights
    planes [E][8][N][K/32], scales [E][N][K/128] (reading R23)."""
    u = unpack_bitplanes(planes, 8)                       # [E][N][K] full codes
    E, N, K = u.shape
    s = bf16_to_f32(s_bits).astype(np.float64)             # [E][N][K/128]
    s_full = np.repeat(s, GROUP, axis=-1)                  # [E][N][K]
    out = np.zeros((E, 8, K), dtype=np.float64)
    for b in range(1, 9):
        err = (prefix_reconstruct(u, b) - u).astype(np.float64) * s_full
        out[:, b - 1, :] = np.sum(err * err, axis=1)
    return out


def activation_moments(x_bits: np.ndarray) -> np.ndarray:
    """m [H] float64: mean over tokens of x^2 (reading R24); x bf16 bits [T][H]."""
    x = bf16_to_f32(x_bits).astype(np.float64)
    return np.mean(x * x, axis=0)


def expert_distortion(delta: np.ndarray, m: np.ndarray, choices) -> np.ndarray:
    """D [E][len(choices)] float64: one dot product per expert and candidate (R25)."""
    return np.stack([delta[:, b - 1, :] @ m for b in choices], axis=1)


def choose(D: np.ndarray, choices, lam: float) -> np.ndarray:
    """Per-expert argmin_b D[e][b] + lam * b, ties to the larger b (R26); returns the
    index into `choices` per expert."""
    c = np.asarray(choices, dtype=np.float64)
    cost = D + lam * c[None, :]
    best = np.zeros(D.shape[0], dtype=np.int64)
    for e in range(D.shape[0]):
        bi = 0
        for i in range(1, len(choices)):
            if cost[e, i] < cost[e, bi] or (cost[e, i] == cost[e, bi] and c[i] > c[bi]):
                bi = i
        best[e] = bi
    return best


def read_rate(idx: np.ndarray, f: np.ndarray, choices) -> float:
    """sum_e f_e * b_e (the routing-weighted decode rate, bits per weight)."""
    c = np.asarray(choices, dtype=np.float64)
    return float(np.sum(f * c[idx]))


def lambda_upper(D: np.ndarray, choices) -> float:
    """A multiplier at which every expert takes the smallest candidate: the largest
    distortion saving per bit over the smallest candidate, doubled, plus one."""
    c = np.asarray(choices, dtype=np.float64)
    i0 = int(np.argmin(c))
    hi = 0.0
    for i in range(len(choices)):
        if c[i] > c[i0]:
            hi = max(hi, float(np.max((D[:, i0] - D[:, i]) / (c[i] - c[i0]))))
    return 2.0 * hi + 1.0


def within_budget(idx: np.ndarray, counts: np.ndarray, choices, budget: float) -> bool:
    """sum_e n_e * b_e <= budget * sum_e n_e, the left side an exact integer (R27)."""
    c = [int(v) for v in choices]
    lhs = sum(int(n) * c[int(i)] for n, i in zip(counts, idx))
    return float(lhs) <= float(np.float64(budget) * np.float64(int(np.sum(counts))))


def allocate_bits(D: np.ndarray, counts: np.ndarray, choices, budget: float, steps: int = BISECT_STEPS):
    """Bits per expert (uint8 [E]) and the final multiplier (R27); counts[e] = pairs
    routed to expert e (f_e = counts[e] / sum(counts))."""
    c = np.asarray(choices, dtype=np.float64)
    counts = np.asarray(counts, dtype=np.int64)
    i0 = int(np.argmin(c))
    E = D.shape[0]
    lo, hi = 0.0, lambda_upper(D, choices)
    idx_lo = choose(D, choices, lo)
    if within_budget(idx_lo, counts, choices, budget):
        idx = idx_lo
        lam = lo
    elif not within_budget(choose(D, choices, hi), counts, choices, budget):
        idx = np.full(E, i0, dtype=np.int64)    # infeasible budget: the smallest candidate
        lam = hi
    else:
        for _ in range(steps):
            mid = 0.5 * (lo + hi)
            if within_budget(choose(D, choices, mid), counts, choices, budget):
                hi = mid
            else:
                lo = mid
        idx = choose(D, choices, hi)
        lam = hi
    idx = np.where(counts > 0, idx, i0)
    return c[idx].astype(np.uint8), lam


def expert_counts(offsets: np.ndarray) -> np.ndarray:
    """n_e from the routing offsets [E+1]: pairs routed to expert e."""
    return np.diff(np.asarray(offsets, dtype=np.int64))


def expand_bits(ids: np.ndarray, bits_e: np.ndarray) -> np.ndarray:
    """Per-pair bit-widths bits[t*k + j] = bits_e[ids[t][j]]."""
    return np.asarray(bits_e)[np.asarray(ids).reshape(-1)].astype(np.uint8)
