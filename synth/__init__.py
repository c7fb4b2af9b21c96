"""Seeded synthetic inputs for the low-bit MoE layer: the one module that both the
CPU oracle's tests and the GPU path's tests/benchmark draw their inputs from.

It holds none of the layer's arithmetic: no quantisation, routing or FFN math.
Only random numbers.

Every stream is counter-based, so element ``i`` of a stream with seed ``s`` is a
pure function of ``(s, i)``; any slice (one expert's rows, one token) can be
regenerated on the host without producing the rest, and the CUDA generator in
``moe_synth.h`` computes the very same bits on the device.

Definitions (each restated from its published source, in integer or
correctly-rounded IEEE arithmetic only, so host and device agree bit for bit):

* counter hash: SplitMix64 (Steele, Lea & Flood, "Fast Splittable Pseudorandom
  Number Generators", OOPSLA 2014).  Word ``j`` of stream ``s`` is
  ``mix64(s + (j + 1) * 0x9E3779B97F4A7C15 mod 2**64)``.
* uniform in [0, 1): the top 53 bits of a word times 2**-53.
* approximately-normal deviates: the Irwin-Hall sum of twelve uniforms minus
  six (mean 0, variance 1, support [-6, 6]).  Element ``i`` takes the four
  16-bit fields of words ``3i, 3i+1, 3i+2``; field ``v`` stands for the
  uniform ``(v + 0.5) / 65536``, so the deviate is exactly
  ``(sum(v) - 393210) / 65536`` -- no transcendental function is involved, so
  no libm difference between host and device can change a bit.
* scaling: ``float64(z) * float64(std)`` (one IEEE rounding), then fp32
  (round-to-nearest-even), then bf16 (round-to-nearest-even).
* uniform(lo, hi): ``lo + (hi - lo) * u`` in float64 (two IEEE roundings, no
  fused multiply-add), then fp32, then bf16.
"""
from __future__ import annotations

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

#: Offsets added to a workload's base seed to obtain each tensor's stream.
SEED_X, SEED_WR, SEED_W13, SEED_W2, SEED_BIAS, SEED_RESID = 1, 2, 3, 4, 5, 6


def mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 finaliser on a uint64 array (wrapping arithmetic)."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def words(seed: int, j: np.ndarray) -> np.ndarray:
    """Word ``j`` (uint64 array) of the stream with the given seed."""
    j = np.asarray(j, dtype=np.uint64)
    with np.errstate(over="ignore"):
        ctr = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + (j + np.uint64(1)) * GAMMA
    return mix64(ctr)


def uniform01(seed: int, idx: np.ndarray) -> np.ndarray:
    """float64 uniform in [0, 1) for element indices ``idx``."""
    w = words(seed, idx)
    return (w >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def _ih12_chunk(seed: int, idx: np.ndarray) -> np.ndarray:
    """Sum of the twelve 16-bit fields of words 3i, 3i+1, 3i+2 (two fields per
    32-bit half added first, then the halves), as int64."""
    lanes = np.uint64(0x0000FFFF0000FFFF)
    acc = np.zeros(idx.shape, dtype=np.uint64)
    base = idx * np.uint64(3)
    for m in range(3):
        w = words(seed, base + np.uint64(m))
        acc += (w & lanes) + ((w >> np.uint64(16)) & lanes)
    return ((acc & np.uint64(0xFFFFFFFF)) + (acc >> np.uint64(32))).astype(np.int64)


def irwin_hall12(seed: int, idx: np.ndarray) -> np.ndarray:
    """Exact float64 deviate with mean 0 and variance 1 for indices ``idx``."""
    idx = np.asarray(idx, dtype=np.uint64)
    return (_ih12_chunk(seed, idx) - 393210).astype(np.float64) / 65536.0


def f32_to_bf16_bits(f: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round-to-nearest-even (inputs are finite here)."""
    u = np.ascontiguousarray(f, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    return ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _index(start: int, n: int) -> np.ndarray:
    return np.arange(start, start + n, dtype=np.uint64)


_CHUNK = 1 << 20


def _parallel_chunks(n: int, fn) -> np.ndarray:
    """Evaluates fn(lo, hi) -> uint16 array over [0, n) in chunks on a thread pool
    (numpy releases the GIL inside its loops); the result does not depend on the
    chunking."""
    out = np.empty(n, dtype=np.uint16)
    spans = [(lo, min(n, lo + _CHUNK)) for lo in range(0, n, _CHUNK)]
    if len(spans) <= 1:
        for lo, hi in spans:
            out[lo:hi] = fn(lo, hi)
        return out
    import concurrent.futures as cf
    import os
    with cf.ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 1)) as ex:
        for (lo, hi), part in zip(spans, ex.map(lambda s: fn(*s), spans)):
            out[lo:hi] = part
    return out


def normal_bf16(seed: int, n: int, std: float, start: int = 0) -> np.ndarray:
    """``n`` bf16 bit patterns (uint16) of std * Irwin-Hall(12) deviates, elements start..start+n-1."""
    def part(lo, hi):
        z = irwin_hall12(seed, _index(start + lo, hi - lo))
        return f32_to_bf16_bits((z * np.float64(std)).astype(np.float32))
    return _parallel_chunks(n, part)


def uniform_bf16(seed: int, n: int, lo: float, hi: float, start: int = 0) -> np.ndarray:
    """``n`` bf16 bit patterns of lo + (hi - lo) * U[0,1), elements start..start+n-1."""
    d = np.float64(hi) - np.float64(lo)

    def part(a, b):
        u = uniform01(seed, _index(start + a, b - a))
        return f32_to_bf16_bits((np.float64(lo) + d * u).astype(np.float32))
    return _parallel_chunks(n, part)


def normal_rows_bf16(seed: int, shape_tail: tuple, std: float, first_row: int, n_rows: int) -> np.ndarray:
    """Rows ``first_row .. first_row+n_rows-1`` of a tensor whose row length is prod(shape_tail)."""
    row = int(np.prod(shape_tail))
    flat = normal_bf16(seed, n_rows * row, std, start=first_row * row)
    return flat.reshape((n_rows,) + tuple(shape_tail))


def permutation(seed: int, n: int) -> np.ndarray:
    """A seeded permutation of 0..n-1 (Fisher-Yates, Durstenfeld's variant),
    drawing word i of the stream for step i; integer arithmetic only."""
    p = np.arange(n, dtype=np.int64)
    w = words(seed, np.arange(max(n - 1, 0), dtype=np.uint64))
    for step, i in enumerate(range(n - 1, 0, -1)):
        j = int(w[step] % np.uint64(i + 1))
        p[i], p[j] = p[j], p[i]
    return p


def zipf_rank_bias(seed: int, E: int, s: float = 1.1) -> np.ndarray:
    """Per-expert additive router-logit bias -s * ln(rank_e), rank_e a seeded
    permutation of 1..E; adding it to the logits scales expert e's softmax mass
    by rank_e**-s, i.e. expert popularity follows a Zipf(s) law.  fp32."""
    rank = permutation(seed, E) + 1
    return (-np.float64(s) * np.log(rank.astype(np.float64))).astype(np.float32)
