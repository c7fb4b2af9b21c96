"""Weight formats of the routed experts: quantise, pack, unpack, dequantise.

Weights are bf16 matrices stored row-major as [E][N][K] (K contiguous); for the
gate/up projection N = 2I (rows 0..I-1 gate, I..2I-1 up), for the down
projection N = H, K = I.  All integer decisions are taken in fp32 with IEEE
round-to-nearest-even division, exactly as written below, so that a device
implementation can reproduce every bit.
"""
from __future__ import annotations

import numpy as np

from .numerics import (bf16_round_bits, bf16_to_f32, e2m1_decode, e2m1_from_f32_satfinite,
                       e4m3_decode, e4m3_from_f32_satfinite)

GROUP = 128


def _groups(w_bits: np.ndarray) -> np.ndarray:
    """bf16 bits [..., K] -> fp32 values [..., K/128, 128]."""
    w = bf16_to_f32(w_bits)
    K = w.shape[-1]
    assert K % GROUP == 0
    return w.reshape(w.shape[:-1] + (K // GROUP, GROUP))


def _symmetric_codes(w_bits: np.ndarray, qmax: int, qmin: int):
    """Per-group symmetric integer codes: s = bf16(max|w| / qmax) (fp32 division,
    then round-to-nearest-even into bf16: reading R1 / R5); q = clamp(rint(w / s),
    qmin, qmax) with fp32 division and ties-to-even rounding (reading R2); an
    all-zero group has s = 0 and q = 0.  Returns (q int64 [..., K], s bits)."""
    g = _groups(w_bits)
    amax = np.max(np.abs(g), axis=-1)
    s_bits = bf16_round_bits(amax / np.float32(qmax))
    s = bf16_to_f32(s_bits)
    safe = np.where(s == 0, np.float32(1), s)[..., None]
    q = np.rint(g / safe).astype(np.int64)
    q = np.clip(q, qmin, qmax)
    q = np.where((s == 0)[..., None], 0, q)
    return q.reshape(w_bits.shape), s_bits


# ----------------------------------------------------------------------------
# INT4, symmetric, group 128 (W4A16)
# ----------------------------------------------------------------------------
def quantize_w4g128(w_bits: np.ndarray):
    """Symmetric group-128 four-bit quantisation of the routed experts' weights
    (ExactMoE abstract: group-128 symmetric 4-bit, routed experts only).

    scale = bf16(max|w| / 7) per group of 128 consecutive K elements of a row;
    q = clamp(rint(w / scale), -8, 7).  Storage (reading R3): offset binary
    u = q + 8; element k of a row sits in bits 4*(k % 8) .. 4*(k % 8) + 3 of
    32-bit word k // 8.

    Returns packed uint32 [..., K/8] and scales as bf16 bit patterns [..., K/128].
    """
    q, s_bits = _symmetric_codes(w_bits, 7, -8)
    u = (q + 8).astype(np.uint32)
    u = u.reshape(u.shape[:-1] + (u.shape[-1] // 8, 8))
    shifts = (4 * np.arange(8)).astype(np.uint32)
    packed = np.bitwise_or.reduce(u << shifts, axis=-1).astype(np.uint32)
    return packed, s_bits


def unpack_w4(packed: np.ndarray) -> np.ndarray:
    """uint32 [..., K/8] -> signed codes q int64 [..., K]."""
    shifts = (4 * np.arange(8)).astype(np.uint32)
    u = (packed[..., None] >> shifts) & np.uint32(0xF)
    return u.reshape(packed.shape[:-1] + (packed.shape[-1] * 8,)).astype(np.int64) - 8


def dequant_w4g128(packed: np.ndarray, s_bits: np.ndarray) -> np.ndarray:
    """w' = scale * q, as float64 [..., K]."""
    q = unpack_w4(packed).astype(np.float64)
    s = bf16_to_f32(s_bits).astype(np.float64)
    return (q.reshape(q.shape[:-1] + (-1, GROUP)) * s[..., None]).reshape(q.shape)


# ----------------------------------------------------------------------------
# Eight bitplanes of a signed 8-bit code (variable precision prefixes)
# ----------------------------------------------------------------------------
def pack_bitplanes(w_bits: np.ndarray):
    """Quantise to signed 8-bit group-128 codes and store them as eight bitplanes
    (PagedMoE abstract: one stored expert state in a bitplane layout whose lower
    precisions are prefixes of the higher ones).

    scale = bf16(max|w| / 127) (reading R5); q = clamp(rint(w / scale), -127, 127);
    u = q + 128 in 1..255.  Plane p (p = 0..7) holds bit 7 - p of u, so plane 0
    is the most significant (reading R6) and a b-bit prefix is planes 0..b-1.
    Layout (reading R7): planes [E][8][N][K/32] uint32, element k of a row in bit
    k % 32 of word k // 32.

    Input [E][N][K] bf16 bits; returns (planes uint32 [E][8][N][K/32], scales bf16 bits [E][N][K/128]).
    """
    assert w_bits.ndim == 3
    q, s_bits = _symmetric_codes(w_bits, 127, -127)
    u = (q + 128).astype(np.uint32)  # [E][N][K]
    E, N, K = u.shape
    planes = np.zeros((E, 8, N, K // 32), dtype=np.uint32)
    ub = u.reshape(E, N, K // 32, 32)
    bitpos = np.arange(32, dtype=np.uint32)
    for p in range(8):
        bit = (ub >> np.uint32(7 - p)) & np.uint32(1)
        planes[:, p] = np.bitwise_or.reduce(bit << bitpos, axis=-1).astype(np.uint32)
    return planes, s_bits


def unpack_bitplanes(planes: np.ndarray, b: int = 8) -> np.ndarray:
    """Planes [E][8][N][K/32] -> the top-b-bit prefix of u, i.e. (u >> (8-b)) << (8-b),
    as int64 [E][N][K], reading only planes 0..b-1."""
    E, _, N, KW = planes.shape
    bitpos = np.arange(32, dtype=np.uint32)
    u = np.zeros((E, N, KW * 32), dtype=np.int64)
    for p in range(b):
        bits = (planes[:, p][..., None] >> bitpos) & np.uint32(1)
        u += bits.reshape(E, N, KW * 32).astype(np.int64) << (7 - p)
    return u


def prefix_reconstruct(u: np.ndarray, b: int) -> np.ndarray:
    """Floor-and-compensation reconstruction at b bits (MatMoE abstract: floor and
    compensation; reading R8): keep the top b bits of u (the floor) and add half
    of the dropped range, 2**(7-b), for b < 8 (the compensation), so the code
    lands on the midpoint of the bin it denotes.  u is the full 8-bit code."""
    assert 1 <= b <= 8
    u = np.asarray(u, dtype=np.int64)
    floor = (u >> (8 - b)) << (8 - b)
    return floor + ((1 << (7 - b)) if b < 8 else 0)


def dequant_bitplane(planes: np.ndarray, s_bits: np.ndarray, b: int) -> np.ndarray:
    """w' = scale * (u'_b - 128) from the b-plane prefix, as float64 [E][N][K]."""
    floor = unpack_bitplanes(planes, b)
    u_b = floor + ((1 << (7 - b)) if b < 8 else 0)
    s = bf16_to_f32(s_bits).astype(np.float64)
    q = (u_b - 128).astype(np.float64)
    return (q.reshape(q.shape[:-1] + (-1, GROUP)) * s[..., None]).reshape(q.shape)


# ----------------------------------------------------------------------------
# NVFP4: E2M1 elements, E4M3 scale per 16 elements, fp32 scale per tensor
# ----------------------------------------------------------------------------
NVFP4_BLOCK = 16


def quantize_nvfp4(w_bits: np.ndarray):
    """NVFP4 quantisation of [E][N][K] bf16 weights (format named on the "MoET in
    FP4 MoE Inference" page; recipe reading R9, per-tensor scope reading R10).

    Per expert matrix: g = amax / (6 * 448) in fp32.  Per block of 16
    consecutive K elements: sb = E4M3_satfinite(amax_block / (6 * g)) (the
    product 6*g rounded to fp32 first, then fp32 division).  Per element:
    code = E2M1_satfinite(w / (float(sb) * g)) (product to fp32 first, then fp32
    division).  g == 0 or sb == 0 gives codes 0.  Element 2i sits in the low
    nibble of byte i (reading R12).

    Returns (codes uint8 [E][N][K/2], block scales uint8 E4M3 codes [E][N][K/16],
    g float32 [E]).
    """
    assert w_bits.ndim == 3
    return quantize_nvfp4_f32(bf16_to_f32(w_bits))


def quantize_nvfp4_f32(w: np.ndarray):
    """The NVFP4 recipe of quantize_nvfp4 on float32 values [E][N][K] (one tensor per
    leading index); the same steps, for inputs that are not bf16 (activations)."""
    w = np.asarray(w, dtype=np.float32)
    assert w.ndim == 3
    E, N, K = w.shape
    amax_t = np.max(np.abs(w.reshape(E, -1)), axis=-1).astype(np.float32)
    g = (amax_t / np.float32(6 * 448)).astype(np.float32)
    blocks = w.reshape(E, N, K // NVFP4_BLOCK, NVFP4_BLOCK)
    amax_b = np.max(np.abs(blocks), axis=-1)
    denom = (np.float32(6) * g).astype(np.float32)[:, None, None]
    safe_denom = np.where(denom == 0, np.float32(1), denom)
    sb = e4m3_from_f32_satfinite((amax_b / safe_denom).astype(np.float32))
    sb = np.where(denom == 0, np.uint8(0), sb).astype(np.uint8)
    sbv = e4m3_decode(sb).astype(np.float32)
    prod = (sbv * g[:, None, None]).astype(np.float32)
    safe_prod = np.where(prod == 0, np.float32(1), prod)[..., None]
    v = (blocks / safe_prod).astype(np.float32)
    codes = e2m1_from_f32_satfinite(v)
    codes = np.where((prod == 0)[..., None], np.uint8(0), codes).reshape(E, N, K)
    packed = (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)
    return packed, sb, g


def dequant_nvfp4(packed: np.ndarray, sb: np.ndarray, g: np.ndarray) -> np.ndarray:
    """w' = E2M1(code) * E4M3(sb) * g, float64 [E][N][K]."""
    E, N, K2 = packed.shape
    codes = np.empty((E, N, K2 * 2), dtype=np.uint8)
    codes[..., 0::2] = packed & 0xF
    codes[..., 1::2] = packed >> 4
    vals = e2m1_decode(codes).reshape(E, N, -1, NVFP4_BLOCK)
    scale = e4m3_decode(sb) * np.asarray(g, dtype=np.float64)[:, None, None]
    return (vals * scale[..., None]).reshape(E, N, K2 * 2)
