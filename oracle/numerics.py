"""Number formats used by the oracle, written from their definitions.

* bf16: IEEE-754 binary32 with the low 16 fraction bits dropped (1 sign, 8
  exponent, 7 fraction bits); fp32 -> bf16 rounds to nearest, ties to even.
* E4M3 (OCP 8-bit floating point specification, "E4M3" variant): 1 sign, 4
  exponent (bias 7), 3 fraction bits; subnormals at exponent 0; no infinities;
  S.1111.111 is NaN, so the largest finite magnitude is 1.75 * 2**8 = 448.
* E2M1 (OCP Microscaling formats specification, FP4 element type): 1 sign, 2
  exponent (bias 1), 1 fraction bit; magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}.

The "satfinite" conversions clamp magnitudes above the largest finite value to
it, and round everything else to the nearest representable value with ties
going to the code whose least significant (fraction) bit is 0.

The NVFP4 scheme (E2M1 elements, one E4M3 scale per 16 elements, one fp32
scale per tensor) is the format named on the "MoET in FP4 MoE Inference" page,
references list ("NVIDIA NVFP4 for efficient low-precision inference").
"""
from __future__ import annotations

import numpy as np


# ----------------------------------------------------------------------------
# bf16
# ----------------------------------------------------------------------------
def bf16_round_bits(f32: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit pattern (uint16), round to nearest, ties to even.

    Adding 0x7FFF plus the kept LSB to the 32-bit pattern and truncating is
    round-half-even on the dropped 16 bits; a carry out of the fraction bumps
    the exponent, which is the correct rounding up to the next binade (and to
    infinity past the largest finite value).  NaNs map to the quiet NaN 0x7FC0.
    """
    a = np.ascontiguousarray(f32, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)
    return np.where(np.isnan(a), np.uint16(0x7FC0), r)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit pattern -> the fp32 value it denotes (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_round(f32: np.ndarray) -> np.ndarray:
    """fp32 -> fp32 value of its bf16 rounding."""
    return bf16_to_f32(bf16_round_bits(f32))


# ----------------------------------------------------------------------------
# E4M3
# ----------------------------------------------------------------------------
def e4m3_decode(code: np.ndarray) -> np.ndarray:
    """E4M3 code (0..255) -> float64 value (NaN for S.1111.111)."""
    c = np.asarray(code, dtype=np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    normal = np.ldexp(1.0 + m / 8.0, e - 7)
    sub = np.ldexp(m / 8.0, -6)
    v = s * np.where(e == 0, sub, normal)
    return np.where((c & 0x7F) == 0x7F, np.nan, v)


_E4M3_POS = e4m3_decode(np.arange(0x7F))  # codes 0..126: all finite non-negative values, ascending


def _nearest_ties_even(mag: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Index into the ascending ``grid`` of the nearest value to each ``mag``
    (all mag within [grid[0], grid[-1]]), ties to the even index.  Grid index
    parity equals the code's fraction LSB for both E4M3 and E2M1."""
    hi = np.searchsorted(grid, mag, side="left")  # first grid >= mag
    hi = np.clip(hi, 0, len(grid) - 1)
    lo = np.clip(hi - 1, 0, len(grid) - 1)
    dlo = mag - grid[lo]
    dhi = grid[hi] - mag
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    exact = grid[hi] == mag
    return np.where(exact | pick_hi, hi, lo)


def e4m3_from_f32_satfinite(f32: np.ndarray) -> np.ndarray:
    """fp32 -> E4M3 code (uint8), round to nearest even, saturate to +-448.

    Distances are taken in float64, where every fp32 input and every E4M3 value
    and every midpoint between neighbours is exact, so the tie test is exact.
    """
    x = np.asarray(f32, dtype=np.float32).astype(np.float64)
    sign = np.signbit(x)
    mag = np.minimum(np.abs(x), 448.0)
    idx = _nearest_ties_even(mag, _E4M3_POS)
    code = idx.astype(np.uint8) | np.where(sign, np.uint8(0x80), np.uint8(0))
    return np.where(np.isnan(x), np.uint8(0x7F), code).astype(np.uint8)


# ----------------------------------------------------------------------------
# E2M1
# ----------------------------------------------------------------------------
E2M1_POS = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e2m1_decode(code: np.ndarray) -> np.ndarray:
    """E2M1 code (0..15) -> float64 value, from sign/exponent/fraction fields."""
    c = np.asarray(code, dtype=np.int64)
    s = np.where(c & 0x8, -1.0, 1.0)
    e = (c >> 1) & 0x3
    m = c & 0x1
    normal = np.ldexp(1.0 + m / 2.0, e - 1)
    sub = m / 2.0
    return s * np.where(e == 0, sub, normal)


def e2m1_from_f32_satfinite(f32: np.ndarray) -> np.ndarray:
    """fp32 -> E2M1 code (uint8, low nibble), round to nearest even, saturate to
    +-6.  Reading R11: a value whose magnitude rounds to 0 gets code 0 (+0),
    whatever its sign, so there is one encoding of zero."""
    x = np.asarray(f32, dtype=np.float32).astype(np.float64)
    mag = np.minimum(np.abs(x), 6.0)
    idx = _nearest_ties_even(mag, E2M1_POS).astype(np.uint8)
    neg = np.signbit(x) & (idx != 0)
    return (idx | np.where(neg, np.uint8(0x8), np.uint8(0))).astype(np.uint8)
