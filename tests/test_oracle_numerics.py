"""Pins for oracle.numerics: bf16 / E4M3 / E2M1 conversions against their
definitions, exhaustive enumeration and an independent library routine (torch's
own dtype conversions, which share no code with the oracle)."""
import numpy as np
import pytest
import torch

from oracle.numerics import (E2M1_POS, bf16_round_bits, bf16_to_f32, e2m1_decode,
                             e2m1_from_f32_satfinite, e4m3_decode, e4m3_from_f32_satfinite)


def _rand_f32(n, seed=0, scale=1.0):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal(n) * scale).astype(np.float32)


# ---------------------------------------------------------------- bf16
def test_bf16_matches_torch_on_random_values():
    x = np.concatenate([_rand_f32(200000, 1), _rand_f32(50000, 2, 1e-30), _rand_f32(50000, 3, 1e30)])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bf16_round_bits(x), ref)


def test_bf16_halfway_cases_round_to_even():
    # 1 + 2^-8 is exactly halfway between bf16 1.0 (0x3F80) and 1.0078125 (0x3F81): even -> 0x3F80
    # 1 + 3*2^-8 is halfway between 0x3F81 and 0x3F82: even -> 0x3F82
    vals = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8), 1 + 2.0 ** -8 + 2.0 ** -20],
                    dtype=np.float32)
    assert list(bf16_round_bits(vals)) == [0x3F80, 0x3F82, 0xBF80, 0x3F81]


def test_bf16_roundtrip_is_identity_on_every_finite_pattern():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    f = bf16_to_f32(bits)
    finite = np.isfinite(f)
    assert np.array_equal(bf16_round_bits(f[finite]), bits[finite])


def test_bf16_overflow_to_inf_and_nan():
    big = np.array([3.4e38, np.inf, -np.inf, np.nan], dtype=np.float32)
    r = bf16_round_bits(big)
    assert r[0] == 0x7F80 and r[1] == 0x7F80 and r[2] == 0xFF80 and r[3] == 0x7FC0


# ---------------------------------------------------------------- E4M3
def test_e4m3_decode_known_codes():
    # Closed forms from the field layout: 0x38 = 2^0, 0x7E = 1.75 * 2^8, 0x01 = 2^-9 (min subnormal),
    # 0x08 = 2^-6 (min normal), 0x07 = 7/8 * 2^-6 (max subnormal).
    assert e4m3_decode(0x38) == 1.0
    assert e4m3_decode(0x7E) == 448.0
    assert e4m3_decode(0x01) == 2.0 ** -9
    assert e4m3_decode(0x08) == 2.0 ** -6
    assert e4m3_decode(0x07) == 7 / 8 * 2.0 ** -6
    assert e4m3_decode(0xB8) == -1.0
    assert np.isnan(e4m3_decode(0x7F)) and np.isnan(e4m3_decode(0xFF))


def test_e4m3_decode_matches_torch_for_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = e4m3_decode(codes)
    assert np.array_equal(np.isnan(ref), np.isnan(mine))
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], mine[ok])


def test_e4m3_encode_matches_torch_inside_range():
    x = np.concatenate([_rand_f32(100000, 4, 30.0), _rand_f32(50000, 5, 0.01), _rand_f32(20000, 6, 1e-3)])
    x = x[np.abs(x) <= 448]
    # midpoints between every pair of neighbouring codes: the tie rule decides each one
    pos = e4m3_decode(np.arange(0x7F))
    mids = ((pos[1:] + pos[:-1]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids, pos.astype(np.float32)])
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    mine = e4m3_from_f32_satfinite(x)
    # torch keeps the sign of zero; the oracle does too for E4M3
    assert np.array_equal(mine, ref)


def test_e4m3_saturates():
    x = np.array([448.0, 449.0, 463.99, 464.0, 1e6, -1e6, 3.0e38], dtype=np.float32)
    assert list(e4m3_from_f32_satfinite(x)) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0x7E]


# ---------------------------------------------------------------- E2M1
def test_e2m1_decode_all_codes():
    vals = e2m1_decode(np.arange(16))
    assert list(vals[:8]) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert list(vals[8:]) == [-0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]


def test_e2m1_tie_table():
    # every midpoint between neighbours goes to the even code (fraction bit 0)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], dtype=np.float32)
    want = [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0]
    got = e2m1_decode(e2m1_from_f32_satfinite(mids))
    assert list(got) == want
    assert list(e2m1_decode(e2m1_from_f32_satfinite(-mids))) == [-v if v else 0.0 for v in want]


def test_e2m1_bruteforce_nearest():
    x = np.linspace(-7, 7, 20001).astype(np.float32)
    got = e2m1_decode(e2m1_from_f32_satfinite(x))
    grid = np.concatenate([-E2M1_POS[::-1], E2M1_POS])
    xc = np.clip(x.astype(np.float64), -6, 6)
    dist = np.abs(xc[:, None] - grid[None, :])
    best = dist.min(axis=1)
    assert np.all(np.abs(got - xc) == best)  # got is one of the nearest
    assert np.all(np.abs(x[np.abs(x) > 6]) > 6) and np.all(np.abs(got[np.abs(x) >= 6]) == 6)


def test_e2m1_zero_is_positive():
    codes = e2m1_from_f32_satfinite(np.array([-0.0, -0.1, -0.25, 0.1], dtype=np.float32))
    assert list(codes) == [0, 0, 0, 0]
    assert e2m1_from_f32_satfinite(np.array([-0.26], dtype=np.float32))[0] == 0x9


def test_e2m1_golden_ties():
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "e2m1_ties.txt")
    rows = [l.split() for l in open(path) if l.strip() and not l.startswith("#")]
    x = np.array([float(r[0]) for r in rows], dtype=np.float32)
    want = [float(r[1]) for r in rows]
    assert list(e2m1_decode(e2m1_from_f32_satfinite(x))) == want
