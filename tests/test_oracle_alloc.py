"""Pins of the budgeted bit allocation oracle (oracle/alloc.py) against brute force,
hand-worked examples and the optimality property of a Lagrangian allocation."""
import itertools
from fractions import Fraction

import numpy as np
import pytest

import synth
from oracle.alloc import (activation_moments, allocate_bits, bitplane_distortion, choose, expand_bits,
                          expert_counts, expert_distortion, read_rate)
from oracle.numerics import bf16_to_f32
from oracle.quant import pack_bitplanes


def test_distortion_matches_integer_brute_force():
    # one expert, three rows, two groups; every term recomputed with exact rationals
    w = synth.normal_bf16(41, 3 * 256, 0.02).reshape(1, 3, 256)
    planes, s_bits = pack_bitplanes(w)
    delta = bitplane_distortion(planes, s_bits)
    # the full codes from the planes, bit by bit
    u = np.zeros((3, 256), dtype=np.int64)
    for p in range(8):
        for n in range(3):
            for k in range(256):
                u[n, k] |= ((int(planes[0, p, n, k // 32]) >> (k % 32)) & 1) << (7 - p)
    s = bf16_to_f32(s_bits[0])
    for b in (1, 2, 3, 5, 8):
        for k in (0, 7, 127, 128, 200, 255):
            tot = Fraction(0)
            for n in range(3):
                ub = ((int(u[n, k]) >> (8 - b)) << (8 - b)) + ((1 << (7 - b)) if b < 8 else 0)
                err = Fraction(float(s[n, k // 128])) * (ub - int(u[n, k]))
                tot += err * err
            assert delta[0, b - 1, k] == pytest.approx(float(tot), rel=1e-15, abs=0.0)
    assert np.all(delta[:, 7, :] == 0.0)  # the 8-bit prefix is the full code


def test_activation_moments_worked_example():
    x = np.array([[1.0, -1.0, 2.0], [3.0, 0.0, -2.0]], dtype=np.float32)
    xb = (x.view(np.uint32) >> 16).astype(np.uint16)  # exact in bf16
    assert np.array_equal(activation_moments(xb), np.array([5.0, 0.5, 4.0]))


def test_allocation_worked_example():
    # dropping expert 1 to 2 bits costs 4 per unit frequency, expert 0 costs 10: a budget
    # of 5 bits per weight (one expert at 2, one at 8) keeps expert 0 at 8 bits
    D = np.array([[10.0, 0.0], [4.0, 0.0]])
    n = np.array([3, 3])
    bits, lam = allocate_bits(D, n, (2, 8), 5.0)   # rate exactly at the budget: within it
    assert bits.tolist() == [8, 2]
    assert 4.0 / 6.0 < lam <= 10.0 / 6.0 + 1e-12
    assert allocate_bits(D, n, (2, 8), 4.999)[0].tolist() == [2, 2]
    assert allocate_bits(D, n, (2, 8), 8.0)[0].tolist() == [8, 8]    # budget covers everything
    assert allocate_bits(D, n, (2, 8), 1.0)[0].tolist() == [2, 2]    # infeasible: the smallest
    assert allocate_bits(D, np.array([5, 0]), (2, 8), 8.0)[0].tolist() == [8, 2]  # unread expert


def test_ties_go_to_the_larger_width():
    D = np.array([[6.0, 0.0]])
    assert choose(D, (2, 8), 1.0).tolist() == [1]  # 6 + 2 == 0 + 8
    assert choose(D, (2, 8), 1.0 + 1e-9).tolist() == [0]


@pytest.mark.parametrize("seed", range(6))
def test_allocation_is_optimal_at_its_own_rate(seed):
    # Lagrangian sandwich: no allocation of rate <= the chosen one has lower distortion
    rng = np.random.default_rng(seed)
    choices = (2, 3, 4, 8)
    E = 4
    D = np.sort(rng.random((E, 4)) * 10, axis=1)[:, ::-1].copy()  # more bits, less distortion
    n = rng.integers(1, 50, size=E)
    f = n / n.sum()
    budget = float(rng.uniform(2.5, 7.5))
    bits, lam = allocate_bits(D, n, choices, budget)
    idx = np.array([choices.index(int(b)) for b in bits])
    rate = read_rate(idx, f, choices)
    dist = float(np.sum(f * D[np.arange(E), idx]))
    assert rate <= budget + 1e-12
    for combo in itertools.product(range(4), repeat=E):
        c = np.array(combo)
        if read_rate(c, f, choices) <= rate + 1e-12:
            assert float(np.sum(f * D[np.arange(E), c])) >= dist - 1e-12


def test_more_budget_never_lowers_a_width():
    rng = np.random.default_rng(9)
    D = np.sort(rng.random((16, 4)) * 10, axis=1)[:, ::-1].copy()
    n = rng.integers(1, 50, size=16)
    prev = None
    for budget in np.linspace(2.0, 8.0, 25):
        bits = allocate_bits(D, n, (2, 3, 4, 8), float(budget))[0].astype(int)
        if prev is not None:
            assert np.all(bits >= prev)
        prev = bits


def test_frequencies_and_expansion():
    offsets = np.array([0, 3, 3, 8])
    assert expert_counts(offsets).tolist() == [3, 0, 5]
    ids = np.array([[2, 0], [0, 1]])
    assert expand_bits(ids, np.array([4, 2, 8], np.uint8)).tolist() == [8, 4, 4, 2]


def test_end_to_end_distortion_dot_products():
    w = synth.normal_bf16(43, 2 * 4 * 256, 0.02).reshape(2, 4, 256)
    planes, s_bits = pack_bitplanes(w)
    delta = bitplane_distortion(planes, s_bits)
    m = activation_moments(synth.normal_bf16(44, 5 * 256, 1.0).reshape(5, 256))
    D = expert_distortion(delta, m, (2, 4, 8))
    assert D.shape == (2, 3) and np.all(D[:, 2] == 0.0)
    assert D[0, 0] == pytest.approx(float(delta[0, 1] @ m), rel=1e-15)


def test_expert_distortion_against_explicit_sums():
    import math
    rng = np.random.default_rng(17)
    delta = rng.random((3, 8, 40))
    m = rng.random(40)
    choices = (1, 5, 8)
    D = expert_distortion(delta, m, choices)
    for e in range(3):
        for c, b in enumerate(choices):
            assert D[e, c] == pytest.approx(math.fsum(m[k] * delta[e, b - 1, k] for k in range(40)), rel=1e-14)


def test_read_rate_does_not_increase_with_lambda():
    rng = np.random.default_rng(23)
    D = np.sort(rng.random((32, 4)) * 10, axis=1)[:, ::-1].copy()
    f = rng.random(32)
    f /= f.sum()
    rates = [read_rate(choose(D, (2, 3, 4, 8), lam), f, (2, 3, 4, 8)) for lam in np.linspace(0.0, 12.0, 200)]
    assert all(b <= a + 1e-15 for a, b in zip(rates, rates[1:]))
    assert rates[0] == pytest.approx(8.0) and rates[-1] == pytest.approx(2.0)


def test_routing_frequency_cancels():
    # scaling every expert's pair count by the same factor leaves every decision unchanged
    rng = np.random.default_rng(31)
    D = np.sort(rng.random((24, 4)) * 10, axis=1)[:, ::-1].copy()
    n = rng.integers(0, 40, size=24)
    for budget in (2.3, 3.1, 4.6, 6.0):
        a = allocate_bits(D, n, (2, 3, 4, 8), budget)[0]
        b = allocate_bits(D, 7 * n, (2, 3, 4, 8), budget)[0]
        assert np.array_equal(a, b)
