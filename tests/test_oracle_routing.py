"""Pins for oracle.routing: the fixed fp32 summation order, top-k and its
weights, the bit-width rule and the stable permutation, against hand-derived
values, exact integer arithmetic, float64 and brute force."""
import math

import numpy as np

from oracle.numerics import bf16_round_bits, bf16_to_f32
from oracle.routing import (active_experts, permute, router_logits, router_logits_f64, select_bits,
                            topk_softmax)
from synth import normal_bf16


def _bf16(vals):
    a = np.asarray(vals, dtype=np.float32)
    b = bf16_round_bits(a)
    assert np.array_equal(bf16_to_f32(b), a)
    return b


def test_summation_order_worked_example():
    # H = 256: lane L owns h = 8L .. 8L+7.  Put x*w = 2^24 at h = 0 (lane 0), 1 at h = 8 (lane 1),
    # -2^24 at h = 16 (lane 2).  Pairwise by distance 16, 8, 4 changes nothing; distance 2 gives
    # lane0 + lane2 = 0 and lane1 + lane3 = 1; distance 1 gives 0 + 1 = 1.
    # A left-to-right sum would give fl(2^24 + 1) - 2^24 = 0 instead.
    x = np.zeros((1, 256), dtype=np.float32)
    w = np.zeros((1, 256), dtype=np.float32)
    x[0, [0, 8, 16]] = [4096.0, 1.0, -4096.0]
    w[0, [0, 8, 16]] = [4096.0, 1.0, 4096.0]
    assert router_logits(_bf16(x), _bf16(w))[0, 0] == 1.0
    # within one lane the order is sequential: h = 0, 1, 2 in lane 0 gives fl(fl(2^24 + 1) - 2^24) = 0
    x = np.zeros((1, 256), dtype=np.float32)
    x[0, [0, 1, 2]] = [4096.0, 1.0, -4096.0]
    w = np.zeros((1, 256), dtype=np.float32)
    w[0, [0, 1, 2]] = [4096.0, 1.0, 4096.0]
    assert router_logits(_bf16(x), _bf16(w))[0, 0] == 0.0
    # the j loop is outer: h = 0 (j=0) then h = 256 (j=1) in lane 0
    x = np.zeros((1, 512), dtype=np.float32)
    w = np.zeros((1, 512), dtype=np.float32)
    x[0, [0, 1, 256]] = [4096.0, -4096.0, 1.0]
    w[0, [0, 1, 256]] = [4096.0, 4096.0, 1.0]
    assert router_logits(_bf16(x), _bf16(w))[0, 0] == 1.0  # (2^24 - 2^24) + 1


def test_integer_inputs_give_exact_dot_products():
    rng = np.random.default_rng(3)
    T, E, H = 5, 7, 512
    x = rng.integers(-8, 9, size=(T, H)).astype(np.float32)
    w = rng.integers(-8, 9, size=(E, H)).astype(np.float32)
    bias = rng.integers(-4, 5, size=E).astype(np.float32)
    got = router_logits(_bf16(x), _bf16(w), bias)
    exact = [[sum(int(a) * int(b) for a, b in zip(x[t], w[e])) + int(bias[e]) for e in range(E)]
             for t in range(T)]
    assert np.array_equal(got, np.array(exact, dtype=np.float32))


def test_logits_close_to_float64():
    T, E, H = 6, 16, 1024
    x = normal_bf16(21, T * H, 1.0).reshape(T, H)
    w = normal_bf16(22, E * H, 0.02).reshape(E, H)
    l32 = router_logits(x, w).astype(np.float64)
    l64 = router_logits_f64(x, w)
    mag = np.abs(bf16_to_f32(x).astype(np.float64)) @ np.abs(bf16_to_f32(w).astype(np.float64)).T
    assert np.all(np.abs(l32 - l64) <= mag * 64 * 2.0 ** -24)  # ~ (H/32 + 5) roundings


def test_topk_bruteforce_ties_and_weights():
    rng = np.random.default_rng(4)
    T, E, k = 40, 12, 4
    l = rng.integers(-3, 4, size=(T, E)).astype(np.float32)  # many exact ties
    ids, w = topk_softmax(l, k)
    for t in range(T):
        ref = sorted(range(E), key=lambda e: (-float(l[t, e]), e))[:k]
        assert list(ids[t]) == ref
        ex = [math.exp(float(l[t, e])) for e in range(E)]
        full = [v / sum(ex) for v in ex]
        renorm = [full[e] / sum(full[i] for i in ref) for e in ref]
        assert np.allclose(w[t], renorm, rtol=0, atol=1e-7)
    assert np.allclose(w.sum(-1), 1.0, atol=1e-6)
    assert np.all(np.diff(w, axis=-1) <= 0)
    assert all(len(set(r)) == k for r in ids.tolist())


def test_select_bits_thresholds():
    t = [np.float32(0.05), np.float32(0.15), np.float32(0.30)]
    below = [np.nextafter(v, np.float32(0)) for v in t]
    w = np.array([[0.0, below[0], t[0], below[1], t[1], below[2], t[2], 1.0]], dtype=np.float32)
    assert list(select_bits(w)[0]) == [2, 2, 3, 3, 4, 4, 8, 8]


def test_permute_bruteforce_and_invariants():
    rng = np.random.default_rng(5)
    for T, E, k in [(1, 4, 1), (7, 9, 3), (33, 16, 8), (64, 64, 8)]:
        ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
        offsets, sp, p2r = permute(ids, E)
        pairs = [(int(ids[p // k, p % k]), p) for p in range(T * k)]
        ref = [p for _, p in sorted(pairs)]
        assert list(sp) == ref
        assert np.array_equal(p2r[sp], np.arange(T * k))
        assert offsets[0] == 0 and offsets[-1] == T * k
        for e in range(E):
            seg = sp[offsets[e]:offsets[e + 1]]
            assert np.all(ids.reshape(-1)[seg] == e) and np.all(np.diff(seg) > 0)
        # every token appears exactly k times
        assert np.array_equal(np.bincount(sp // k, minlength=T), np.full(T, k))
        assert list(active_experts(offsets)) == sorted(set(ids.reshape(-1).tolist()))
