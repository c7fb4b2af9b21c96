"""Pins for oracle.quant: hand-derived worked examples of each storage layout,
round-trip error bounds, pack/unpack bijections, prefix invariants."""
import numpy as np

from oracle.numerics import bf16_round_bits, bf16_to_f32, e2m1_decode, e4m3_decode
from oracle.quant import (dequant_bitplane, dequant_nvfp4, dequant_w4g128, pack_bitplanes,
                          prefix_reconstruct, quantize_nvfp4, quantize_w4g128, unpack_bitplanes, unpack_w4)
from synth import normal_bf16


def _bf16(vals):
    a = np.asarray(vals, dtype=np.float32)
    b = bf16_round_bits(a)
    assert np.array_equal(bf16_to_f32(b), a), "test values must be exact in bf16"
    return b


def _weights(E, N, K, seed=7, std=0.02):
    return normal_bf16(seed, E * N * K, std).reshape(E, N, K)


# ================================================================ INT4 g128
def test_w4_worked_group_packing():
    # q[k] = (k % 15) - 7 with scale 2^-3: max|q| = 7 so scale = bf16(0.875 / 7) = 0.125 exactly,
    # u = q + 8 = (k % 15) + 1.  Words by hand: k=0..7 -> u = 1..8 -> 0x87654321;
    # k=8..15 -> 9,10,..,15,1 -> 0x1FEDCBA9; k=16..23 -> 2..9 -> 0x98765432.
    k = np.arange(128)
    w = _bf16(((k % 15) - 7) * 0.125).reshape(1, 1, 128)
    packed, s = quantize_w4g128(w)
    assert packed.shape == (1, 1, 16) and s.shape == (1, 1, 1)
    assert bf16_to_f32(s)[0, 0, 0] == 0.125
    assert packed[0, 0, 0] == 0x87654321
    assert packed[0, 0, 1] == 0x1FEDCBA9
    assert packed[0, 0, 2] == 0x98765432


def test_w4_scale_rounding_and_ties():
    # max|w| = 1: 1/7 in fp32 is 0x3E124925, which rounds down to bf16 0x3E12 = 0.142578125.
    w = np.zeros(128, dtype=np.float32)
    w[0], w[1], w[2] = 1.0, 0.5, -1.0
    packed, s = quantize_w4g128(_bf16(w).reshape(1, 1, 128))
    assert s[0, 0, 0] == 0x3E12
    q = unpack_w4(packed)[0, 0]
    # 1/0.142578125 = 7.0137 -> 7; 0.5/0.142578125 = 3.5068 -> 4
    assert list(q[:4]) == [7, 4, -7, 0]
    # exact halves round to even: scale 2^-3, w/s = 2.5 -> 2, 3.5 -> 4, -2.5 -> -2, 0.5 -> 0
    w = np.zeros(128, dtype=np.float32)
    w[:5] = np.array([0.875, 2.5, 3.5, -2.5, 0.5]) * 0.125 * np.array([8, 1, 1, 1, 1])
    packed, s = quantize_w4g128(_bf16(w).reshape(1, 1, 128))
    assert bf16_to_f32(s)[0, 0, 0] == 0.125
    assert list(unpack_w4(packed)[0, 0, :5]) == [7, 2, 4, -2, 0]


def test_w4_zero_group():
    packed, s = quantize_w4g128(np.zeros((1, 2, 256), dtype=np.uint16))
    assert np.all(s == 0) and np.all(packed == 0x88888888)
    assert np.all(dequant_w4g128(packed, s) == 0)


def test_w4_roundtrip_bound_and_bijection():
    w = _weights(3, 16, 512)
    packed, s = quantize_w4g128(w)
    wf = bf16_to_f32(w).astype(np.float64)
    wd = dequant_w4g128(packed, s)
    sf = np.repeat(bf16_to_f32(s).astype(np.float64), 128, axis=-1)
    assert np.all(np.abs(wf - wd) <= sf * (0.5 + 2.0 ** -20))
    q = unpack_w4(packed)
    assert q.min() >= -7 and q.max() <= 7
    # every group reaches |q| = 7 at its largest element
    assert np.all(np.abs(q.reshape(3, 16, 4, 128)).max(axis=-1) == 7)
    # re-pack the codes independently (python ints) and compare
    row = q[1, 5]
    words = []
    for j in range(row.size // 8):
        v = 0
        for i in range(8):
            v |= (int(row[8 * j + i]) + 8) << (4 * i)
        words.append(v)
    assert [int(x) for x in packed[1, 5]] == words


# ================================================================ bitplanes
def test_prefix_worked_examples():
    # u -> u' at b = 1, 2, 3, 4, 8 derived by hand from floor (keep top b bits) + 2^(7-b)
    table = {200: [192, 224, 208, 200, 200], 1: [64, 32, 16, 8, 1],
             255: [192, 224, 240, 248, 255], 128: [192, 160, 144, 136, 128]}
    for u, want in table.items():
        got = [int(prefix_reconstruct(np.array([u]), b)[0]) for b in (1, 2, 3, 4, 8)]
        assert got == want, (u, got, want)


def test_bitplane_worked_layout():
    # u[k] = 1 + 8k for k < 32 (q = 8k - 127, scale 2^-7 exactly since max|q| = 127), u = 128 after.
    # plane 0 = bit 7: u >= 128 iff k >= 16 -> 0xFFFF0000; plane 7 = bit 0: always 1 -> 0xFFFFFFFF;
    # plane 4 = bit 3 of 1 + 8k = bit 0 of k -> odd k -> 0xAAAAAAAA; plane 3 = bit 4 = bit 1 of k -> 0xCCCCCCCC.
    k = np.arange(128)
    q = np.where(k < 32, 8 * k - 127, 0)
    w = _bf16(q * 2.0 ** -7).reshape(1, 1, 128)
    planes, s = pack_bitplanes(w)
    assert planes.shape == (1, 8, 1, 4)
    assert bf16_to_f32(s)[0, 0, 0] == 2.0 ** -7
    assert planes[0, 0, 0, 0] == 0xFFFF0000
    assert planes[0, 7, 0, 0] == 0xFFFFFFFF
    assert planes[0, 4, 0, 0] == 0xAAAAAAAA
    assert planes[0, 3, 0, 0] == 0xCCCCCCCC
    # words 1..3 hold u = 128 = 0b10000000: plane 0 all ones, the others zero
    assert np.all(planes[0, 0, 0, 1:] == 0xFFFFFFFF) and np.all(planes[0, 1:, 0, 1:] == 0)


def test_bitplane_b8_equals_full_code_and_bound():
    w = _weights(2, 8, 256, seed=11)
    planes, s = pack_bitplanes(w)
    wf = bf16_to_f32(w).astype(np.float64)
    sf = np.repeat(bf16_to_f32(s).astype(np.float64), 128, axis=-1)
    full = dequant_bitplane(planes, s, 8)
    assert np.all(np.abs(wf - full) <= sf * (0.5 + 2.0 ** -20))
    u = unpack_bitplanes(planes, 8)
    assert u.min() >= 1 and u.max() <= 255
    assert np.array_equal(full, sf * (u - 128))


def test_bitplane_prefixes_are_top_bits():
    w = _weights(2, 8, 256, seed=12)
    planes, s = pack_bitplanes(w)
    u = unpack_bitplanes(planes, 8)
    for b in range(1, 9):
        top = unpack_bitplanes(planes, b)
        assert np.array_equal(top, (u >> (8 - b)) << (8 - b))
        rec = prefix_reconstruct(u, b)
        assert np.all(np.abs(rec - u) <= (1 << (7 - b)) if b < 8 else rec == u)
        d = dequant_bitplane(planes, s, b)
        sf = np.repeat(bf16_to_f32(s).astype(np.float64), 128, axis=-1)
        assert np.array_equal(d, sf * (rec - 128))


def test_bitplane_zero_group():
    planes, s = pack_bitplanes(np.zeros((1, 1, 128), dtype=np.uint16))
    assert np.all(s == 0)
    assert np.all(planes[0, 0] == 0xFFFFFFFF) and np.all(planes[0, 1:] == 0)  # u = 128


# ================================================================ NVFP4
def test_nvfp4_worked_example():
    # tensor amax 2.625 = 2688 * 2^-10 -> g = 2^-10 exactly; 6g = 6 * 2^-10.
    # block 0: amax 2.625 -> 2.625 / (6 * 2^-10) = 448 -> sb = 0x7E (448); v = w / (448 * 2^-10)
    # block 1: amax 0.375 -> 64 -> sb = 0x68 (2^6, exponent field 13); v = 16 w:
    #   0.375 -> 6 (code 7), 0.1875 -> 3 (5), 0.03125 -> 0.5 (1), 0.0390625 -> 0.625 -> 0.5 (1),
    #   -0.125 -> -2 (0xC), 0 -> 0 (0)
    w = np.zeros((1, 1, 32), dtype=np.float32)
    w[0, 0, 0] = 2.625
    w[0, 0, 1] = 0.4375  # v = 0.4375 * 1024 / 448 = 1.0 -> code 2
    w[0, 0, 16:22] = [0.375, 0.1875, 0.03125, 0.0390625, -0.125, 0.0]
    codes, sb, g = quantize_nvfp4(_bf16(w))
    assert g[0] == np.float32(2.0 ** -10)
    assert list(sb[0, 0]) == [0x7E, 0x68]
    assert e4m3_decode(0x68) == 64.0
    lo, hi = codes[0, 0] & 0xF, codes[0, 0] >> 4
    assert lo[0] == 7 and hi[0] == 2  # 2.625 -> v = 6; 0.4375 -> v = 1
    assert list(lo[8:11]) == [7, 1, 0xC] and list(hi[8:11]) == [5, 1, 0]


def test_nvfp4_roundtrip_bound():
    w = _weights(2, 16, 256, seed=13)
    codes, sb, g = quantize_nvfp4(w)
    wf = bf16_to_f32(w).astype(np.float64)
    wd = dequant_nvfp4(codes, sb, g)
    scale = np.repeat(e4m3_decode(sb) * g.astype(np.float64)[:, None, None], 16, axis=-1)
    v = wf / scale
    # half the E2M1 grid spacing at |v|: 0.25 below 2, 0.5 below 4, 1 up to 6 (plus fp32 rounding of v)
    half = np.where(np.abs(v) < 2, 0.25, np.where(np.abs(v) < 4, 0.5, 1.0))
    over = np.maximum(np.abs(v) - 6, 0)
    assert np.all(np.abs(wf - wd) <= (half + over + 1e-6) * scale)
    vals = e2m1_decode(np.concatenate([codes & 0xF, codes >> 4], axis=-1))
    assert np.abs(vals).max() == 6.0


def test_nvfp4_zero_tensor_and_zero_block():
    w = np.zeros((2, 1, 32), dtype=np.float32)
    w[1, 0, 0] = 1.0  # expert 1: block 0 nonzero, block 1 all zero
    codes, sb, g = quantize_nvfp4(_bf16(w))
    assert g[0] == 0 and np.all(sb[0] == 0) and np.all(codes[0] == 0)
    assert sb[1, 0, 1] == 0 and np.all(codes[1, 0, 8:] == 0)
    assert np.all(dequant_nvfp4(codes, sb, g)[0] == 0)


def _golden(name):
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", name)
    rows = [l.split() for l in open(path) if l.strip() and not l.startswith("#")]
    return [[float(v) for v in r] for r in rows]


def test_prefix_golden_table():
    for row in _golden("bitplane_prefix.txt"):
        u, want = int(row[0]), [int(v) for v in row[1:]]
        assert [int(prefix_reconstruct(np.array([u]), b)[0]) for b in (1, 2, 3, 4, 8)] == want
