"""Pins of the W4A4 (NVFP4 activations) oracle: a hand-worked activation tensor whose
scales and codes follow from the recipe by hand, the quantisation error bound, the block
scaled product against exact rational arithmetic, and the grouped FFN against a dense
brute force that never permutes."""
from fractions import Fraction

import numpy as np
import pytest

import synth
from oracle.ffn import FMT_NVFP4, Experts
from oracle.numerics import e2m1_decode, e4m3_decode
from oracle.quant import quantize_nvfp4
from oracle.routing import permute, router_logits, topk_softmax
from oracle.w4a4 import dequant_act_nvfp4, quantize_act_nvfp4, w4a4_gemm, w4a4_grouped_ffn


def _codes(packed):
    c = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), np.uint8)
    c[..., 0::2] = packed & 0xF
    c[..., 1::2] = packed >> 4
    return c


def test_hand_worked_activation_tensor():
    # amax 6 => g = 6 / 2688; block 0 (amax 6) => sb = 448, elements / (448 g) = themselves;
    # block 1 (amax 3) => sb = 224, elements are doubled before E2M1 rounding
    row0 = [6, 3, -1.5, 0.5, 0, 4, -6, 2, 1, -1, 0.5, 0, 0, 0, 0, 0]
    row1 = [3, 1.5, -0.75, 0.25, 0, 2, -3, 1, 0.5, -0.5, 0.25, 0, 0, 0, 0, 0]
    a = np.array([row0 + row1], dtype=np.float32)
    codes, sb, g = quantize_act_nvfp4(a)
    assert g == np.float32(np.float32(6) / np.float32(6 * 448))
    assert e4m3_decode(sb).tolist() == [[448.0, 224.0]]
    vals = e2m1_decode(_codes(codes))[0]
    assert vals[:16].tolist() == row0
    assert vals[16:].tolist() == [2 * v for v in row1]
    # 448 g and 224 g are 1 and 1/2 up to the fp32 rounding of g
    np.testing.assert_allclose(dequant_act_nvfp4(codes, sb, g), a, rtol=1e-6)


def test_zero_tensor_and_zero_block():
    a = np.zeros((2, 32), np.float32)
    codes, sb, g = quantize_act_nvfp4(a)
    assert g == 0 and not codes.any() and not sb.any()
    a[1, 16:] = np.linspace(-1, 1, 16, dtype=np.float32)
    codes, sb, g = quantize_act_nvfp4(a)
    assert not sb[0].any() and not sb[1, 0] and sb[1, 1]


@pytest.mark.parametrize("seed", range(4))
def test_quantisation_error_within_one_block_unit(seed):
    a = (np.random.default_rng(seed).standard_normal((8, 64)) * 3).astype(np.float32)
    codes, sb, g = quantize_act_nvfp4(a)
    unit = np.repeat(e4m3_decode(sb) * float(g), 16, axis=1)  # E4M3 scale x g per element
    err = np.abs(dequant_act_nvfp4(codes, sb, g) - a)
    assert np.all(err <= unit * 1.0 + 1e-12)        # half of the widest E2M1 step (2) is 1 unit
    assert np.max(err / np.maximum(np.abs(a), 1e-30)) > 0  # and quantisation did something


def test_block_scaled_product_is_exact():
    rng = np.random.default_rng(11)
    R, N, K = 3, 2, 32
    a = (rng.standard_normal((R, K)) * 2).astype(np.float32)
    w_bits = synth.normal_bf16(12, N * K, 0.5).reshape(1, N, K)
    ac, asb, ag = quantize_act_nvfp4(a)
    wc, wsb, wg = quantize_nvfp4(w_bits)
    got = w4a4_gemm(ac, asb, ag, wc[0], wsb[0], wg[0])
    av, wv = e2m1_decode(_codes(ac)), e2m1_decode(_codes(wc[0]))
    sa, sw = e4m3_decode(asb), e4m3_decode(wsb[0])
    for r in range(R):
        for n in range(N):
            tot = Fraction(0)
            for kk in range(K):
                tot += (Fraction(float(av[r, kk])) * Fraction(float(sa[r, kk // 16])) *
                        Fraction(float(wv[n, kk])) * Fraction(float(sw[n, kk // 16])))
            want = float(tot * Fraction(float(ag)) * Fraction(float(wg[0])))
            assert got[r, n] == pytest.approx(want, rel=1e-15, abs=1e-300)


def test_grouped_w4a4_ffn_matches_dense_brute_force():
    T, H, I, E, k = 6, 256, 32, 4, 2
    x = synth.normal_bf16(21, T * H, 1.0).reshape(T, H)
    wr = synth.normal_bf16(22, E * H, 0.05).reshape(E, H)
    w13 = synth.normal_bf16(23, E * 2 * I * H, 0.05).reshape(E, 2 * I, H)
    w2 = synth.normal_bf16(24, E * H * I, 0.05).reshape(E, H, I)
    a, b = quantize_nvfp4(w13), quantize_nvfp4(w2)
    ex = Experts(FMT_NVFP4, a[0], a[1], b[0], b[1], a[2], b[2])
    ids, _ = topk_softmax(router_logits(x, wr), k)
    offsets, sp, _ = permute(ids, E)
    y = w4a4_grouped_ffn(x, offsets, sp, k, ex)
    # dense: every pair in pair order, no permutation; h quantised over the same rows
    from oracle.numerics import bf16_to_f32
    xq = dequant_act_nvfp4(*quantize_act_nvfp4(bf16_to_f32(x)))
    hs = []
    for t in range(T):
        for j in range(k):
            e = int(ids[t, j])
            W13, _ = ex.dequant(e)
            gu = np.array([np.dot(xq[t], W13[n]) for n in range(2 * I)])
            g_, u_ = gu[:I], gu[I:]
            hs.append((g_ / (1 + np.exp(-g_)) * u_).astype(np.float32))
    hq = dequant_act_nvfp4(*quantize_act_nvfp4(np.stack(hs)))
    for t in range(T):
        for j in range(k):
            p = t * k + j
            _, W2 = ex.dequant(int(ids[t, j]))
            want = np.array([np.dot(hq[p], W2[m]) for m in range(H)])
            r = int(np.nonzero(sp == p)[0][0])
            np.testing.assert_allclose(y[r], want, rtol=1e-9, atol=1e-12)


def test_one_scale_for_the_whole_tensor():
    # a second row with amax 0.75 shares the tensor's g (from amax 6): its block scale is
    # E4M3(0.75 / (6 g)) = 56, not the 448 a per-row scale would give
    a = np.zeros((2, 16), np.float32)
    a[0, 0], a[1, 0], a[1, 1] = 6.0, 0.75, -0.375
    codes, sb, g = quantize_act_nvfp4(a)
    assert e4m3_decode(sb).tolist() == [[448.0], [56.0]]
    assert e2m1_decode(_codes(codes))[1, :2].tolist() == [6.0, -3.0]
