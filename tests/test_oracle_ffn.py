"""Pins for oracle.ffn: the grouped path against a dense brute force that never
permutes, the single-expert case against a dense SwiGLU MLP evaluated with
torch's own silu and float64 matmul, and combine / stack invariants."""
import numpy as np
import torch

from oracle.ffn import (FMT_BITPLANE8, FMT_NVFP4, FMT_W4G128, Experts, combine, dense_bruteforce,
                        grouped_ffn, moe_layer, stack_layer_step)
from oracle.numerics import bf16_round_bits, bf16_to_f32
from oracle.quant import pack_bitplanes, quantize_nvfp4, quantize_w4g128
from oracle.routing import permute, select_bits, topk_softmax, router_logits
from synth import normal_bf16


def make_experts(fmt, E, H, I, seed=31, std=0.02):
    w13 = normal_bf16(seed, E * 2 * I * H, std).reshape(E, 2 * I, H)
    w2 = normal_bf16(seed + 1, E * H * I, std).reshape(E, H, I)
    if fmt == FMT_W4G128:
        a, b = quantize_w4g128(w13), quantize_w4g128(w2)
        return Experts(fmt, a[0], a[1], b[0], b[1])
    if fmt == FMT_BITPLANE8:
        a, b = pack_bitplanes(w13), pack_bitplanes(w2)
        return Experts(fmt, a[0], a[1], b[0], b[1])
    a, b = quantize_nvfp4(w13), quantize_nvfp4(w2)
    return Experts(fmt, a[0], a[1], b[0], b[1], a[2], b[2])


def _tiny_case(fmt, T=9, E=6, k=3, H=256, I=128, seed=40):
    x = normal_bf16(seed, T * H, 1.0).reshape(T, H)
    wr = normal_bf16(seed + 1, E * H, 0.02).reshape(E, H)
    return x, wr, make_experts(fmt, E, H, I, seed=seed + 2)


def test_grouped_equals_dense_bruteforce_all_formats():
    for fmt in (FMT_W4G128, FMT_BITPLANE8, FMT_NVFP4):
        T, k = 9, 3
        x, wr, ex = _tiny_case(fmt, T=T, k=k)
        out, r = moe_layer(x, wr, None, ex, k)
        ref = dense_bruteforce(x, r.weights, r.ids, ex, r.bits)
        assert np.allclose(out, ref, rtol=1e-12, atol=1e-12), fmt


def test_bitplane_mixed_precision_pairs():
    T, E, k, H, I = 12, 5, 4, 256, 128
    x, wr, ex = _tiny_case(FMT_BITPLANE8, T=T, E=E, k=k, H=H, I=I, seed=50)
    logits = router_logits(x, wr)
    ids, w = topk_softmax(logits, k)
    rng = np.random.default_rng(0)
    bits = rng.choice(np.array([2, 3, 4, 8], dtype=np.uint8), size=(T, k))
    offsets, sp, p2r = permute(ids, E)
    y = grouped_ffn(x, offsets, sp, k, ex, bits)
    out = combine(y, w, p2r)
    ref = dense_bruteforce(x, w, ids, ex, bits)
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12)
    # at all-8 bits the result differs from all-2 bits (the prefix length is honoured)
    y8 = grouped_ffn(x, offsets, sp, k, ex, np.full((T, k), 8, np.uint8))
    y2 = grouped_ffn(x, offsets, sp, k, ex, np.full((T, k), 2, np.uint8))
    assert np.abs(y8 - y2).max() > 1e-3


def test_single_expert_equals_torch_swiglu_mlp():
    # E = 1, k = 1: the layer is a dense SwiGLU MLP.  Weights are s * q with s = 2^-3 and integer
    # q in [-7, 7] reaching |q| = 7 in every group, so W4 quantisation is exact and the torch
    # reference can use the original bf16 weights without any of the oracle's dequantisation.
    T, H, I = 5, 256, 128
    rng = np.random.default_rng(8)

    def exact_w4(n, kdim):
        q = rng.integers(-7, 8, size=(n, kdim))
        q[:, ::128] = 7
        return (q * 0.125).astype(np.float32)

    wg, wu, w2 = exact_w4(I, H), exact_w4(I, H), exact_w4(H, I)
    w13 = np.concatenate([wg, wu], axis=0)
    x = normal_bf16(9, T * H, 1.0).reshape(T, H)
    wr = np.zeros((1, H), dtype=np.uint16)
    a, b = quantize_w4g128(bf16_round_bits(w13)[None]), quantize_w4g128(bf16_round_bits(w2)[None])
    ex = Experts(FMT_W4G128, a[0], a[1], b[0], b[1])
    out, r = moe_layer(x, wr, None, ex, 1)
    assert np.all(r.weights == 1.0)
    xt = torch.from_numpy(bf16_to_f32(x).astype(np.float64))
    ref = (torch.nn.functional.silu(xt @ torch.from_numpy(wg.astype(np.float64)).T)
           * (xt @ torch.from_numpy(wu.astype(np.float64)).T)) @ torch.from_numpy(w2.astype(np.float64)).T
    assert np.allclose(out, ref.numpy(), rtol=1e-12, atol=1e-9)


def test_combine_one_hot_and_residual():
    T, k, H = 4, 3, 8
    y = np.arange(T * k * H, dtype=np.float64).reshape(T * k, H)
    p2r = np.array([5, 0, 11, 3, 7, 1, 2, 9, 4, 8, 6, 10], dtype=np.int32)
    w = np.zeros((T, k), dtype=np.float32)
    w[:, 1] = 1.0
    res = bf16_round_bits(np.full((T, H), 0.5, dtype=np.float32))
    out = combine(y, w, p2r, res)
    for t in range(T):
        assert np.array_equal(out[t], y[p2r[t * k + 1]] + 0.5)


def test_stack_with_zero_experts_is_identity():
    T, E, k, H, I = 3, 4, 2, 256, 128
    x = normal_bf16(60, T * H, 1.0).reshape(T, H)
    wr = normal_bf16(61, E * H, 0.02).reshape(E, H)
    z13, z2 = np.zeros((E, 2 * I, H), np.uint16), np.zeros((E, H, I), np.uint16)
    a, b = quantize_w4g128(z13), quantize_w4g128(z2)
    ex = Experts(FMT_W4G128, a[0], a[1], b[0], b[1])
    cur = x
    for _ in range(3):
        cur, _r = stack_layer_step(cur, wr, ex, k)
    assert np.array_equal(cur, x)


def test_bit_rule_uses_routing_weights():
    x, wr, ex = _tiny_case(FMT_BITPLANE8, T=16, E=6, k=3, seed=70)
    out, r = moe_layer(x, wr, None, ex, 3)
    assert np.array_equal(r.bits, select_bits(r.weights))
