"""GPU parity of the W4A4 prefill path (NVFP4 weights and NVFP4 activations quantised on the
fly): the fp32 activation quantiser bit for bit against the oracle's recipe (codes, block
scales, tensor scale), and the grouped FFN against the oracle's W4A4 FFN within the FFN
tolerance, over shapes that span several GEMM tiles and ragged tails."""
import numpy as np
import pytest
import torch

import synth
from layer_inputs import check_close, dev_bf16, host_bits, make_layer, oracle_experts
from oracle.ffn import FMT_NVFP4, combine
from oracle.routing import permute, router_logits, topk_softmax
from oracle.w4a4 import quantize_act_nvfp4, w4a4_grouped_ffn

pytestmark = pytest.mark.gpu


def _f32_tensor(seed, R, C):
    rng = np.random.default_rng(seed)
    a = (rng.standard_normal((R, C)) * rng.choice([0.01, 1.0, 40.0], size=(R, 1))).astype(np.float32)
    a[0, :16] = 0.0                              # an all-zero block
    a[-1, -16:] = np.float32(1e-30)              # tiny values (E4M3 scale underflows to 0)
    a[R // 2, 5] = np.float32(-3000.0)           # the tensor's amax, negative
    return a


@pytest.mark.parametrize("R,C", [(1, 16), (7, 256), (300, 1024), (64, 7168)])
def test_quantize_nvfp4_f32_bitexact(moe, cuda_device, R, C):
    a = _f32_tensor(R * 7 + C, R, C)
    codes, sb, g = moe.moe_quantize_nvfp4_f32(torch.from_numpy(a).cuda())
    rc, rsb, rg = quantize_act_nvfp4(a)
    assert g.item() == rg
    assert np.array_equal(sb.cpu().numpy(), rsb)
    assert np.array_equal(codes.cpu().numpy(), rc)


def test_quantize_nvfp4_f32_zero_tensor(moe, cuda_device):
    a = np.zeros((4, 32), np.float32)
    codes, sb, g = moe.moe_quantize_nvfp4_f32(torch.from_numpy(a).cuda())
    assert g.item() == 0.0 and not codes.any().item() and not sb.any().item()


W4A4_CASES = [
    # T, H, I, E, k, zipf
    (96, 256, 128, 4, 2, False),     # one or two row tiles per expert
    (700, 512, 256, 16, 4, True),    # skewed: experts with several row tiles and empty ones
    (129, 768, 384, 4, 1, False),    # ragged row tiles, K = 768
    (5, 1024, 512, 8, 2, False),     # decode-sized batch on the GEMM
    (300, 2048, 1024, 8, 2, False),  # OLMoE-like expert shape
    (512, 7168, 2048, 4, 2, False),  # the benchmark's expert shape: 28 K stages, 2 row tiles per expert
    (64, 256, 128, 520, 2, False),   # E > 256: larger per-CTA tables, one CTA per SM; most experts empty
]


@pytest.mark.parametrize("T,H,I,E,k,zipf", W4A4_CASES)
def test_w4a4_ffn_matches_oracle(moe, cuda_device, T, H, I, E, k, zipf):
    L = make_layer(5000 + T + H, T, H, I, E, k, zipf=zipf)
    ex_o = oracle_experts(FMT_NVFP4, L.w13, L.w2)
    ex_g = moe.quantize_experts(FMT_NVFP4, dev_bf16(L.w13), dev_bf16(L.w2))
    bias = None if L.bias is None else torch.from_numpy(L.bias).cuda()
    r = moe.moe_route_topk(dev_bf16(L.x), dev_bf16(L.wr), bias, k)
    y = moe.moe_grouped_ffn_w4a4(dev_bf16(L.x), r, ex_g, I, E, k)
    out = moe.moe_combine(y, r, T, k)
    moe.moe_check_device_errors()
    ids, w = topk_softmax(router_logits(L.x, L.wr, L.bias), k)
    offsets, sp, p2r = permute(ids, E)
    assert np.array_equal(r.sorted_pair.cpu().numpy(), sp)
    y_ref = w4a4_grouped_ffn(L.x, offsets, sp, k, ex_o)
    got = synth.bf16_bits_to_f32(host_bits(y)).astype(np.float64)[:T * k]
    check_close(got, y_ref, "W4A4 y_rows")
    check_close(synth.bf16_bits_to_f32(host_bits(out)).astype(np.float64), combine(y_ref, w, p2r, None),
                "W4A4 layer output")


def test_w4a4_differs_from_w4a16(moe, cuda_device):
    # the activation quantisation is really applied: the W4A4 layer moves away from the
    # NVFP4-weight layer with bf16 activations by about the activations' quantisation error
    T, H, I, E, k = 300, 512, 256, 8, 2
    L = make_layer(6123, T, H, I, E, k)
    ex_g = moe.quantize_experts(FMT_NVFP4, dev_bf16(L.w13), dev_bf16(L.w2))
    r = moe.moe_route_topk(dev_bf16(L.x), dev_bf16(L.wr), None, k)
    a = synth.bf16_bits_to_f32(host_bits(moe.moe_grouped_ffn_w4a4(dev_bf16(L.x), r, ex_g, I, E, k))).astype(np.float64)
    b = synth.bf16_bits_to_f32(host_bits(moe.moe_grouped_ffn(dev_bf16(L.x), r, ex_g, I, E, k))).astype(np.float64)
    rel = np.linalg.norm(a - b) / np.linalg.norm(b)
    assert 1e-3 < rel < 0.3, rel
