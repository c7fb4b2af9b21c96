"""GPU parity at oracle-sized shapes: every C-ABI call against the CPU oracle on
the same seeded inputs, element by element.  Bit-exact for packing, scales,
routing ids and the permutation; the FFN and combine within the stated
tolerance.  Shapes span several tiles, ragged tails, single-token experts and
experts with more tokens than one 16-token pass."""
import numpy as np
import pytest
import torch

import synth
from layer_inputs import (as_u32, assert_routing_equals_oracle, check_close, dev_bf16, host_bits, make_layer,
                          oracle_experts, sentinel_routing)
from oracle.ffn import FMT_BITPLANE8, FMT_NVFP4, FMT_W4G128, combine, grouped_ffn
from oracle.quant import pack_bitplanes, quantize_nvfp4, quantize_w4g128
from oracle.routing import permute, router_logits, router_logits_f64, select_bits, topk_softmax

pytestmark = pytest.mark.gpu


# ---------------------------------------------------------------- input generator
def test_synth_device_equals_host(moe, cuda_device):
    for seed, n, start, std in [(1, 10000, 0, 1.0), (77, 4097, 123456789, 0.02), (5, 3, 2 ** 40, 0.5)]:
        t = torch.empty(n, dtype=torch.bfloat16, device=cuda_device)
        moe.moe_synth_normal_bf16(t, seed, std, start)
        assert np.array_equal(host_bits(t), synth.normal_bf16(seed, n, std, start))
    for seed, n, start, lo, hi in [(3, 9999, 0, -0.02, 0.02), (4, 100, 10 ** 9, -1.0, 3.0)]:
        t = torch.empty(n, dtype=torch.bfloat16, device=cuda_device)
        moe.moe_synth_uniform_bf16(t, seed, lo, hi, start)
        assert np.array_equal(host_bits(t), synth.uniform_bf16(seed, n, lo, hi, start))


# ---------------------------------------------------------------- quantisers
def _weights_with_edges(seed, E, N, K):
    w = synth.normal_bf16(seed, E * N * K, 0.02).reshape(E, N, K).copy()
    w[0, 0, :128] = 0                      # an all-zero group
    w[-1, -1, -128:] = synth.normal_bf16(seed + 9, 128, 1e-30)  # tiny values (subnormal fp32 range)
    w[0, min(1, N - 1), 5] = synth.f32_to_bf16_bits(np.array([3.0], np.float32))[0]  # an outlier
    return w


QSHAPES = [(3, 64, 256), (2, 48, 2048), (1, 16, 7168), (5, 1, 128)]


@pytest.mark.parametrize("E,N,K", QSHAPES)
def test_quantize_w4g128_bitexact(moe, cuda_device, E, N, K):
    w = _weights_with_edges(11, E, N, K)
    packed, scales = moe.moe_quantize_w4g128(dev_bf16(w))
    rp, rs = quantize_w4g128(w)
    assert np.array_equal(as_u32(packed), rp)
    assert np.array_equal(host_bits(scales), rs)


@pytest.mark.parametrize("E,N,K", QSHAPES)
def test_pack_bitplanes_bitexact(moe, cuda_device, E, N, K):
    w = _weights_with_edges(12, E, N, K)
    planes, scales = moe.moe_pack_bitplanes(dev_bf16(w))
    rp, rs = pack_bitplanes(w)
    assert np.array_equal(as_u32(planes), rp)
    assert np.array_equal(host_bits(scales), rs)


@pytest.mark.parametrize("E,N,K", QSHAPES + [(2, 8, 32)])
def test_quantize_nvfp4_bitexact(moe, cuda_device, E, N, K):
    w = _weights_with_edges(13, E, N, K) if K >= 256 else synth.normal_bf16(13, E * N * K, 0.02).reshape(E, N, K)
    codes, sb, g = moe.moe_quantize_nvfp4(dev_bf16(w))
    rc, rsb, rg = quantize_nvfp4(w)
    assert np.array_equal(g.cpu().numpy(), rg)
    assert np.array_equal(sb.cpu().numpy(), rsb)
    assert np.array_equal(codes.cpu().numpy(), rc)


# ---------------------------------------------------------------- routing
ROUTE_CASES = [
    # T, H, E, k, router, zipf
    (1, 2048, 64, 8, "normal", False),
    (16, 2048, 64, 8, "normal", False),
    (64, 2048, 64, 8, "normal", False),
    (65, 512, 64, 8, "normal", False),      # past the single-CTA top-k path
    (300, 512, 128, 8, "normal", True),     # skewed (Zipf) routing
    (259, 7168, 256, 8, "uniform", False),  # tiled logits path, wide hidden size
    (40, 256, 1024, 32, "normal", False),   # largest E and k
    (3, 256, 1, 1, "normal", False),        # a single expert
    (33, 256, 5, 5, "normal", False),       # k = E: every expert for every token
    # single-launch path for few tokens (T <= 16, staged tokens <= 64 KiB)
    (4, 7168, 256, 8, "uniform", False),    # wide hidden size, 56 KiB of staged tokens
    (13, 512, 37, 6, "normal", True),       # E not a multiple of the 8 experts per CTA
    (16, 256, 1024, 32, "normal", False),   # largest E and k with the last-CTA permutation
    (9, 7168, 256, 8, "uniform", False),    # too many staged bytes: the multi-launch path
]


def _route_both(moe, L, k):
    out = moe.moe_route_topk(dev_bf16(L.x), dev_bf16(L.wr),
                             None if L.bias is None else torch.from_numpy(L.bias).cuda(), k)
    logits = router_logits(L.x, L.wr, L.bias)
    ids, w = topk_softmax(logits, k)
    offsets, sp, p2r = permute(ids, L.E)
    return out, (logits, ids, w, offsets, sp, p2r)


@pytest.mark.parametrize("T,H,E,k,router,zipf", ROUTE_CASES)
def test_route_topk_bitexact(moe, cuda_device, T, H, E, k, router, zipf):
    L = make_layer(100 + T + E, T, H, 128, E, k, router=router, zipf=zipf, with_experts=False)
    out, (logits, ids, w, offsets, sp, p2r) = _route_both(moe, L, k)
    torch.cuda.synchronize()
    assert np.array_equal(out.topk_ids.cpu().numpy().reshape(T, k), ids)
    assert np.abs(out.topk_w.cpu().numpy().reshape(T, k) - w).max() <= 1e-6
    assert np.array_equal(out.expert_offsets.cpu().numpy(), offsets)
    assert np.array_equal(out.sorted_pair.cpu().numpy(), sp)
    assert np.array_equal(out.pair_to_row.cpu().numpy(), p2r)
    el = out.expert_list.cpu().numpy()
    act = np.nonzero(np.diff(offsets) > 0)[0]
    assert el[0] == act.size and np.array_equal(el[1:1 + act.size], act)


@pytest.mark.parametrize("T,H,E,k", [(8, 2048, 64, 8), (1, 256, 8, 2), (100, 512, 64, 8)])
def test_route_workspace_reuse(moe, cuda_device, T, H, E, k):
    # one workspace for several calls: the completion counter is left at zero each time
    ws = moe.moe_route_workspace(T, E, k, "cuda")
    out = moe.Routing.empty(T, E, k)
    for rep in range(3):
        L = make_layer(900 + rep, T, H, 128, E, k, with_experts=False)
        moe.moe_route_topk(dev_bf16(L.x), dev_bf16(L.wr), None, k, out=out, workspace=ws)
        ids, w = topk_softmax(router_logits(L.x, L.wr, None), k)
        offsets, sp, p2r = permute(ids, E)
        assert np.array_equal(out.topk_ids.cpu().numpy().reshape(T, k), ids)
        assert np.array_equal(out.sorted_pair.cpu().numpy(), sp)
        assert not ws[:256].any().item()  # the completion counter, left at zero


# (T, E) sequence through one workspace sized for (64, 64): the one-launch router (T <= 16)
# after larger multi-launch calls, smaller E after larger, and back.
REUSE_SEQUENCE = [(64, 64), (16, 64), (8, 64), (1, 64), (13, 64), (64, 64), (8, 32), (16, 64), (3, 8), (64, 64)]


def test_route_workspace_reuse_across_batches(moe, cuda_device):
    k = 8
    ws = moe.moe_route_workspace(64, 64, k, "cuda")
    for i, (T, E) in enumerate(REUSE_SEQUENCE):
        kk = min(k, E)
        L = make_layer(4400 + 31 * i, T, 2048, 128, E, kk, with_experts=False)
        out = sentinel_routing(moe, T, E, kk)
        moe.moe_route_topk(dev_bf16(L.x), dev_bf16(L.wr), None, kk, out=out, workspace=ws)
        moe.moe_check_device_errors()
        assert_routing_equals_oracle(out, L, kk, f"call {i} (T={T}, E={E})")
        assert not ws[:256].any().item(), f"call {i}: completion counter not left at zero"


def test_route_empty_batch(moe, cuda_device):
    L = make_layer(5, 1, 256, 128, 8, 2, with_experts=False)
    x = dev_bf16(L.x)[:0]
    out = moe.Routing.empty(0, 8, 2)
    moe.moe_route_topk(x, dev_bf16(L.wr), None, 2, out=out)
    moe.moe_check_device_errors()


def test_select_bits_matches_oracle(moe, cuda_device):
    rng = np.random.default_rng(0)
    w = rng.random(5000).astype(np.float32)
    w[:4] = [0.05, 0.15, 0.3, np.nextafter(np.float32(0.05), np.float32(0))]
    bits = moe.moe_select_bits(torch.from_numpy(w).cuda(), 8 if w.size % 8 == 0 else 1)
    assert np.array_equal(bits.cpu().numpy(), select_bits(w))


# ---------------------------------------------------------------- FFN + combine
FFN_CASES = [
    # T, H, I, E, k
    (9, 256, 128, 6, 3),
    (64, 512, 256, 16, 4),     # ~16 tokens per expert: the second n8 tile
    (200, 256, 128, 4, 2),     # ~100 tokens per expert: several 16-token passes
    (16, 2048, 1024, 16, 4),   # OLMoE-like expert shape, decode-sized
    (3, 768, 384, 8, 2),       # K = 768 / 384: uneven split of groups over warps
    (90, 1024, 256, 4, 1),     # ~22 tokens per expert: two token chunks per weight pass
    (20, 7168, 384, 3, 1),     # K = 7168: seven weight stages per unit, 56 scale groups
    (1, 2048, 1024, 64, 8),    # batch 1 (OLMoE-like): one token per expert
    (2, 768, 384, 8, 2),       # batch 2; down K = 384 has an odd number of scale groups
]


def _bits_for(T, k, seed):
    rng = np.random.default_rng(seed)
    return rng.choice(np.array([2, 3, 4, 8], dtype=np.uint8), size=(T, k))


@pytest.mark.parametrize("fmt", [FMT_W4G128, FMT_BITPLANE8, FMT_NVFP4])
@pytest.mark.parametrize("T,H,I,E,k", FFN_CASES)
def test_grouped_ffn_and_combine(moe, cuda_device, fmt, T, H, I, E, k):
    L = make_layer(1000 + 7 * T + E, T, H, I, E, k)
    ex_o = oracle_experts(fmt, L.w13, L.w2)
    ex_g = moe.quantize_experts(fmt, dev_bf16(L.w13), dev_bf16(L.w2))
    out, (logits, ids, w, offsets, sp, p2r) = _route_both(moe, L, k)
    assert np.array_equal(out.topk_ids.cpu().numpy().reshape(T, k), ids)
    bits = _bits_for(T, k, T) if fmt == FMT_BITPLANE8 else None
    bits_d = torch.from_numpy(bits.reshape(-1)).cuda() if bits is not None else None
    x_d = dev_bf16(L.x)
    y = moe.moe_grouped_ffn(x_d, out, ex_g, I, E, k, bits=bits_d)
    resid = synth.normal_bf16(77, T * H, 1.0).reshape(T, H)
    o = moe.moe_combine(y, out, T, k, residual=dev_bf16(resid))
    moe.moe_check_device_errors()
    y_ref = grouped_ffn(L.x, offsets, sp, k, ex_o, bits)
    check_close(bf16_f64(host_bits(y)), y_ref, f"y_rows fmt={fmt}")
    o_ref = combine(y_ref, w, p2r, resid)
    check_close(bf16_f64(host_bits(o)), o_ref, f"out fmt={fmt}")


def bf16_f64(b):
    return synth.bf16_bits_to_f32(b).astype(np.float64)


# Batches with 32 or more rows per expert on average take the tensor-core GEMM
# path (tcgen05; W4 group-128 in bf16, NVFP4 in fp16): 128-row weight tiles, up to
# 192 routed rows per tile.
GEMM_CASES = [
    # T, H, I, E, k, zipf
    (512, 256, 128, 8, 2, False),     # ~128 rows per expert: one or two row tiles
    (700, 512, 256, 16, 4, True),     # skewed: experts with several row tiles and empty ones
    (300, 2048, 1024, 8, 2, False),   # OLMoE-like expert shape, 32 / 16 K-blocks
    (129, 768, 384, 4, 1, False),     # ragged row tiles (MMA N not a multiple of 32), K = 768
    (64, 256, 128, 1, 1, False),      # a single expert
]


@pytest.mark.parametrize("fmt", [FMT_W4G128, FMT_NVFP4])
@pytest.mark.parametrize("T,H,I,E,k,zipf", GEMM_CASES)
def test_grouped_gemm_path(moe, cuda_device, fmt, T, H, I, E, k, zipf):
    assert T * k >= 32 * E
    L = make_layer(3000 + T + E, T, H, I, E, k, zipf=zipf)
    ex_o = oracle_experts(fmt, L.w13, L.w2)
    ex_g = moe.quantize_experts(fmt, dev_bf16(L.w13), dev_bf16(L.w2))
    out, (logits, ids, w, offsets, sp, p2r) = _route_both(moe, L, k)
    assert np.array_equal(out.sorted_pair.cpu().numpy(), sp)
    y = moe.moe_grouped_ffn(dev_bf16(L.x), out, ex_g, I, E, k)
    o = moe.moe_combine(y, out, T, k)
    moe.moe_check_device_errors()
    y_ref = grouped_ffn(L.x, offsets, sp, k, ex_o, None)
    check_close(bf16_f64(host_bits(y)), y_ref, f"y_rows (GEMM path, fmt={fmt})")
    check_close(bf16_f64(host_bits(o)), combine(y_ref, w, p2r, None), f"out (GEMM path, fmt={fmt})")
