"""GPU parity of the budgeted per-expert bit allocation: the distortion tensor and the
activation moments against the fp64 oracle (relative 1e-12: both sum fp64 terms, in
different orders), the per-expert widths exactly (the oracle's decisions on the same
delta, m and routing counts), the per-pair expansion bit for bit, and the bitplane FFN
run at the allocated widths against the oracle FFN at the oracle's widths."""
import numpy as np
import pytest
import torch

import synth
from layer_inputs import check_close, dev_bf16, host_bits, make_layer, oracle_experts
from oracle.alloc import (activation_moments, allocate_bits, bitplane_distortion, expand_bits, expert_counts,
                          expert_distortion)
from oracle.ffn import FMT_BITPLANE8, grouped_ffn
from oracle.quant import pack_bitplanes
from oracle.routing import permute, router_logits, topk_softmax

pytestmark = pytest.mark.gpu

REL = 1e-12


def _close_rel(got, ref, rel=REL):
    got, ref = np.asarray(got), np.asarray(ref)
    assert got.shape == ref.shape
    assert np.all(np.abs(got - ref) <= rel * np.abs(ref)), float(np.max(np.abs(got - ref) / (np.abs(ref) + 1e-300)))


@pytest.mark.parametrize("E,N,K", [(1, 1, 128), (3, 64, 256), (8, 256, 2048), (2, 7, 768)])
def test_bitplane_distortion_matches_oracle(moe, cuda_device, E, N, K):
    w = synth.normal_bf16(900 + E * N, E * N * K, 0.02).reshape(E, N, K)
    planes, s_bits = pack_bitplanes(w)
    d = moe.moe_bitplane_distortion(torch.from_numpy(planes.view(np.int32)).cuda(), dev_bf16(s_bits))
    moe.moe_check_device_errors()
    ref = bitplane_distortion(planes, s_bits)
    got = d.cpu().numpy()
    assert np.all(got[:, 7, :] == 0.0)
    _close_rel(got, ref)


def test_bitplane_distortion_of_device_packed_weights(moe, cuda_device):
    # the library's own packer feeds the distortion kernel: same planes, same delta
    E, N, K = 4, 128, 1024
    w = synth.normal_bf16(77, E * N * K, 0.02).reshape(E, N, K)
    planes_d = torch.empty((E, 8, N, K // 32), dtype=torch.int32, device="cuda")
    s_d = torch.empty((E, N, K // 128), dtype=torch.bfloat16, device="cuda")
    moe.moe_pack_bitplanes(dev_bf16(w), planes_d, s_d)
    d = moe.moe_bitplane_distortion(planes_d, s_d)
    planes, s_bits = pack_bitplanes(w)
    _close_rel(d.cpu().numpy(), bitplane_distortion(planes, s_bits))


@pytest.mark.parametrize("T,H", [(1, 64), (37, 300), (2048, 2048)])
def test_activation_moments_matches_oracle(moe, cuda_device, T, H):
    x = synth.normal_bf16(5 + T, T * H, 1.0).reshape(T, H)
    m = moe.moe_activation_moments(dev_bf16(x))
    moe.moe_check_device_errors()
    _close_rel(m.cpu().numpy(), activation_moments(x))


def _offsets_from_counts(counts):
    return np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)


CHOICE_SETS = [(2, 3, 4, 8), (8, 4, 2), (1, 2, 3, 4, 5, 6, 7, 8), (4,), (3, 8)]
BUDGETS = [0.0, 1.5, 2.0, 2.4, 3.0, 3.7, 5.0, 7.99, 8.0, 100.0]


@pytest.mark.parametrize("choices", CHOICE_SETS)
@pytest.mark.parametrize("E,K,zipf", [(64, 2048, False), (128, 512, True), (1024, 256, True), (5, 128, False)])
def test_allocate_bits_matches_oracle(moe, cuda_device, choices, E, K, zipf):
    rng = np.random.default_rng(E * 7 + K + len(choices))
    # delta from real packed weights (the monotone-in-b structure of the method), m from tokens
    w = synth.normal_bf16(E + K, E * 16 * K, 0.02).reshape(E, 16, K)
    planes, s_bits = pack_bitplanes(w)
    delta = bitplane_distortion(planes, s_bits) * rng.uniform(0.5, 2.0, size=(E, 1, 1))
    m = activation_moments(synth.normal_bf16(K, 8 * K, 1.0).reshape(8, K))
    if zipf:
        counts = rng.zipf(1.5, size=E).clip(0, 4000) * (rng.random(E) < 0.8)
    else:
        counts = rng.integers(0, 50, size=E)
    offsets = _offsets_from_counts(counts)
    D = expert_distortion(delta, m, choices)
    delta_d = torch.from_numpy(delta).cuda()
    m_d = torch.from_numpy(m).cuda()
    off_d = torch.from_numpy(offsets).cuda()
    lam_d = torch.zeros((), dtype=torch.float64, device="cuda")
    total = int(np.sum(counts))
    for budget in BUDGETS:
        bits_ref, lam_ref = allocate_bits(D, counts, choices, budget)
        bits = moe.moe_allocate_bits(delta_d, m_d, off_d, budget, choices=choices, lam=lam_d)
        moe.moe_check_device_errors()
        got = bits.cpu().numpy()
        assert np.array_equal(got, bits_ref), (budget, got, bits_ref)
        lam = lam_d.item()
        assert lam == pytest.approx(lam_ref, rel=1e-9, abs=0.0), budget
        if total and min(choices) <= budget:
            assert int(np.sum(counts * got.astype(np.int64))) <= budget * total  # the read budget holds


def test_allocate_bits_degenerate_cases(moe, cuda_device):
    E, K = 16, 256
    delta = np.abs(np.random.default_rng(3).normal(size=(E, 8, K)))
    delta[:, 7, :] = 0.0
    choices = (2, 3, 4, 8)
    cases = [
        (np.zeros(K), np.arange(E) % 5, 3.0),   # m = 0: every D ties, any lam > 0 takes the smallest
        (np.ones(K), np.zeros(E, int), 3.0),    # nothing routed: every expert unread, smallest width
        (np.ones(K), np.eye(1, E, 0, int)[0] * 9, 8.0),  # one expert read, budget at the top
        (np.ones(K), np.full(E, 3), 1.0),       # infeasible budget: the smallest width everywhere
    ]
    for m, counts, budget in cases:
        D = expert_distortion(delta, m, choices)
        bits_ref, _ = allocate_bits(D, counts, choices, budget)
        bits = moe.moe_allocate_bits(torch.from_numpy(delta).cuda(), torch.from_numpy(m.astype(np.float64)).cuda(),
                                     torch.from_numpy(_offsets_from_counts(counts)).cuda(), budget, choices=choices)
        moe.moe_check_device_errors()
        assert np.array_equal(bits.cpu().numpy(), bits_ref), (budget, counts)


@pytest.mark.parametrize("T,k,E", [(1, 1, 4), (333, 8, 64), (4096, 8, 128)])
def test_expand_bits_bitexact(moe, cuda_device, T, k, E):
    rng = np.random.default_rng(T)
    ids = rng.integers(0, E, size=(T, k)).astype(np.int32)
    bits_e = rng.choice(np.array([2, 3, 4, 8], np.uint8), size=E)
    got = moe.moe_expand_bits(torch.from_numpy(ids).cuda(), torch.from_numpy(bits_e).cuda(), k)
    assert np.array_equal(got.cpu().numpy()[:T * k], expand_bits(ids, bits_e))


@pytest.mark.parametrize("T,H,I,E,k,budget", [(48, 512, 256, 16, 4, 3.3), (16, 2048, 1024, 16, 4, 2.6)])
def test_allocated_bitplane_layer(moe, cuda_device, T, H, I, E, k, budget):
    # route -> profile -> distortion of the gate/up matrix -> allocation -> per-pair widths
    # -> bitplane FFN at those widths, every step on the device, against the oracle chain
    L = make_layer(4242 + T, T, H, I, E, k)
    ex_o = oracle_experts(FMT_BITPLANE8, L.w13, L.w2)
    ex_g = moe.quantize_experts(FMT_BITPLANE8, dev_bf16(L.w13), dev_bf16(L.w2))
    x_d = dev_bf16(L.x)
    r = moe.moe_route_topk(x_d, dev_bf16(L.wr), None, k)
    delta_d = moe.moe_bitplane_distortion(ex_g.w13, ex_g.w13_scale)
    m_d = moe.moe_activation_moments(x_d)
    bits_e_d = moe.moe_allocate_bits(delta_d, m_d, r.expert_offsets, budget)
    bits_d = moe.moe_expand_bits(r.topk_ids, bits_e_d, k)
    y = moe.moe_grouped_ffn(x_d, r, ex_g, I, E, k, bits=bits_d)
    moe.moe_check_device_errors()

    ids, w = topk_softmax(router_logits(L.x, L.wr, None), k)
    offsets, sp, _ = permute(ids, E)
    assert np.array_equal(r.expert_offsets.cpu().numpy(), offsets)
    delta = bitplane_distortion(ex_o.w13, ex_o.w13_s)
    D = expert_distortion(delta, activation_moments(L.x), (2, 3, 4, 8))
    bits_e, _ = allocate_bits(D, expert_counts(offsets), (2, 3, 4, 8), budget)
    assert np.array_equal(bits_e_d.cpu().numpy(), bits_e)
    assert len(set(bits_e[expert_counts(offsets) > 0].tolist())) >= 2  # the budget mixes widths
    bits = expand_bits(ids, bits_e).reshape(T, k)
    assert np.array_equal(bits_d.cpu().numpy()[:T * k].reshape(T, k), bits)
    y_ref = grouped_ffn(L.x, offsets, sp, k, ex_o, bits)
    check_close(synth.bf16_bits_to_f32(host_bits(y)).astype(np.float64), y_ref, "y_rows at allocated widths")
