"""GPU parity of the device-side expert slot cache: the one-CTA step against the oracle's
plan (served experts, slots, plane ranges, the state after the step, every pair's slot),
the fetch against the host store byte for byte, and a cached layer (experts in pinned host
memory, S device slots) against the same layer with every expert resident (bit for bit)
and against the oracle (tolerance)."""
import numpy as np
import pytest
import torch

import synth
from layer_inputs import check_close, dev_bf16, host_bits, make_layer, oracle_experts
from oracle.cache import SlotCache, need_from_routing
from oracle.ffn import FMT_BITPLANE8, FMT_NVFP4, FMT_W4G128, combine, grouped_ffn
from oracle.routing import permute, router_logits, topk_softmax

pytestmark = pytest.mark.gpu


def _ids(rng, T, E, k):
    return np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)


def _host_state_view(state):
    return np.ascontiguousarray(state.cpu().numpy()).view(np.int64).copy()


@pytest.mark.parametrize("E,S,P,T,k", [(64, 16, 8, 2, 8), (64, 64, 1, 8, 8), (128, 40, 8, 4, 8), (8, 8, 8, 3, 2),
                                       (1024, 64, 8, 8, 8)])
def test_cache_step_matches_oracle(moe, cuda_device, E, S, P, T, k):
    rng = np.random.default_rng(E + S + T)
    state = moe.moe_cache_state_device(E, S, P)
    ref = SlotCache(E=E, S=S, P=P)
    routing = moe.Routing.empty(T, E, k)
    for step in range(50):
        ids = _ids(rng, T, E, k)
        offsets, sp, p2r = permute(ids, E)
        bits = rng.choice(np.array([2, 3, 4, 8], np.uint8), size=T * k) if P == 8 else None
        routing.topk_ids.copy_(torch.from_numpy(ids.reshape(-1)))
        moe.moe_permute(routing.topk_ids, T, k, E, out=routing)
        assert np.array_equal(routing.expert_offsets.cpu().numpy(), offsets)
        assert np.array_equal(routing.sorted_pair.cpu().numpy()[:T * k], sp)
        assert np.array_equal(routing.pair_to_row.cpu().numpy()[:T * k], p2r)
        bits_d = torch.from_numpy(bits).cuda() if bits is not None else None
        slot_ids, plan = moe.moe_cache_step(state, E, S, routing, T, k, bits=bits_d)
        moe.moe_check_device_errors()
        rounds = ref.plan(need_from_routing(offsets, sp, bits, planes=P))
        assert len(rounds) == 1 and plan.overflow.item() == 0
        n = plan.nserved.item()
        assert n == len(rounds[0])
        assert plan.served_expert.cpu().numpy()[:n].tolist() == [sv.expert for sv in rounds[0]]
        assert plan.served_slot.cpu().numpy()[:n].tolist() == [sv.slot for sv in rounds[0]]
        assert plan.fetch_lo.cpu().numpy()[:n].tolist() == [sv.lo for sv in rounds[0]]
        assert plan.fetch_hi.cpu().numpy()[:n].tolist() == [sv.hi for sv in rounds[0]]
        eo, pl = moe.moe_cache_slots(_host_state_view(state), S)
        assert eo.tolist() == ref.expert_of and pl.tolist() == ref.planes
        assert slot_ids.cpu().numpy()[:T * k].tolist() == [ref.slot_of[int(e)] for e in ids.reshape(-1)]


def _stores(moe, fmt, E, H, I, seed):
    w13 = synth.normal_bf16(seed, E * 2 * I * H, 0.02).reshape(E, 2 * I, H)
    w2 = synth.normal_bf16(seed + 1, E * H * I, 0.02).reshape(E, H, I)
    dev = moe.quantize_experts(fmt, dev_bf16(w13), dev_bf16(w2))
    pin = lambda t: None if t is None else t.cpu().pin_memory()
    host = moe.Experts(fmt, pin(dev.w13), pin(dev.w13_scale), pin(dev.w2), pin(dev.w2_scale), pin(dev.w13_gscale),
                       pin(dev.w2_gscale))
    return dev, host, w13, w2


def _slot_store(moe, dev, S):
    z = lambda t: None if t is None else torch.zeros((S,) + tuple(t.shape[1:]), dtype=t.dtype, device="cuda")
    return moe.Experts(dev.fmt, z(dev.w13), z(dev.w13_scale), z(dev.w2), z(dev.w2_scale), z(dev.w13_gscale),
                       z(dev.w2_gscale))


@pytest.mark.parametrize("fmt", [FMT_W4G128, FMT_BITPLANE8, FMT_NVFP4])
def test_cache_fetch_copies_the_planned_planes(moe, cuda_device, fmt):
    E, S, H, I, T, k = 16, 6, 256, 128, 3, 2
    P = 8 if fmt == FMT_BITPLANE8 else 1
    dev, host, _, _ = _stores(moe, fmt, E, H, I, 31 + fmt)
    slots = _slot_store(moe, dev, S)
    state = moe.moe_cache_state_device(E, S, P)
    ref = SlotCache(E=E, S=S, P=P)
    rng = np.random.default_rng(fmt)
    routing = moe.Routing.empty(T, E, k)
    for step in range(25):
        ids = _ids(rng, T, E, k)
        offsets, sp, _ = permute(ids, E)
        bits = rng.choice(np.array([2, 3, 4, 8], np.uint8), size=T * k) if P == 8 else None
        routing.topk_ids.copy_(torch.from_numpy(ids.reshape(-1)))
        moe.moe_permute(routing.topk_ids, T, k, E, out=routing)
        _, plan = moe.moe_cache_step(state, E, S, routing, T, k,
                                     bits=torch.from_numpy(bits).cuda() if bits is not None else None)
        moe.moe_cache_fetch(plan, E, host, slots, H, I)
        moe.moe_check_device_errors()
        ref.plan(need_from_routing(offsets, sp, bits, planes=P))
        for s, e in enumerate(ref.expert_of):
            if e < 0:
                continue
            h = ref.planes[s]
            for hw, sw in ((host.w13, slots.w13), (host.w2, slots.w2)):
                want = hw[e, :h] if P == 8 else hw[e]
                got = sw[s, :h].cpu() if P == 8 else sw[s].cpu()
                assert torch.equal(got, want), (step, s, e)
            for hs, ss in ((host.w13_scale, slots.w13_scale), (host.w2_scale, slots.w2_scale)):
                assert torch.equal(ss[s].cpu().view(torch.uint8), hs[e].view(torch.uint8))
            if fmt == FMT_NVFP4:
                assert slots.w13_gscale[s].item() == host.w13_gscale[e].item()
                assert slots.w2_gscale[s].item() == host.w2_gscale[e].item()


@pytest.mark.parametrize("fmt", [FMT_W4G128, FMT_BITPLANE8])
def test_cached_layer_equals_resident_layer(moe, cuda_device, fmt):
    T, H, I, E, k, S = 4, 512, 256, 16, 4, 16
    P = 8 if fmt == FMT_BITPLANE8 else 1
    L = make_layer(777 + fmt, T, H, I, E, k)
    dev = moe.quantize_experts(fmt, dev_bf16(L.w13), dev_bf16(L.w2))
    pin = lambda t: t.cpu().pin_memory()
    host = moe.Experts(fmt, pin(dev.w13), pin(dev.w13_scale), pin(dev.w2), pin(dev.w2_scale))
    slots = _slot_store(moe, dev, S)
    state = moe.moe_cache_state_device(E, S, P)
    ex_o = oracle_experts(fmt, L.w13, L.w2)
    rng = np.random.default_rng(3)
    for step in range(6):
        x = synth.normal_bf16(900 + step, T * H, 1.0).reshape(T, H)
        xd = dev_bf16(x)
        r = moe.moe_route_topk(xd, dev_bf16(L.wr), None, k)
        bits = torch.from_numpy(rng.choice(np.array([2, 3, 4, 8], np.uint8), size=T * k)).cuda() \
            if fmt == FMT_BITPLANE8 else None
        # resident: every expert on the device
        y_res = moe.moe_grouped_ffn(xd, r, dev, I, E, k, bits=bits)
        out_res = moe.moe_combine(y_res, r, T, k, residual=xd)
        # cached: plan, slot routing, fetch, FFN on the slots, combine with the slot routing
        slot_ids, plan = moe.moe_cache_step(state, E, S, r, T, k, bits=bits)
        rs = moe.Routing(slot_ids, r.topk_w, torch.empty(S + 1, dtype=torch.int32, device="cuda"),
                         torch.empty_like(r.sorted_pair), torch.empty_like(r.pair_to_row),
                         torch.empty(S + 1, dtype=torch.int32, device="cuda"))
        moe.moe_permute(slot_ids, T, k, S, out=rs)
        moe.moe_cache_fetch(plan, E, host, slots, H, I)
        # per-pair widths follow the pairs, not the rows: the same array serves both routings
        y_c = moe.moe_grouped_ffn(xd, rs, slots, I, S, k, bits=bits)
        out_c = moe.moe_combine(y_c, rs, T, k, residual=xd)
        moe.moe_check_device_errors()
        assert torch.equal(out_c.view(torch.int16), out_res.view(torch.int16)), step
        ids, w = topk_softmax(router_logits(x, L.wr, None), k)
        offsets, sp, p2r = permute(ids, E)
        b = bits.cpu().numpy().reshape(T, k) if bits is not None else None
        ref = combine(grouped_ffn(x, offsets, sp, k, ex_o, b), w, p2r, x)
        check_close(synth.bf16_bits_to_f32(host_bits(out_c)).astype(np.float64), ref, f"cached layer step {step}")
