"""GPU parity at the five benchmark configurations' full sizes.

Weights are generated on the device by the library's seeded generator (the same
stream the host generator reproduces) and quantised there; the oracle regenerates
on the host only the experts that the sampled tokens route to.  Routing ids and the
permutation are compared for every token; FFN outputs element by element for the
sampled tokens (all tokens where the oracle finishes in seconds)."""
import numpy as np
import pytest
import torch

import synth
from layer_inputs import ATOL, REL_L2, bf16_to_f64, check_close, dev_bf16, host_bits
from oracle.ffn import FMT_BITPLANE8, FMT_NVFP4, FMT_W4G128, Experts, swiglu_expert
from oracle.quant import (dequant_bitplane, dequant_nvfp4, dequant_w4g128, pack_bitplanes, quantize_nvfp4,
                          quantize_w4g128)
from oracle.routing import permute, router_logits, select_bits, topk_softmax

pytestmark = pytest.mark.gpu


class DeviceLayer:
    """One layer's weights made and quantised on the GPU, in chunks of experts."""

    def __init__(self, moe, fmt, seed, H, I, E, wstd=0.02, chunk=16):
        self.moe, self.fmt, self.seed, self.H, self.I, self.E = moe, fmt, seed, H, I, E
        dev = torch.device("cuda")
        if fmt == FMT_W4G128:
            mk = lambda n, k: (torch.empty((E, n, k // 8), dtype=torch.int32, device=dev),
                               torch.empty((E, n, k // 128), dtype=torch.bfloat16, device=dev), None)
        elif fmt == FMT_BITPLANE8:
            mk = lambda n, k: (torch.empty((E, 8, n, k // 32), dtype=torch.int32, device=dev),
                               torch.empty((E, n, k // 128), dtype=torch.bfloat16, device=dev), None)
        else:
            mk = lambda n, k: (torch.empty((E, n, k // 2), dtype=torch.uint8, device=dev),
                               torch.empty((E, n, k // 16), dtype=torch.uint8, device=dev),
                               torch.empty((E,), dtype=torch.float32, device=dev))
        self.w13 = mk(2 * I, H)
        self.w2 = mk(H, I)
        for which, (n, k), store, tag in ((0, (2 * I, H), self.w13, synth.SEED_W13),
                                          (1, (H, I), self.w2, synth.SEED_W2)):
            tmp = torch.empty((chunk, n, k), dtype=torch.bfloat16, device=dev)
            for e0 in range(0, E, chunk):
                ne = min(chunk, E - e0)
                t = tmp[:ne]
                moe.moe_synth_normal_bf16(t, seed + tag, wstd, start=e0 * n * k)
                if fmt == FMT_W4G128:
                    moe.moe_quantize_w4g128(t, store[0][e0:e0 + ne], store[1][e0:e0 + ne])
                elif fmt == FMT_BITPLANE8:
                    moe.moe_pack_bitplanes(t, store[0][e0:e0 + ne], store[1][e0:e0 + ne])
                else:
                    moe.moe_quantize_nvfp4(t, store[0][e0:e0 + ne], store[1][e0:e0 + ne], store[2][e0:e0 + ne])
            del tmp
        self.experts = moe.Experts(fmt, self.w13[0], self.w13[1], self.w2[0], self.w2[1], self.w13[2], self.w2[2])

    def host_expert(self, e, check_device=True):
        """Oracle dequantisation of expert e from host-regenerated bf16 weights;
        also checks the device's packed bytes of that expert bit for bit."""
        H, I = self.H, self.I
        w13 = synth.normal_rows_bf16(self.seed + synth.SEED_W13, (2 * I, H), 0.02, e, 1)
        w2 = synth.normal_rows_bf16(self.seed + synth.SEED_W2, (H, I), 0.02, e, 1)
        out = []
        for w, store in ((w13, self.w13), (w2, self.w2)):
            if self.fmt == FMT_W4G128:
                p, s = quantize_w4g128(w)
                if check_device:
                    assert np.array_equal(store[0][e].cpu().numpy().view(np.uint32), p[0])
                    assert np.array_equal(host_bits(store[1][e]), s[0])
                out.append(lambda b, p=p, s=s: dequant_w4g128(p[0], s[0]))
            elif self.fmt == FMT_BITPLANE8:
                p, s = pack_bitplanes(w)
                if check_device:
                    assert np.array_equal(store[0][e].cpu().numpy().view(np.uint32), p[0])
                    assert np.array_equal(host_bits(store[1][e]), s[0])
                out.append(lambda b, p=p, s=s: dequant_bitplane(p, s, b)[0])
            else:
                c, sb, g = quantize_nvfp4(w)
                if check_device:
                    assert np.array_equal(store[0][e].cpu().numpy(), c[0])
                    assert np.array_equal(store[1][e].cpu().numpy(), sb[0])
                    assert store[2][e].item() == g[0]
                out.append(lambda b, c=c, sb=sb, g=g: dequant_nvfp4(c, sb, g)[0])
        return out


GEMM_ROW_TILE = 192  # routed rows per tile of the tensor-core GEMM path


def tile_rows(offsets: np.ndarray, e: int, tile: int = GEMM_ROW_TILE) -> list[int]:
    """Sorted rows of expert e that cover each of its row tiles: the first and the last
    row of every tile (the last tile is usually ragged)."""
    lo, hi = int(offsets[e]), int(offsets[e + 1])
    rows = []
    for t0 in range(lo, hi, tile):
        rows += [t0, min(hi, t0 + tile) - 1]
    return sorted(set(rows))


def pick_experts(offsets: np.ndarray, ids: np.ndarray, tokens, n: int | None) -> list[int]:
    """Experts whose row tiles are checked: all routed experts (n None), else those of the
    sampled tokens, the experts with the most and the fewest rows, and evenly spaced
    ones, n in all (at least)."""
    counts = np.diff(offsets)
    routed = [int(e) for e in np.nonzero(counts > 0)[0]]
    if n is None or n >= len(routed):
        return routed
    chosen = {int(e) for t in tokens for e in ids[t]}
    by_count = sorted(routed, key=lambda e: (counts[e], e))
    chosen.update(by_count[:2] + by_count[-2:])
    step = max(1, len(routed) // max(1, n - len(chosen)))
    for e in routed[::step]:
        if len(chosen) >= n:
            break
        chosen.add(e)
    return sorted(chosen)


def run_config(moe, fmt, seed, T, H, I, E, k, router="normal", zipf=False, sample=None, bit_rule=False,
               tile_experts: int | None = -1):
    """tile_experts: -1 checks only the sampled tokens' outputs; None also checks every
    routed expert's row tiles in y_rows (first and last row of each tile); n checks the
    row tiles of n experts (pick_experts)."""
    layer = DeviceLayer(moe, fmt, seed, H, I, E)
    x = synth.normal_bf16(seed + synth.SEED_X, T * H, 1.0).reshape(T, H)
    if router == "uniform":
        wr = synth.uniform_bf16(seed + synth.SEED_WR, E * H, -0.02, 0.02).reshape(E, H)
    else:
        wr = synth.normal_bf16(seed + synth.SEED_WR, E * H, 0.02).reshape(E, H)
    bias = synth.zipf_rank_bias(seed + synth.SEED_BIAS, E) if zipf else None
    xd = dev_bf16(x)
    r = moe.moe_route_topk(xd, dev_bf16(wr), None if bias is None else torch.from_numpy(bias).cuda(), k)
    bits_d = moe.moe_select_bits(r.topk_w, k) if bit_rule else None
    y = moe.moe_grouped_ffn(xd, r, layer.experts, I, E, k, bits=bits_d)
    out = moe.moe_combine(y, r, T, k)
    moe.moe_check_device_errors()

    # routing: every token (oracle logits in the prescribed order)
    ids, w = topk_softmax(router_logits(x, wr, bias), k)
    assert np.array_equal(r.topk_ids.cpu().numpy().reshape(T, k), ids)
    assert np.abs(r.topk_w.cpu().numpy().reshape(T, k) - w).max() <= 1e-6
    offsets, sp, p2r = permute(ids, E)
    assert np.array_equal(r.expert_offsets.cpu().numpy(), offsets)
    assert np.array_equal(r.sorted_pair.cpu().numpy(), sp)
    bits = None
    if bit_rule:
        bits = select_bits(w)
        gb = bits_d.cpu().numpy().reshape(T, k)
        thr = np.array([0.05, 0.15, 0.30], np.float32)
        near = np.min(np.abs(w[..., None] - thr), axis=-1) <= 1e-6
        assert np.array_equal(gb[~near], bits[~near])
        bits = np.where(near, gb, bits)  # at a threshold tie both tiers are valid; follow the device

    toks = list(range(T)) if sample is None else list(sample)
    got = bf16_to_f64(host_bits(out))
    got_y = bf16_to_f64(host_bits(y))
    xf = bf16_to_f64(x)
    tile_set = [] if tile_experts == -1 else pick_experts(offsets, ids, toks, tile_experts)
    need = sorted({int(e) for t in toks for e in ids[t]} | set(tile_set))
    worst = [0.0, 0.0]

    def expert_check(e, first):
        deq = layer.host_expert(e, check_device=first)
        mats = {}

        def ffn(rows_x, b):  # one dequantisation per width
            if b not in mats:
                mats[b] = (deq[0](b), deq[1](b))
            return swiglu_expert(rows_x, *mats[b])

        res = {}
        rows = tile_rows(offsets, e) if e in tile_set else []
        pairs = [int(sp[rr]) for rr in rows]
        for b in sorted({int(bits[p // k, p % k]) if bits is not None else 8 for p in pairs}):
            sel = [(rr, p) for rr, p in zip(rows, pairs)
                   if (int(bits[p // k, p % k]) if bits is not None else 8) == b]
            yr = ffn(xf[[p // k for _, p in sel]], b)
            for (rr, _), yv in zip(sel, yr):
                res[rr] = check_close(got_y[rr], yv, f"y_rows row {rr} (expert {e})")
        # this expert's contribution to the sampled tokens' outputs
        contrib = {}
        for t in toks:
            for j in range(k):
                if int(ids[t, j]) == e:
                    b = int(bits[t, j]) if bits is not None else 8
                    contrib[(t, j)] = ffn(xf[t:t + 1], b)[0]
        return res, contrib

    import concurrent.futures as cf
    import os
    contribs = {}
    with cf.ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as pool:
        for i0 in range(0, len(need), 16):  # bounded memory: 16 dequantised experts at a time
            for res, c in pool.map(lambda a: expert_check(*a), [(e, i < 2) for i, e in enumerate(need[i0:i0 + 16],
                                                                                                  start=i0)]):
                for m, rel in res.values():
                    worst = [max(worst[0], m), max(worst[1], rel)]
                contribs.update(c)
    for t in toks:
        ref = np.zeros(H)
        for j in range(k):
            ref += float(w[t, j]) * contribs[(t, j)]
        m, rel = check_close(got[t], ref, f"token {t}")
        worst = [max(worst[0], m), max(worst[1], rel)]
    return tuple(worst)


def test_config_olmoe_layer_16_tokens_w4(moe, cuda_device):
    # every token, every element: H2048 I1024 E64 top-8, 16 tokens
    run_config(moe, FMT_W4G128, 0x5EED0001, 16, 2048, 1024, 64, 8)


def test_config_bitplane_64_tokens(moe, cuda_device):
    # bit-widths from the routing weights, prefixes executed directly; 64 tokens, 16 sampled
    run_config(moe, FMT_BITPLANE8, 0x5EED0004, 64, 2048, 1024, 64, 8, bit_rule=True,
               sample=[0, 1, 2, 7, 13, 20, 31, 32, 40, 47, 50, 55, 60, 61, 62, 63])


def test_config_qwen_prefill_zipf(moe, cuda_device):
    # H2048 I768 E128 top-8, 2048 tokens with Zipf-skewed routing: all ids; every routed
    # expert's row tiles (first and last row of each, incl. the ragged last tile) in y_rows;
    # 6 tokens' combined outputs
    run_config(moe, FMT_W4G128, 0x5EED0003, 2048, 2048, 768, 128, 8, zipf=True, sample=[0, 1, 777, 1500, 2046, 2047],
               tile_experts=None)


@pytest.mark.parametrize("fmt", [FMT_W4G128, FMT_NVFP4])
@pytest.mark.parametrize("T,sample,tiles", [(1, None, -1), (64, [0, 63], None), (4096, [4095], 24)])
def test_config_deepseek_v3_like(moe, cuda_device, fmt, T, sample, tiles):
    # H7168 I2048 E256 top-8, uniform-random router weights.  T=64: every routed expert's
    # rows; T=4096: the row tiles of 24 experts (the sampled token's, the largest and
    # smallest, evenly spaced ones)
    run_config(moe, fmt, 0x5EED0005, T, 7168, 2048, 256, 8, router="uniform", sample=sample, tile_experts=tiles)
