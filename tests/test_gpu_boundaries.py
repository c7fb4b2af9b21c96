"""Expert sizes at the tensor-core paths' boundaries, with routings built directly instead of
by the router, so that every size is hit exactly: experts of 0 and 1 rows; 15, 16 and 17 rows
(in a GEMM batch, experts with at most 16 rows go to the GEMV pass); 191, 192 and 193 rows (the
W4 / NVFP4 GEMM's row tiles of 192); 127, 128, 129, 255 and 256 rows (the W4A4 GEMM's row tiles
of 128).  Each output row is compared with the oracle's grouped FFN on the same routing."""
import numpy as np
import pytest
import torch

import synth
from layer_inputs import check_close, dev_bf16, host_bits, make_layer, oracle_experts
from oracle.ffn import FMT_NVFP4, FMT_W4G128, grouped_ffn
from oracle.routing import permute
from oracle.w4a4 import w4a4_grouped_ffn

pytestmark = pytest.mark.gpu


def routing_for_counts(moe, counts, seed):
    """A top-1 routing in which expert e gets exactly counts[e] tokens (seeded order)."""
    E, T = len(counts), int(sum(counts))
    ids = np.repeat(np.arange(E, dtype=np.int32), counts)
    np.random.default_rng(seed).shuffle(ids)
    ids = ids.reshape(T, 1)
    offsets, sp, p2r = permute(ids, E)
    act = np.nonzero(np.diff(offsets) > 0)[0]
    el = np.zeros(E + 1, np.int32)
    el[0] = act.size
    el[1:1 + act.size] = act
    d = lambda a, dt=np.int32: torch.from_numpy(np.ascontiguousarray(a, dtype=dt).reshape(-1)).cuda()
    r = moe.Routing(d(ids), d(np.ones(T), np.float32), d(offsets), d(sp), d(p2r), d(el))
    return r, np.asarray(offsets), np.asarray(sp)


def _check_rows(got, ref, offsets, what):
    for e in range(len(offsets) - 1):
        lo, hi = offsets[e], offsets[e + 1]
        if hi > lo:
            check_close(got[lo:hi], ref[lo:hi], f"{what}: expert {e} ({hi - lo} rows)")


@pytest.mark.parametrize("fmt", [FMT_W4G128, FMT_NVFP4])
def test_gemm_batch_expert_sizes(moe, cuda_device, fmt):
    counts = [16, 17, 0, 1, 192, 193, 15, 32, 191, 64]
    E, T, H, I = len(counts), sum(counts), 256, 128
    assert T >= 32 * E  # the tensor-core path
    L = make_layer(9100 + fmt, T, H, I, E, 1)
    r, offsets, sp = routing_for_counts(moe, counts, 9101)
    ex_o = oracle_experts(fmt, L.w13, L.w2)
    ex_g = moe.quantize_experts(fmt, dev_bf16(L.w13), dev_bf16(L.w2))
    y = moe.moe_grouped_ffn(dev_bf16(L.x), r, ex_g, I, E, 1)
    moe.moe_check_device_errors()
    got = synth.bf16_bits_to_f32(host_bits(y)).astype(np.float64)[:T]
    _check_rows(got, grouped_ffn(L.x, offsets, sp, 1, ex_o, None), offsets, f"fmt={fmt}")


@pytest.mark.parametrize("H,I", [(512, 256), (768, 384)])  # K = 384: a half-filled last K stage in down
def test_w4a4_expert_sizes(moe, cuda_device, H, I):
    counts = [128, 129, 0, 1, 127, 256, 255, 64]
    E, T = len(counts), sum(counts)
    L = make_layer(9200 + H, T, H, I, E, 1)
    r, offsets, sp = routing_for_counts(moe, counts, 9201)
    ex_o = oracle_experts(FMT_NVFP4, L.w13, L.w2)
    ex_g = moe.quantize_experts(FMT_NVFP4, dev_bf16(L.w13), dev_bf16(L.w2))
    y = moe.moe_grouped_ffn_w4a4(dev_bf16(L.x), r, ex_g, I, E, 1)
    moe.moe_check_device_errors()
    got = synth.bf16_bits_to_f32(host_bits(y)).astype(np.float64)[:T]
    _check_rows(got, w4a4_grouped_ffn(L.x, offsets, sp, 1, ex_o), offsets, "W4A4")
