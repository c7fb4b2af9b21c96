"""Pins of the expert-parallel oracle (oracle/ep.py): ownership and the dispatch plan on a
hand-worked case, conservation of rows, and the layer on G ranks against the same layer
on one device (expert placement must not change the result)."""
import numpy as np
import pytest

import synth
from oracle.ep import dispatch_plan, ep_layer, owner
from oracle.ffn import FMT_NVFP4, FMT_W4G128, Experts, moe_layer
from oracle.quant import quantize_nvfp4, quantize_w4g128
from oracle.routing import permute


def test_owner_and_hand_worked_plan():
    assert [owner(e, 8, 2) for e in range(8)] == [0, 0, 0, 0, 1, 1, 1, 1]
    assert [owner(e, 8, 4) for e in range(8)] == [0, 0, 1, 1, 2, 2, 3, 3]
    # rank 0: two tokens, k = 2: ids (0, 5), (5, 7); rank 1: one token: ids (3, 4)
    off0, _, _ = permute(np.array([[0, 5], [5, 7]]), 8)
    off1, _, _ = permute(np.array([[3, 4]]), 8)
    send, recv = dispatch_plan([off0, off1], 8, 2)
    assert send.tolist() == [[1, 3], [1, 1]]
    assert recv[0, 0].tolist() == [1, 0, 0, 0] and recv[0, 1].tolist() == [0, 0, 0, 1]
    assert recv[1, 0].tolist() == [0, 2, 0, 1] and recv[1, 1].tolist() == [1, 0, 0, 0]


@pytest.mark.parametrize("G", [2, 4])
def test_rows_are_conserved(G):
    rng = np.random.default_rng(G)
    E, k = 16, 4
    offs = [permute(np.stack([rng.choice(E, k, replace=False) for _ in range(int(rng.integers(1, 9)))]), E)[0]
            for _ in range(G)]
    send, recv = dispatch_plan(offs, E, G)
    for s in range(G):
        assert send[s].sum() == offs[s][-1]
        for d in range(G):
            assert recv[d, s].sum() == send[s, d]


@pytest.mark.parametrize("fmt,G", [(FMT_W4G128, 1), (FMT_W4G128, 2), (FMT_W4G128, 4), (FMT_NVFP4, 2)])
def test_ep_layer_equals_single_device_layer(fmt, G):
    H, I, E, k = 256, 128, 8, 2
    w13 = synth.normal_bf16(60, E * 2 * I * H, 0.05).reshape(E, 2 * I, H)
    w2 = synth.normal_bf16(61, E * H * I, 0.05).reshape(E, H, I)
    if fmt == FMT_W4G128:
        a, b = quantize_w4g128(w13), quantize_w4g128(w2)
        ex = Experts(fmt, a[0], a[1], b[0], b[1])
    else:
        a, b = quantize_nvfp4(w13), quantize_nvfp4(w2)
        ex = Experts(fmt, a[0], a[1], b[0], b[1], a[2], b[2])
    wr = synth.normal_bf16(62, E * H, 0.05).reshape(E, H)
    xs = [synth.normal_bf16(70 + r, (3 + r) * H, 1.0).reshape(3 + r, H) for r in range(G)]
    got = ep_layer(xs, wr, None, ex, k, G)
    for x, g in zip(xs, got):
        want, _ = moe_layer(x, wr, None, ex, k, residual_bits=x)
        np.testing.assert_allclose(g, want, rtol=1e-12, atol=1e-12)
