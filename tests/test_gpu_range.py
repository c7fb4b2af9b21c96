"""Activations across the range of the fp16 staging inside the W4 and NVFP4 kernels, through
the GEMV (few rows per expert) and the tcgen05 GEMM (many rows per expert), against the float64
oracle.

The kernels stage the activations in fp16 scaled by a power of two (x/16 and x/256, h/16 or
h/256), which is exact for bf16 values inside fp16's normal range and keeps |x|, |h| below
2^20 (W4) or 2^24 (NVFP4) finite; smaller magnitudes become fp16 subnormals or zero.  Tokens
come at three scales, powers of two of the same seeded rows (exact in bf16):

* unit rows: the FFN tolerance of the other parity tests, per routed row;
* large rows, |h| up to about 2^18 (W4) or 2^22 (NVFP4): max |err| <= 1e-2 max |y_ref| of the row
  plus bf16's half spacing, and relative L2 <= 1e-2 (exact staging of x, h rounded to fp16
  with relative error 2^-11, fp32 sums: the relative error does not grow with the scale);
* tiny rows (x scaled by 2^-9, h around 1e-7: subnormal or zero once staged): the absolute
  staging error, at most eps = 2^-16 per staged x or h value, carried through the down
  projection, |err_i| <= 4 eps sum_j |W2_ij| (4: slack for the quantised weights and the
  x error's small share through gate/up and SiLU), plus bf16's half spacing.
"""
import numpy as np
import pytest
import torch

import synth
from layer_inputs import bf16_half_ulp, check_close, dev_bf16, host_bits, make_layer, oracle_experts
from oracle.ffn import FMT_NVFP4, FMT_W4G128, grouped_ffn
from oracle.routing import permute, router_logits, topk_softmax

pytestmark = pytest.mark.gpu

EPS_STAGE = 2.0 ** -16
BIG = {FMT_W4G128: 2.0 ** 9, FMT_NVFP4: 2.0 ** 11}
TINY = 2.0 ** -9


def _scaled_layer(seed, T, H, I, E, k, big):
    L = make_layer(seed, T, H, I, E, k)
    scale = np.where(np.arange(T) % 3 == 0, big, np.where(np.arange(T) % 3 == 1, TINY, 1.0))
    x = synth.bf16_bits_to_f32(L.x).astype(np.float64) * scale[:, None]
    L.x = synth.f32_to_bf16_bits(x.astype(np.float32)).reshape(T, H)
    return L, scale


@pytest.mark.parametrize("fmt", [FMT_W4G128, FMT_NVFP4])
@pytest.mark.parametrize("T,E,k", [(8, 8, 2), (256, 4, 2)])  # GEMV path, GEMM path
def test_ffn_activation_range(moe, cuda_device, fmt, T, E, k):
    H, I = 256, 128
    L, scale = _scaled_layer(8100 + T + fmt, T, H, I, E, k, BIG[fmt])
    assert (T * k >= 32 * E) == (T == 256)
    ex_o = oracle_experts(fmt, L.w13, L.w2)
    ex_g = moe.quantize_experts(fmt, dev_bf16(L.w13), dev_bf16(L.w2))
    r = moe.moe_route_topk(dev_bf16(L.x), dev_bf16(L.wr), None, k)
    y = moe.moe_grouped_ffn(dev_bf16(L.x), r, ex_g, I, E, k)
    moe.moe_check_device_errors()
    ids, _ = topk_softmax(router_logits(L.x, L.wr, None), k)
    offsets, sp, _ = permute(ids, E)
    assert np.array_equal(r.sorted_pair.cpu().numpy()[:T * k], sp)
    y_ref = grouped_ffn(L.x, offsets, sp, k, ex_o)
    got = synth.bf16_bits_to_f32(host_bits(y)).astype(np.float64)[:T * k]
    assert np.all(np.isfinite(got))
    w2_abs = np.abs(synth.bf16_bits_to_f32(L.w2).astype(np.float64)).sum(axis=2)  # [E][H]
    h_max = 0.0
    for e in range(E):
        for rr in range(offsets[e], offsets[e + 1]):
            s = scale[sp[rr] // k]
            g, want = got[rr], y_ref[rr]
            what = f"fmt={fmt} row {rr} (expert {e}, scale {s})"
            if s == 1.0:
                check_close(g, want, what)
            elif s > 1.0:
                err = np.abs(g - want)
                bound = 1e-2 * np.abs(want).max() + bf16_half_ulp(want)
                assert np.all(err <= bound), f"{what}: abs err {err.max():.3e}"
                assert np.linalg.norm(g - want) <= 1e-2 * np.linalg.norm(want), what
                h_max = max(h_max, np.abs(want).max())
            else:
                bound = 4 * EPS_STAGE * w2_abs[e] + bf16_half_ulp(want)
                assert np.all(np.abs(g - want) <= bound), f"{what}: abs err {np.abs(g - want).max():.3e}"
    assert h_max > 1e3  # the large rows did reach large outputs
