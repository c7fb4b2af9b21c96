"""The binding checks caller-provided buffers (element type and count) before any
pointer reaches the C entry points, which cannot check sizes themselves.  Runs on the
CPU: every rejection happens before a device pointer is taken."""
import pytest
import torch

import bit_mixed_precision_router_b200 as moe


def test_quantiser_outputs():
    w = torch.zeros((2, 16, 256), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="packed"):
        moe.moe_quantize_w4g128(w, packed=torch.zeros((2, 16, 31), dtype=torch.int32))
    with pytest.raises(TypeError, match="scales"):
        moe.moe_quantize_w4g128(w, scales=torch.zeros((2, 16, 2), dtype=torch.float32))
    with pytest.raises(ValueError, match="planes"):
        moe.moe_pack_bitplanes(w, planes=torch.zeros((2, 8, 16, 7), dtype=torch.int32))
    with pytest.raises(ValueError, match="gscale"):
        moe.moe_quantize_nvfp4(w, gscale=torch.zeros(1, dtype=torch.float32))


def test_routing_buffers():
    x = torch.zeros((4, 256), dtype=torch.bfloat16)
    wr = torch.zeros((8, 256), dtype=torch.bfloat16)
    short = moe.Routing.empty(3, 8, 2, "cpu")
    with pytest.raises(ValueError, match="topk_ids"):
        moe.moe_route_topk(x, wr, None, 2, out=short)
    with pytest.raises(ValueError, match="w_router"):  # router rows shorter than the tokens' H
        moe.moe_route_topk(x, torch.zeros((8, 128), dtype=torch.bfloat16), None, 2)
    with pytest.raises(TypeError, match="bias"):
        moe.moe_route_topk_noalloc(x, wr, torch.zeros(8, dtype=torch.float64), 2)
    with pytest.raises(ValueError, match="bits"):
        moe.moe_select_bits(torch.zeros(8), 2, bits=torch.zeros(7, dtype=torch.uint8))


def test_ffn_and_combine_buffers():
    T, H, I, E, k = 4, 256, 128, 8, 2
    x = torch.zeros((T, H), dtype=torch.bfloat16)
    r = moe.Routing.empty(T, E, k, "cpu")
    ex = moe.Experts(moe.FMT_W4G128, torch.zeros((E, 2 * I, H // 8), dtype=torch.int32),
                     torch.zeros((E, 2 * I, H // 128), dtype=torch.bfloat16),
                     torch.zeros((E, H, I // 8), dtype=torch.int32), torch.zeros((E, H, 1), dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="experts buffer 0"):  # 9 experts do not fit the 8-expert buffers
        moe.moe_grouped_ffn(x, moe.Routing.empty(T, E + 1, k, "cpu"), ex, I, E + 1, k)
    with pytest.raises(ValueError, match="y_rows"):
        moe.moe_grouped_ffn(x, r, ex, I, E, k, y_rows=torch.zeros((T * k - 1, H), dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="bits"):
        moe.moe_grouped_ffn(x, r, ex, I, E, k, bits=torch.zeros(T * k - 1, dtype=torch.uint8))
    nv = moe.Experts(moe.FMT_NVFP4, torch.zeros(1, dtype=torch.uint8), torch.zeros(1, dtype=torch.uint8),
                     torch.zeros(1, dtype=torch.uint8), torch.zeros(1, dtype=torch.uint8))
    with pytest.raises(ValueError, match="per-expert scales"):
        moe.moe_grouped_ffn(x, r, nv, I, E, k)
    y = torch.zeros((T * k, H), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="residual"):
        moe.moe_combine(y, r, T, k, residual=torch.zeros((T - 1, H), dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="out"):
        moe.moe_combine(y, r, T, k, out=torch.zeros((T, H - 1), dtype=torch.bfloat16))


def test_allocation_buffers():
    with pytest.raises(ValueError, match="delta"):
        moe.moe_bitplane_distortion(torch.zeros((2, 8, 4, 8), dtype=torch.int32),
                                    torch.zeros((2, 4, 2), dtype=torch.bfloat16),
                                    delta=torch.zeros((2, 8, 255), dtype=torch.float64))
    with pytest.raises(TypeError, match="m"):
        moe.moe_activation_moments(torch.zeros((2, 256), dtype=torch.bfloat16), m=torch.zeros(256))
    with pytest.raises(ValueError, match="expert_offsets"):
        moe.moe_allocate_bits(torch.zeros((4, 8, 128), dtype=torch.float64), torch.zeros(128, dtype=torch.float64),
                              torch.zeros(4, dtype=torch.int32), 3.0)
    with pytest.raises(ValueError, match="bits"):
        moe.moe_expand_bits(torch.zeros(8, dtype=torch.int32), torch.zeros(4, dtype=torch.uint8), 2,
                            bits=torch.zeros(7, dtype=torch.uint8))
