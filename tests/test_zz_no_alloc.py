"""The allocation-free router entry point (moe_route_topk_noalloc).

It serves callers that cannot give the library device workspace -- engines that
plan all device memory up front, custom-op hosts that pass only inputs and
outputs, code that runs while a CUDA graph is being captured in global mode --
by keeping the logits scratch in a fixed device array inside the library.  This
file is collected last on purpose: it must pass both on its own in a fresh
process (where its first call performs the per-device set-up) and after the
other GPU tests have used the library."""
import ctypes

import numpy as np
import pytest
import torch

from layer_inputs import dev_bf16, make_layer

MAX_LOGITS = 65536


def _routing_arrays(r):
    return [t.cpu().numpy() for t in (r.topk_ids, r.topk_w, r.expert_offsets, r.sorted_pair, r.pair_to_row,
                                      r.expert_list)]


def _compare(moe, L, k):
    x, wr = dev_bf16(L.x), dev_bf16(L.wr)
    bias = None if L.bias is None else torch.from_numpy(L.bias).cuda()
    ref = moe.moe_route_topk(x, wr, bias, k)
    got = moe.moe_route_topk_noalloc(x, wr, bias, k)
    moe.moe_check_device_errors()
    a, b = _routing_arrays(got), _routing_arrays(ref)
    names = ["topk_ids", "topk_w", "expert_offsets", "sorted_pair", "pair_to_row", "expert_list"]
    for name, u, v in zip(names, a, b):
        if name == "topk_w":
            assert np.abs(u - v).max() <= 1e-6, name
        elif name == "expert_list":
            n = int(v[0])
            assert u[0] == n and np.array_equal(u[1:1 + n], v[1:1 + n]), name
        else:
            assert np.array_equal(u, v), name


@pytest.mark.gpu
def test_noalloc_router_matches_workspace_router_twice(moe, cuda_device):
    # Two calls in a row through the C ABI: different shapes, so the second call reuses the
    # shared array after the first one filled a different region of it.
    _compare(moe, make_layer(901, 64, 2048, 128, 64, 8, with_experts=False), 8)      # T*E = 4096
    _compare(moe, make_layer(902, 250, 512, 128, 256, 8, zipf=True, with_experts=False), 8)  # T*E = 64000


def test_noalloc_router_rejects_too_many_logits():
    import bit_mixed_precision_router_b200 as moe
    lib = moe.load()
    A = 0x10000
    r = moe.RoutingT(A, A, A, A, A, A)
    # T * E = 65537 > the fixed array: a clear shape error, nothing launched
    assert lib.moe_route_topk_noalloc(A, A, None, 65537, 256, 1, 1, ctypes.byref(r), None) == 2
    assert lib.moe_route_topk_noalloc(A, A, None, 257, 256, 256, 8, ctypes.byref(r), None) == 2
    assert lib.moe_route_topk_noalloc(A, A, None, 0, 256, 256, 8, ctypes.byref(r), None) == 0
