"""The allocation-free router entry point (moe_route_topk_noalloc).

It serves callers that cannot give the library device workspace -- engines that
plan all device memory up front, custom-op hosts that pass only inputs and
outputs, code that runs while a CUDA graph is being captured in global mode --
by keeping the logits scratch and the one-launch router's completion counter in
a fixed device array inside the library.  This file is collected last on
purpose: it must pass both on its own in a fresh process (where its first call
performs the per-device set-up) and after the other GPU tests have used the
library."""
import ctypes

import numpy as np
import pytest
import torch

from layer_inputs import assert_routing_equals_oracle, dev_bf16, make_layer, sentinel_routing

MAX_LOGITS = 65536


def _routing_arrays(r, T, k):
    P = T * k
    return [r.topk_ids.cpu().numpy()[:P], r.topk_w.cpu().numpy()[:P], r.expert_offsets.cpu().numpy(),
            r.sorted_pair.cpu().numpy()[:P], r.pair_to_row.cpu().numpy()[:P], r.expert_list.cpu().numpy()]


def _call_and_compare(moe, L, k, what):
    """One no-alloc call into sentinel-filled outputs, checked against the oracle and
    against moe_route_topk with a fresh workspace."""
    x, wr = dev_bf16(L.x), dev_bf16(L.wr)
    bias = None if L.bias is None else torch.from_numpy(L.bias).cuda()
    got = moe.moe_route_topk_noalloc(x, wr, bias, k, out=sentinel_routing(moe, L.T, L.E, k))
    moe.moe_check_device_errors()
    assert_routing_equals_oracle(got, L, k, what)
    ref = moe.moe_route_topk(x, wr, bias, k, out=sentinel_routing(moe, L.T, L.E, k))
    moe.moe_check_device_errors()
    names = ["topk_ids", "topk_w", "expert_offsets", "sorted_pair", "pair_to_row", "expert_list"]
    for name, u, v in zip(names, _routing_arrays(got, L.T, k), _routing_arrays(ref, L.T, k)):
        if name == "topk_w":
            assert np.abs(u - v).max() <= 1e-6, (what, name)
        elif name == "expert_list":
            n = int(v[0])
            assert u[0] == n and np.array_equal(u[1:1 + n], v[1:1 + n]), (what, name)
        else:
            assert np.array_equal(u, v), (what, name)


# (T, H, E, k, zipf): T * E = 4096, 1024, 512, 64000, 512, 1024, 512.  Calls with T <= 16
# take the one-launch router, which uses the completion counter; the others take the
# multi-launch router and fill a larger part of the array with logits first.
SEQUENCE = [
    (64, 2048, 64, 8, False),
    (16, 2048, 64, 8, False),
    (8, 2048, 64, 8, False),
    (250, 512, 256, 8, True),
    (8, 2048, 64, 8, False),
    (8, 2048, 128, 8, False),
    (8, 2048, 64, 8, False),
]


@pytest.mark.gpu
def test_noalloc_router_matches_oracle_and_workspace_router(moe, cuda_device):
    # Consecutive calls through the C ABI share the one fixed array; shapes change from call
    # to call, so every call finds the array as a different earlier call left it.
    for i, (T, H, E, k, zipf) in enumerate(SEQUENCE):
        L = make_layer(901 + i, T, H, 128, E, k, zipf=zipf, with_experts=False)
        _call_and_compare(moe, L, k, f"call {i} (T={T}, E={E})")


def test_noalloc_router_rejects_too_many_logits():
    import bit_mixed_precision_router_b200 as moe
    lib = moe.load()
    A = 0x10000
    r = moe.RoutingT(A, A, A, A, A, A)
    # T * E = 65537 > the fixed array: a clear shape error, nothing launched
    assert lib.moe_route_topk_noalloc(A, A, None, 65537, 256, 1, 1, ctypes.byref(r), None) == 2
    assert lib.moe_route_topk_noalloc(A, A, None, 257, 256, 256, 8, ctypes.byref(r), None) == 2
    assert lib.moe_route_topk_noalloc(A, A, None, 0, 256, 256, 8, ctypes.byref(r), None) == 0
