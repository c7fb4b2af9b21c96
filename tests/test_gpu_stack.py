"""GPU parity of the benchmark's decode stack: 16 chained OLMoE-like W4A16 layers
(H2048 I1024 E64 top-8, residual add, no attention), built and graph-captured
exactly as bench.py's DecodeStack, replayed over 256 steps of fresh seeded
batches, at batch 1 and 8.

At steps 0, 1 and 255 every layer is checked teacher-forced: the oracle runs
layer l on the GPU's own bf16 input to layer l (a bf16 rounding difference in the
residual could otherwise flip a near-tie route and diverge legitimately).  The
routing of every layer (ids, weights, permutation) must equal the oracle's, the
layer output within the FFN tolerance.

The oracle's experts are regenerated on the host from the same counter-based
streams (only the experts a checked step routes to), quantised and dequantised by
the oracle."""
import concurrent.futures as cf
import os

import numpy as np
import pytest
import torch

import synth
from layer_inputs import check_close
from oracle.ffn import FMT_W4G128, moe_layer
from oracle.quant import dequant_w4g128, quantize_w4g128
from oracle.routing import permute, router_logits, topk_softmax

pytestmark = pytest.mark.gpu

STEPS = 256
CHECKED = (0, 1, 255)


class LazyW4Experts:
    """Expert weights of one stack layer, materialised per expert on first use: the
    oracle's W4 quantisation of the bf16 stream slice, dequantised (float32 holds every
    dequantised value exactly)."""
    fmt = FMT_W4G128

    def __init__(self, layer_seed: int, H: int, I: int):
        self.seed, self.H, self.I = layer_seed, H, I
        self.cache = {}

    def load(self, e: int):
        if e in self.cache:
            return
        H, I = self.H, self.I
        w13 = synth.normal_bf16(self.seed + synth.SEED_W13, 2 * I * H, 0.02, start=e * 2 * I * H)
        w2 = synth.normal_bf16(self.seed + synth.SEED_W2, H * I, 0.02, start=e * H * I)
        p13, s13 = quantize_w4g128(w13.reshape(1, 2 * I, H))
        p2, s2 = quantize_w4g128(w2.reshape(1, H, I))
        self.cache[e] = (dequant_w4g128(p13[0], s13[0]).astype(np.float32),
                         dequant_w4g128(p2[0], s2[0]).astype(np.float32))

    def dequant(self, e: int, b: int = 8):
        self.load(int(e))
        return self.cache[int(e)]


def _host(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("batch", [1, 8])
def test_decode_stack_teacher_forced(moe, cuda_device, batch):
    import bench
    L, H, I, E, k = bench.LAYERS, bench.H, bench.I, bench.E, bench.K_TOP
    seed = bench.rank_seed(bench.SEED_BASE, 0)
    stack = bench.DecodeStack(moe, torch, cuda_device, batch, seed, L)
    inputs = torch.empty((STEPS, batch, H), dtype=torch.bfloat16, device=cuda_device)
    moe.moe_synth_normal_bf16(inputs, seed + synth.SEED_X, 1.0)
    stack.xs[0].copy_(inputs[0])
    stack.step()  # eager first call before the capture, as the benchmark does
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(cuda_device)
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap):
        with torch.cuda.graph(graph, stream=cap):
            stack.step()
    torch.cuda.current_stream().wait_stream(cap)
    torch.cuda.synchronize()

    seen = {}  # step -> (xs [L+1] bf16 bits, per-layer routing arrays)
    for s in range(STEPS):
        stack.xs[0].copy_(inputs[s])
        graph.replay()
        if s in CHECKED:
            torch.cuda.synchronize()
            xs = [_host(x) for x in stack.xs]
            rts = [(r.topk_ids.cpu().numpy().reshape(batch, k), r.topk_w.cpu().numpy().reshape(batch, k),
                    r.expert_offsets.cpu().numpy(), r.sorted_pair.cpu().numpy(), r.pair_to_row.cpu().numpy())
                   for r in stack.routings]
            seen[s] = (xs, rts)
    moe.moe_check_device_errors()
    del graph

    # the step inputs themselves are the seeded stream
    for s in CHECKED:
        assert np.array_equal(seen[s][0][0].reshape(-1), synth.normal_bf16(seed + synth.SEED_X, batch * H, 1.0,
                                                                            start=s * batch * H))

    workers = min(16, os.cpu_count() or 1)
    for l in range(L):
        ls = seed + 0x100 * (l + 1)
        wr = synth.normal_bf16(ls + synth.SEED_WR, E * H, 0.02).reshape(E, H)
        ex = LazyW4Experts(ls, H, I)
        routed = set()
        for s in CHECKED:
            ids, w = topk_softmax(router_logits(seen[s][0][l].reshape(batch, H), wr, None), k)
            g_ids, g_w, g_off, g_sp, g_p2r = seen[s][1][l]
            assert np.array_equal(g_ids, ids), f"layer {l} step {s}: routing ids"
            assert np.abs(g_w - w).max() <= 1e-6, f"layer {l} step {s}: routing weights"
            offsets, sp, p2r = permute(ids, E)
            assert np.array_equal(g_off, offsets) and np.array_equal(g_sp, sp) and np.array_equal(g_p2r, p2r), \
                f"layer {l} step {s}: permutation"
            routed.update(int(e) for e in ids.reshape(-1))
        with cf.ThreadPoolExecutor(max_workers=workers) as pool:
            list(pool.map(ex.load, sorted(routed)))
        for s in CHECKED:
            x_in = seen[s][0][l].reshape(batch, H)
            ref, _ = moe_layer(x_in, wr, None, ex, k, residual_bits=x_in)
            got = synth.bf16_bits_to_f32(seen[s][0][l + 1].reshape(batch, H)).astype(np.float64)
            check_close(got, ref, f"layer {l} step {s} (batch {batch})")
