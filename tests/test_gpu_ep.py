"""Expert parallelism on one GPU with the ranks emulated in one process: every phase of
the layer (prepare, expert, finish) runs in the library's kernels and only the two
all-to-all exchanges are replaced by device slicing.  Each rank's output must equal the
same layer on one device with every expert, bit for bit (shapes are chosen so that both
sides take the same FFN path), and the dispatch counts must equal the oracle's plan."""
import numpy as np
import pytest
import torch

import synth
from layer_inputs import dev_bf16
from oracle.ep import dispatch_plan

pytestmark = pytest.mark.gpu


def _slice(moe, ex, lo, hi):
    g = lambda t: None if t is None else t[lo:hi]
    return moe.Experts(ex.fmt, ex.w13[lo:hi], ex.w13_scale[lo:hi], ex.w2[lo:hi], ex.w2_scale[lo:hi], g(ex.w13_gscale),
                       g(ex.w2_gscale))


@pytest.mark.parametrize("fmt,G,T_per", [(0, 2, [3, 5]), (0, 4, [1, 2, 8, 4]), (2, 2, [6, 2]), (0, 2, [300, 212]),
                                         (0, 2, [0, 4])])
def test_emulated_ranks_equal_single_device(moe, cuda_device, fmt, G, T_per):
    from bit_mixed_precision_router_b200 import ep
    E, H, I, k = 8, 256, 128, 2
    El = E // G
    w13 = synth.normal_bf16(81, E * 2 * I * H, 0.05).reshape(E, 2 * I, H)
    w2 = synth.normal_bf16(82, E * H * I, 0.05).reshape(E, H, I)
    ex = moe.quantize_experts(fmt, dev_bf16(w13), dev_bf16(w2))
    wr = dev_bf16(synth.normal_bf16(83, E * H, 0.05).reshape(E, H))
    xs = [dev_bf16(synth.normal_bf16(90 + r, max(T, 1) * H, 1.0).reshape(max(T, 1), H))[:T] for r, T in
          enumerate(T_per)]
    sent = [ep.ep_prepare(x, wr, None, k) for x in xs]
    counts = [s.counts.cpu().numpy().astype(np.int64) for s in sent]
    send, recv = dispatch_plan([np.concatenate([[0], np.cumsum(c)]) for c in counts], E, G)
    y_arr, recv_splits = [], []
    for d in range(G):
        rc = torch.stack([s.counts[d * El:(d + 1) * El] for s in sent]).contiguous()
        assert np.array_equal(rc.cpu().numpy(), recv[d])
        parts = [s.rows[int(send[r, :d].sum()):int(send[r, :d + 1].sum())] for r, s in enumerate(sent)]
        rows = torch.cat(parts).contiguous()
        y_arr.append(ep.ep_expert(rows, rc, _slice(moe, ex, d * El, (d + 1) * El), I)[:rows.shape[0]])
    for r, (x, s) in enumerate(zip(xs, sent)):
        T = x.shape[0]
        if T == 0:
            continue
        back = []
        for d in range(G):
            start = int(send[:r, d].sum())
            back.append(y_arr[d][start:start + int(send[r, d])])
        y_back = torch.cat(back).contiguous()
        out = ep.ep_finish(y_back, s, T, k, x)
        ro = moe.moe_route_topk(x, wr, None, k)
        ref = moe.moe_combine(moe.moe_grouped_ffn(x, ro, ex, I, E, k), ro, T, k, residual=x)
        moe.moe_check_device_errors()
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), r
