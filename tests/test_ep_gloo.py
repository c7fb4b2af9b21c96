"""The expert-parallel layer's exchange (bit_mixed_precision_router_b200.ep.ep_moe_layer)
on two and four gloo ranks on the CPU.

ep_moe_layer's three phases run the library's CUDA kernels; here each phase is
replaced, inside the worker processes, by the oracle's restatement of the same step
on the host (route + gather rows in sorted-row order; label received rows by local
expert + grouped FFN + rows back to arrival order; combine), so that what runs
unmodified is the part under test: the counts exchange, the send/receive splits
and the two row all-to-alls.  Every rank's output must match the oracle's
single-device layer within the FFN tolerance, and every owner must receive exactly
the rows the oracle's dispatch plan assigns it."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import synth

H, I, E, K = 256, 128, 8, 2


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16).copy()).view(torch.bfloat16)


def _experts(fmt):
    from oracle.ffn import FMT_W4G128, Experts
    from oracle.quant import quantize_nvfp4, quantize_w4g128
    w13 = synth.normal_bf16(60, E * 2 * I * H, 0.05).reshape(E, 2 * I, H)
    w2 = synth.normal_bf16(61, E * H * I, 0.05).reshape(E, H, I)
    if fmt == FMT_W4G128:
        a, b = quantize_w4g128(w13), quantize_w4g128(w2)
        return Experts(fmt, a[0], a[1], b[0], b[1])
    a, b = quantize_nvfp4(w13), quantize_nvfp4(w2)
    return Experts(fmt, a[0], a[1], b[0], b[1], a[2], b[2])


def _worker(rank, world, port, fmt, tokens, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    from bit_mixed_precision_router_b200 import ep
    from oracle.ep import _slice_experts
    from oracle.ffn import combine, grouped_ffn
    from oracle.numerics import bf16_round_bits
    from oracle.routing import permute, router_logits, topk_softmax

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    got_counts = {}

    def cpu_prepare(x, w_router, bias, k):
        xb, wb = _bits(x), _bits(w_router)
        ids, w = topk_softmax(router_logits(xb, wb, None), k)
        off, sp, p2r = permute(ids, wb.shape[0])
        return ep.Sent((ids, w, off, sp, p2r), _bf16(xb[sp // k]), torch.from_numpy(np.diff(off).astype(np.int32)))

    def cpu_expert(recv_rows, recv_counts, experts_local, I_):
        counts = recv_counts.numpy()
        got_counts["recv"] = counts.copy()
        G_, El = counts.shape
        ids = np.concatenate([[j] * int(counts[s, j]) for s in range(G_) for j in range(El)] + [[]]).astype(np.int64)
        if ids.size == 0:
            return torch.empty((0, H), dtype=torch.bfloat16)
        loff, lsp, lp2r = permute(ids.reshape(-1, 1), El)
        y_sorted = grouped_ffn(_bits(recv_rows), loff, lsp, 1, experts_local)
        return _bf16(bf16_round_bits(y_sorted[lp2r].astype(np.float32)))

    def cpu_finish(y_back, sent, T, k, residual):
        ids, w, off, sp, p2r = sent.routing
        yb = synth.bf16_bits_to_f32(_bits(y_back)).astype(np.float64)
        return combine(yb, w, p2r, None if residual is None else _bits(residual))

    ep.ep_prepare, ep.ep_expert, ep.ep_finish = cpu_prepare, cpu_expert, cpu_finish
    ex = _experts(fmt)
    El = E // world
    wr = synth.normal_bf16(62, E * H, 0.05).reshape(E, H)
    T = tokens[rank]
    x = synth.normal_bf16(70 + rank, max(T, 1) * H, 1.0).reshape(max(T, 1), H)[:T]
    out = ep.ep_moe_layer(_bf16(x), _bf16(wr), None, _slice_experts(ex, rank * El, (rank + 1) * El), I, K)
    q.put((rank, np.asarray(out), got_counts["recv"]))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("fmt,tokens", [(0, [3, 5]), (0, [1, 2, 8, 4]), (2, [6, 2]), (0, [0, 4])])
def test_ep_layer_over_gloo_ranks(fmt, tokens):
    from oracle.ep import dispatch_plan
    from oracle.ffn import moe_layer
    from oracle.routing import permute, router_logits, topk_softmax
    from layer_inputs import check_close
    world = len(tokens)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, fmt, tokens, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r, out, recv = q.get(timeout=180)
        res[r] = (out, recv)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    ex = _experts(fmt)
    wr = synth.normal_bf16(62, E * H, 0.05).reshape(E, H)
    xs = [synth.normal_bf16(70 + r, max(T, 1) * H, 1.0).reshape(max(T, 1), H)[:T] for r, T in enumerate(tokens)]
    offs = [permute(topk_softmax(router_logits(x, wr, None), K)[0], E)[0] if x.shape[0] else np.zeros(E + 1, np.int64)
            for x in xs]
    _, recv_plan = dispatch_plan(offs, E, world)
    for r, x in enumerate(xs):
        out, recv = res[r]
        assert np.array_equal(recv, recv_plan[r]), f"rank {r}: rows received per (source, local expert)"
        if x.shape[0] == 0:
            assert out.shape[0] == 0
            continue
        want, _ = moe_layer(x, wr, None, ex, K, residual_bits=x)
        check_close(out, want, f"rank {r} of {world}")
