"""The N>1 benchmark plumbing on the CPU with two gloo ranks: every rank takes the
same collectives, the reported time is the maximum over ranks, and ranks draw
disjoint synthetic batches (the layer shards by token with no data-path
collective)."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synth


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    r, w, l = bench.dist_env()
    assert (r, w, l) == (rank, world, rank)
    bench.init_dist(world, "gloo")
    bench.barrier(world)
    t = bench.max_over_ranks(1.5 + rank, world, torch.device("cpu"))
    seed = bench.rank_seed(bench.SEED_BASE, rank)
    x = synth.normal_bf16(seed + synth.SEED_X, 64, 1.0)
    q.put((rank, t, seed, x.tobytes()))
    bench.barrier(world)
    dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [2.5, 2.5]  # both ranks report the slowest rank's time
    assert res[0][2] != res[1][2]
    assert res[0][3] != res[1][3]             # disjoint input batches


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.0, 1, torch.device("cpu")) == 3.0
    assert bench.rank_seed(5, 0) == 5
