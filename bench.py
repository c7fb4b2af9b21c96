#!/usr/bin/env python
"""Benchmark of the low-bit routed-expert MoE layer on B200.

Default workload (one JSON line on stdout): the decode stack -- 16 chained
OLMoE-like MoE FFN layers (hidden 2048, expert intermediate 1024, 64 experts,
top-8, SwiGLU, W4A16 group-128 experts, bf16 router), no attention, residual
add between layers, a fresh seeded N(0,1) batch of 8 tokens per step.  One step
= one pass of the whole hot path (router logits, top-k, permutation, grouped
gate/up and down GEMV, combine with residual) through all 16 layers, replayed
as one CUDA graph.  `value` = tokens per second through the 16-layer stack
(a token counts once per step), whole job over all ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--batch B] [--impl reference]
                    [--workload decode|prefill-h2048-e128|prefill-h7168-e256|prefill-h7168-e256-nvfp4|
                                bitplane-h2048-e64]

The prefill workloads (not the default) time one MoE FFN layer on a large batch
of fresh tokens per step -- the tensor-core grouped GEMM path -- and report its
roofline against the measured bf16 tensor peak.  The bitplane workload times one
layer of 8-bitplane experts on 64 tokens per step, each expert read at the width a
budgeted allocation gave it (allocated once, before timing, from a profiling batch;
the allocation kernels' times are reported in the config), against the HBM peak.

Under torchrun each rank runs its own replica on its own seeded batches (the
layer shards by token, no data-path collective): weak scaling, time = max over
ranks of the CUDA-event time of the K steps.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s (decode & prefill); weight-stream HBM GB/s vs B200 peak"
H, I, E, K_TOP, LAYERS = 2048, 1024, 64, 8, 16
SEED_BASE = 0x5EED0002
W4_EXPERT_BYTES = (2 * I * H + H * I) // 2 + (2 * I * (H // 128) + H * (I // 128)) * 2  # packed + bf16 scales
W13_EXPERT_BYTES = 2 * I * H // 2 + 2 * I * (H // 128) * 2
W4_GEMV_LAUNCHES = 2  # kernels of one moe_grouped_ffn call on the W4 weight-streaming path
W2_EXPERT_BYTES = H * I // 2 + H * (I // 128) * 2

# Single-layer workloads (one MoE FFN layer per step on fresh tokens): shapes, routing,
# weight format and seeds.  Decode-sized batches run the weight-streaming GEMV path
# (HBM-bound), prefill-sized ones (T*k >= 32*E, W4 or NVFP4) the tensor-core GEMM path.
_DSV3 = dict(H=7168, I=2048, E=256, k=8, router="uniform", zipf=False, seed=0x5EED0005)
_DSV3_DESC = ("one MoE FFN layer, H7168 I2048 E256 top-8, %s experts, U(-0.02, 0.02) bf16 router, "
              "%d fresh tokens per step")
_W4, _FP4 = "W4A16 g128", "NVFP4 (E2M1, E4M3 per 16, fp32 per tensor)"
LAYER_WORKLOADS = {
    "layer-h2048-e64-t16": dict(T=16, H=2048, I=1024, E=64, k=8, router="normal", zipf=False, seed=0x5EED0001,
                                desc="one MoE FFN layer, H2048 I1024 E64 top-8, W4A16 g128 experts, bf16 router, "
                                     "16 fresh tokens per step"),
    "prefill-h2048-e128": dict(T=2048, H=2048, I=768, E=128, k=8, router="normal", zipf=True, seed=0x5EED0003,
                               desc="one MoE FFN layer, H2048 I768 E128 top-8, W4A16 g128 experts, bf16 router "
                                    "with a Zipf(1.1) rank bias, 2048 fresh tokens per step"),
    "layer-h7168-e256-t1": dict(T=1, desc=_DSV3_DESC % (_W4, 1), **_DSV3),
    "layer-h7168-e256-t64": dict(T=64, desc=_DSV3_DESC % (_W4, 64), **_DSV3),
    "prefill-h7168-e256": dict(T=4096, desc=_DSV3_DESC % (_W4, 4096), **_DSV3),
    "layer-h7168-e256-t1-nvfp4": dict(T=1, fmt="nvfp4", desc=_DSV3_DESC % (_FP4, 1), **_DSV3),
    "layer-h7168-e256-t64-nvfp4": dict(T=64, fmt="nvfp4", desc=_DSV3_DESC % (_FP4, 64), **_DSV3),
    "prefill-h7168-e256-nvfp4": dict(T=4096, fmt="nvfp4", desc=_DSV3_DESC % (_FP4, 4096), **_DSV3),
    "prefill-h7168-e256-w4a4": dict(T=4096, fmt="nvfp4", act="nvfp4",
                                    desc=_DSV3_DESC % (_FP4 + " weights and NVFP4 activations quantised on the fly "
                                                       "(W4A4)", 4096), **_DSV3),
    "bitplane-h2048-e64": dict(T=64, H=2048, I=1024, E=64, k=8, router="normal", zipf=False, seed=0x5EED0004,
                               fmt="bitplane", bits="rule",
                               desc="one MoE FFN layer, H2048 I1024 E64 top-8, 8-bitplane experts, each "
                                    "(token, expert) read at b in {2,3,4,8} planes by routing-score thresholds "
                                    "{0.05,0.15,0.3}, bf16 router, 64 fresh tokens per step"),
    "bitplane-h2048-e64-duorate": dict(T=64, H=2048, I=1024, E=64, k=8, router="normal", zipf=False,
                                       seed=0x5EED0004, fmt="bitplane", bits="allocated", budget=3.0,
                                       choices=(2, 3, 4, 8), profile_tokens=2048,
                                       desc="one MoE FFN layer, H2048 I1024 E64 top-8, 8-bitplane experts read at "
                                            "per-expert widths from a budgeted allocation (3.0 bits per weight of "
                                            "routing-weighted reads over {2,3,4,8}, profiled on 2048 tokens), "
                                            "bf16 router, 64 fresh tokens per step"),
}
PREFILL = LAYER_WORKLOADS

# The records the default run adds to its line (`workloads`), one per benchmark
# configuration besides the headline decode stack at batch 8.
EXTRA_WORKLOADS = ["decode-b1", "layer-h2048-e64-t16", "prefill-h2048-e128", "bitplane-h2048-e64",
                   "bitplane-h2048-e64-duorate", "layer-h7168-e256-t1", "layer-h7168-e256-t64", "prefill-h7168-e256",
                   "layer-h7168-e256-t1-nvfp4", "layer-h7168-e256-t64-nvfp4", "prefill-h7168-e256-nvfp4",
                   "prefill-h7168-e256-w4a4"]
# bitplane experts: bytes of one plane of one expert's w13 + w2, and of their bf16 scales
BP_PLANE_BYTES = (2 * I * H + H * I) // 8
BP_SCALE_BYTES = (2 * I * (H // 128) + H * (I // 128)) * 2


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--workload", choices=["decode"] + sorted(LAYER_WORKLOADS), default="decode")
    ap.add_argument("--workloads", choices=["all", "none"], default="all",
                    help="with the default decode workload at N=1: also time every other benchmark "
                         "configuration and add one record each to the line (`workloads`)")
    ap.add_argument("--steps", type=int, default=None, help="timed steps (default 512 decode, 20 prefill)")
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--batch", type=int, default=8)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cache-slots", type=int, default=0,
                    help="decode with each layer's experts in pinned host memory and this many device slots "
                         "per layer (0: every expert resident in HBM)")
    ap.add_argument("--experts", type=int, default=None,
                    help="single-layer workloads only, for profiling: this many experts instead of the "
                         "configuration's, with the tokens scaled to keep the rows per expert (not a benchmark line)")
    ap.add_argument("--layers", type=int, default=LAYERS,
                    help="layers in the stack (16 is the benchmark workload; fewer only for profiling)")
    args = ap.parse_args(argv)
    if args.steps is None:
        args.steps = default_steps(args.workload)
    return args


def default_steps(workload: str) -> int:
    if workload == "decode":
        return 512
    return 20 if LAYER_WORKLOADS[workload]["T"] >= 2048 else 512 if workload.startswith("bitplane") else 200


# ---------------------------------------------------------------- distributed plumbing
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_dist(world, backend):
    import datetime

    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))


def barrier(world):
    import torch.distributed as dist
    if world > 1:
        dist.barrier()


def max_over_ranks(value: float, world: int, device) -> float:
    """Largest value over all ranks (every rank takes this collective)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(base: int, rank: int) -> int:
    """Per-rank stream of step inputs: ranks process disjoint synthetic batches."""
    return base + 0x10000 * rank


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self) -> dict:
        time.sleep(0.1)
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait(timeout=10)
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        smax = max(r[1] for r in rows)
        loaded = [r for r in rows if r[0] > 0.5 * smax] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[2]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": smax, "reasons": reasons,
                "samples": len(rows)}


# ---------------------------------------------------------------- peaks
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, "fallback"


def committed_traffic(name: str = "traffic.json"):
    """DRAM bytes of moe_grouped_ffn calls (gate/up + down launches) from the committed
    ncu summary, with the kernel source hash it was taken on (None if stale/absent)."""
    path = os.path.join(ROOT, "profiles", name)
    try:
        d = json.load(open(path))
    except (OSError, ValueError):
        return None
    if d.get("source_hash") != kernel_source_hash():
        return None
    return d


def kernel_source_hash() -> str:
    """Hash of the GEMV source's code (comment lines and blank lines left out), which keys
    the committed DRAM-traffic records: they count only for the code they were taken on."""
    import hashlib
    h = hashlib.sha256()
    p = os.path.join(ROOT, "bit_mixed_precision_router_b200", "csrc", "moe_ffn_gemv.cu")
    for line in open(p, encoding="utf-8"):
        t = line.strip()
        if t and not t.startswith("//"):
            h.update(t.encode() + b"\n")
    return h.hexdigest()[:16]


# ---------------------------------------------------------------- the GPU arm
class DecodeStack:
    """16 chained W4A16 layers on one device, with every buffer a step needs."""

    def __init__(self, moe, torch, device, batch: int, seed: int, layers: int = LAYERS):
        self.moe, self.torch, self.dev, self.B = moe, torch, device, batch
        self.L = layers
        import synth
        self.layers = []
        tmp13 = torch.empty((E, 2 * I, H), dtype=torch.bfloat16, device=device)
        tmp2 = torch.empty((E, H, I), dtype=torch.bfloat16, device=device)
        for l in range(layers):
            ls = seed + 0x100 * (l + 1)
            wr = torch.empty((E, H), dtype=torch.bfloat16, device=device)
            moe.moe_synth_normal_bf16(wr, ls + synth.SEED_WR, 0.02)
            moe.moe_synth_normal_bf16(tmp13, ls + synth.SEED_W13, 0.02)
            moe.moe_synth_normal_bf16(tmp2, ls + synth.SEED_W2, 0.02)
            ex = moe.quantize_experts(moe.FMT_W4G128, tmp13, tmp2)
            self.layers.append((wr, ex))
        del tmp13, tmp2
        B = batch
        # one routing per layer: after a step every layer's routing is still readable
        self.routings = [moe.Routing.empty(B, E, K_TOP, device) for _ in range(layers)]
        self.routing = self.routings[0]
        self.route_ws = moe.moe_route_workspace(B, E, K_TOP, device)
        self.ffn_ws = torch.empty(max(moe.moe_ffn_workspace_bytes(B, H, I, E, K_TOP, moe.FMT_W4G128), 16),
                                  dtype=torch.uint8, device=device)
        self.y_rows = torch.empty((B * K_TOP, H), dtype=torch.bfloat16, device=device)
        self.xs = [torch.empty((B, H), dtype=torch.bfloat16, device=device) for _ in range(layers + 1)]
        self.n_active = torch.zeros((layers,), dtype=torch.int32, device=device)
        self.ffn_events = None

    def layer(self, l, log_active=False):
        moe, wr_ex = self.moe, self.layers[l]
        wr, ex = wr_ex
        x, nxt, r = self.xs[l], self.xs[l + 1], self.routings[l]
        moe.moe_route_topk(x, wr, None, K_TOP, out=r, workspace=self.route_ws)
        if self.ffn_events is not None:
            self.ffn_events[l][0].record()
        moe.moe_grouped_ffn(x, r, ex, I, E, K_TOP, y_rows=self.y_rows, workspace=self.ffn_ws)
        if self.ffn_events is not None:
            self.ffn_events[l][1].record()
        moe.moe_combine(self.y_rows, r, self.B, K_TOP, residual=x, out=nxt)
        if log_active:
            self.n_active[l:l + 1].copy_(r.expert_list[:1])

    def step(self, log_active=False):
        for l in range(self.L):
            self.layer(l, log_active)

    @property
    def kernels_per_step(self):
        # router: one launch for up to 16 tokens whose bf16 rows fit 64 KiB, else logits,
        # top-k and permutation; then the grouped FFN (W4_GEMV_LAUNCHES) and the combine
        route = 1 if fused_router(self.B, H) else 3
        return self.L * (route + W4_GEMV_LAUNCHES + 1)


class CachedDecodeStack(DecodeStack):
    """The decode stack with every layer's experts in pinned host memory and S device
    slots per layer: route, plan the step on the device, permute the pairs by slot, fetch
    the missing experts over the host link, FFN on the slots, combine."""

    def __init__(self, moe, torch, device, batch: int, seed: int, layers: int, slots: int):
        super().__init__(moe, torch, device, batch, seed, layers)
        S, B = slots, batch
        self.S = S
        pin = lambda t: t.cpu().pin_memory()
        zeros = lambda t: torch.zeros((S,) + tuple(t.shape[1:]), dtype=t.dtype, device=device)
        self.host, self.slots, self.states, self.plans = [], [], [], []
        for l in range(layers):
            wr, ex = self.layers[l]
            self.host.append(moe.Experts(ex.fmt, pin(ex.w13), pin(ex.w13_scale), pin(ex.w2), pin(ex.w2_scale)))
            self.slots.append(moe.Experts(ex.fmt, zeros(ex.w13), zeros(ex.w13_scale), zeros(ex.w2),
                                          zeros(ex.w2_scale)))
            self.states.append(moe.moe_cache_state_device(E, S, 1, device))
            self.plans.append(moe.CachePlan.empty(E, device))
            self.layers[l] = (wr, None)  # the device copy of the experts is dropped
        torch.cuda.empty_cache()
        i32 = dict(dtype=torch.int32, device=device)
        self.slot_ids = torch.empty(B * K_TOP, **i32)
        self.rs = moe.Routing(self.slot_ids, self.routing.topk_w, torch.empty(S + 1, **i32),
                              torch.empty(B * K_TOP, **i32), torch.empty(B * K_TOP, **i32), torch.empty(S + 1, **i32))
        self.ffn_ws = torch.empty(max(moe.moe_ffn_workspace_bytes(B, H, I, S, K_TOP, moe.FMT_W4G128), 16),
                                  dtype=torch.uint8, device=device)
        self.fetch_events = None

    def layer(self, l, log_active=False):
        moe = self.moe
        wr, _ = self.layers[l]
        x, nxt = self.xs[l], self.xs[l + 1]
        moe.moe_route_topk(x, wr, None, K_TOP, out=self.routing, workspace=self.route_ws)
        moe.moe_cache_step(self.states[l], E, self.S, self.routing, self.B, K_TOP, slot_ids=self.slot_ids,
                           plan=self.plans[l])
        moe.moe_permute(self.slot_ids, self.B, K_TOP, self.S, out=self.rs)
        if self.fetch_events is not None:
            self.fetch_events[l][0].record()
        moe.moe_cache_fetch(self.plans[l], E, self.host[l], self.slots[l], H, I)
        if self.fetch_events is not None:
            self.fetch_events[l][1].record()
        moe.moe_grouped_ffn(x, self.rs, self.slots[l], I, self.S, K_TOP, y_rows=self.y_rows, workspace=self.ffn_ws)
        moe.moe_combine(self.y_rows, self.rs, self.B, K_TOP, residual=x, out=nxt)
        if log_active:
            self.n_active[l:l + 1].copy_(self.routing.expert_list[:1])

    def step(self, log_active=False):
        for l in range(self.L):
            self.layer(l, log_active)

    def fetched(self):
        """(bytes copied over the host link, experts served, hits) of the last step, all layers."""
        total = served = hits = 0
        for plan in self.plans:
            n = int(plan.nserved.item())
            lo = plan.fetch_lo[:n].cpu().tolist()
            hi = plan.fetch_hi[:n].cpu().tolist()
            total += sum(W4_EXPERT_BYTES for a, b in zip(lo, hi) if b > a)
            served += n
            hits += sum(1 for a, b in zip(lo, hi) if a == b)
        return total, served, hits

    @property
    def kernels_per_step(self):
        # router, cache step, permutation by slot, fetch (w13, w2), gate/up, down, combine
        route = 1 if (self.B <= 16 and self.B * H * 2 <= 64 * 1024) else 3
        return self.L * (route + 7)


def measured_h2d_gbs(torch, device, nbytes: int = 256 << 20) -> float:
    """Pinned host -> device copy bandwidth (median of 5 copies of 256 MB), the peak of the
    host link the slot cache reads over."""
    src = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    dst = torch.empty(nbytes, dtype=torch.uint8, device=device)
    dst.copy_(src, non_blocking=True)
    torch.cuda.synchronize()
    ts = []
    for _ in range(5):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        dst.copy_(src, non_blocking=True)
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b) / 1e3)
    return nbytes / statistics.median(ts) / 1e9


def run_gpu(args, rank, world, local):
    import torch
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist(world, "nccl")
    import bit_mixed_precision_router_b200 as moe
    moe.load()
    W = max(args.warmup, 3)
    rec = bench_stack(moe, torch, device, args.batch, args.steps, W, rank, world, local, args.layers,
                      e2e=not args.no_e2e, cache_slots=args.cache_slots)
    extra = []
    if world == 1 and args.workloads == "all" and not args.cache_slots and args.layers == LAYERS:
        for name in EXTRA_WORKLOADS:
            try:
                if name == "decode-b1":
                    r = bench_stack(moe, torch, device, 1, 512, W, rank, world, local, LAYERS, e2e=not args.no_e2e)
                else:
                    r = bench_layer(moe, torch, device, LAYER_WORKLOADS[name], default_steps(name), W, rank, world,
                                    local, e2e=not args.no_e2e)
            except Exception as exc:  # a failed record is reported, the others still run
                r = {"error": f"{type(exc).__name__}: {exc}"}
                torch.cuda.empty_cache()
            r["name"] = name
            extra.append(r)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return None
    line = line_from_record(rec, world)
    if extra:
        line["workloads"] = extra
    return line


def bench_stack(moe, torch, device, B, K, W, rank, world, local, L, e2e=True, cache_slots=0):
    """Times the decode stack: K replays of one CUDA graph holding all L layers, each step on
    a fresh seeded batch of B tokens resident in HBM; then the same through pinned host
    buffers (e2e); then the dominant op's roofline."""
    import synth
    seed = rank_seed(SEED_BASE, rank)
    if cache_slots:
        if not (1 <= cache_slots <= E and cache_slots >= min(E, B * K_TOP)):
            raise SystemExit("--cache-slots must be in [min(E, batch * top-k), E]")
        stack = CachedDecodeStack(moe, torch, device, B, seed, L, cache_slots)
    else:
        stack = DecodeStack(moe, torch, device, B, seed, L)
    # a fresh seeded N(0,1) batch for every step (warm-up and timed), resident in HBM
    n_steps = W + K
    inputs = torch.empty((n_steps, B, H), dtype=torch.bfloat16, device=device)
    moe.moe_synth_normal_bf16(inputs, seed + synth.SEED_X, 1.0)
    torch.cuda.synchronize()

    # eager warm-up (first calls resolve the device symbol before graph capture)
    for s in range(2):
        stack.xs[0].copy_(inputs[s])
        stack.step()
    torch.cuda.synchronize()
    moe.moe_check_device_errors()

    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(device)
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap):
        with torch.cuda.graph(graph, stream=cap):
            stack.step()
    torch.cuda.current_stream().wait_stream(cap)
    torch.cuda.synchronize()

    for s in range(W):
        stack.xs[0].copy_(inputs[s])
        graph.replay()
    torch.cuda.synchronize()
    barrier(world)

    clocks = ClockSampler(local)
    clocks.start()
    torch.cuda.synchronize()
    barrier(world)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    for s in range(W, W + K):
        stack.xs[0].copy_(inputs[s])
        graph.replay()
    ev1.record()
    torch.cuda.synchronize()
    barrier(world)
    ms_local = ev0.elapsed_time(ev1)
    clk = clocks.stop()
    moe.moe_check_device_errors()
    ms = max_over_ranks(ms_local, world, device)
    tokens = B * K * world
    value = tokens / (ms / 1e3)

    # ---- end-to-end through the public API with host buffers (pinned), copies timed
    e2e_rec = None
    if e2e:
        host_in = inputs.cpu().pin_memory()
        host_out = torch.empty((K, B, H), dtype=torch.bfloat16).pin_memory()
        barrier(world)
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        for s in range(W, W + K):
            stack.xs[0].copy_(host_in[s], non_blocking=True)
            graph.replay()
            host_out[s - W].copy_(stack.xs[L], non_blocking=True)
        t1.record()
        torch.cuda.synchronize()
        barrier(world)
        e2e_ms = max_over_ranks(t0.elapsed_time(t1), world, device)
        e2e_rec = {"value": round(tokens / (e2e_ms / 1e3), 1), "unit": "tokens/s", "h2d_bytes_per_step": B * H * 2,
                   "d2h_bytes_per_step": B * H * 2}

    if cache_slots:
        roofline, act = cached_roofline(torch, device, stack, cap, inputs, W, K)
    else:
        roofline, act = resident_roofline(torch, stack, cap, inputs, W, K, B)
    cfg_extra = {} if not cache_slots else {
        "cache": "experts of each layer in pinned host memory, %d device slots per layer, planned on the "
                 "device each step, missing experts read over the host link" % cache_slots}
    rec = {
        "value": round(value, 1), "unit": "tokens/s", "steps": K, "warmup": W, "ms_per_step": round(ms / K, 4),
        "dtype": "bf16", "data": "synthetic (seeded Irwin-Hall N(0,1) activations, N(0,0.02) bf16 weights "
                                 "quantised to W4A16 g128)",
        "config": dict({"workload": "decode stack: %d chained OLMoE-like MoE FFN layers (H2048 I1024 E64 "
                                    "top-8, W4A16 g128 experts, bf16 router), residual add, batch %d "
                                    "tokens/step" % (L, B),
                        "layers": L, "batch": B, "hidden": H, "intermediate": I, "experts": E, "top_k": K_TOP,
                        "parallelism": f"dp{world} (independent replicas)",
                        "l2": "no flush: each step streams ~%.1f GB of distinct expert weights, > 126 MB L2"
                              % (statistics.mean(act) * W4_EXPERT_BYTES * L / 1e9)}, **cfg_extra),
        "gpu_launches": stack.kernels_per_step * K,
        "clocks": clk, "roofline": roofline, "e2e": e2e_rec,
    }
    del graph, stack, inputs
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return rec


def cached_roofline(torch, device, stack, cap, inputs, W, K):
    """The fetch (moe_cache_fetch, both launches) against the measured pinned host ->
    device bandwidth: bytes copied over the host link per call / its event-timed duration."""
    stack.fetch_events = [(torch.cuda.Event(enable_timing=True, external=True),
                           torch.cuda.Event(enable_timing=True, external=True)) for _ in range(stack.L)]
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.stream(cap):
        with torch.cuda.graph(g2, stream=cap):
            stack.step(log_active=True)
    torch.cuda.current_stream().wait_stream(cap)
    ms, nbytes, served, hits, act = 0.0, 0, 0, 0, []
    for s in range(W, W + min(K, 32)):
        stack.xs[0].copy_(inputs[s])
        g2.replay()
        torch.cuda.synchronize()
        ms += sum(a.elapsed_time(b) for a, b in stack.fetch_events)
        b_, n_, h_ = stack.fetched()
        nbytes, served, hits = nbytes + b_, served + n_, hits + h_
        act += stack.n_active.cpu().tolist()
    stack.fetch_events = None
    del g2
    peak = measured_h2d_gbs(torch, device)
    achieved = nbytes / (ms / 1e3) / 1e9 if ms > 0 else 0.0
    return ({"bound": "host-link", "achieved": round(achieved, 1), "peak": round(peak, 1), "unit": "GB/s",
             "frac": round(achieved / peak, 4), "peak_kind": "measured pinned host->device copy in this run",
             "traffic": None, "kernel": "k_cache_fetch (w13 + w2 of the missing experts, one moe_cache_fetch call)",
             "fetched_bytes_per_step": round(nbytes / min(K, 32)),
             "hit_rate": round(hits / served, 4) if served else None}, act)


def resident_roofline(torch, stack, cap, inputs, W, K, B):
    # ---- roofline of the dominant op: the grouped W4 GEMV (gate/up + down launches of
    # moe_grouped_ffn), timed with CUDA events recorded on its stream inside a graph
    stack.ffn_events = [(torch.cuda.Event(enable_timing=True, external=True),
                         torch.cuda.Event(enable_timing=True, external=True)) for _ in range(stack.L)]
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.stream(cap):
        with torch.cuda.graph(g2, stream=cap):
            stack.step(log_active=True)
    torch.cuda.current_stream().wait_stream(cap)
    ffn_ms, act = [], []
    n_meas = min(K, 64)
    for s in range(W, W + n_meas):
        stack.xs[0].copy_(inputs[s])
        g2.replay()
        torch.cuda.synchronize()
        ffn_ms += [a.elapsed_time(b) for a, b in stack.ffn_events]
        act += stack.n_active.cpu().tolist()
    stack.ffn_events = None
    hbm, bf16_peak, peak_kind = measured_peaks()
    act_bytes = B * H * 2 + B * K_TOP * I * 2 * 2 + B * K_TOP * H * 2  # x, h (write+read), y_rows
    algo_bytes = statistics.mean(a * W4_EXPERT_BYTES for a in act) + act_bytes
    avg_ffn_s = statistics.mean(ffn_ms) / 1e3
    achieved = algo_bytes / avg_ffn_s / 1e9
    traffic = committed_traffic()
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(achieved / hbm, 4), "peak_kind": peak_kind,
                "traffic": round(traffic["dram_bytes_per_expert"] * statistics.mean(act)) if traffic else None,
                "kernel": "k_ffn_gemv<W4> gate/up + down (one moe_grouped_ffn call)",
                "algorithmic_bytes_per_call": round(algo_bytes), "avg_call_us": round(avg_ffn_s * 1e6, 2),
                "distinct_experts_per_layer": round(statistics.mean(act), 2)}
    del g2
    return roofline, act


# ---------------------------------------------------------------- single-layer workloads
L2_BYTES = 126 * 1000 ** 2


def expert_bytes(cfg) -> int:
    """Packed weights + scales of one expert (w13 and w2) in the workload's format."""
    n = 3 * cfg["H"] * cfg["I"]  # weights per expert
    fmt = cfg.get("fmt")
    if fmt == "nvfp4":
        return n // 2 + n // 16 + 8
    if fmt == "bitplane":
        return n + n // 128 * 2
    return n // 2 + n // 128 * 2


def gemm_path(cfg) -> bool:
    """moe_grouped_ffn's own choice: the tensor-core GEMM for W4 / NVFP4 batches with
    T*k >= 32*E, else the weight-streaming GEMV (W4A4 always takes the GEMM)."""
    if cfg.get("act") == "nvfp4":
        return True
    return cfg.get("fmt") != "bitplane" and cfg["T"] * cfg["k"] >= 32 * cfg["E"]


def fused_router(T: int, Hh: int) -> bool:
    return T <= 16 and T * Hh * 2 <= 64 * 1024


class PrefillLayer:
    """One MoE FFN layer made on the device (seeded generator, quantised in chunks of
    experts) with every buffer a step needs.  Steps rotate over device copies of the
    weights where one copy would sit in the 126 MB L2 between steps."""

    def __init__(self, moe, torch, device, cfg, chunk=16):
        import synth
        self.moe, self.cfg = moe, cfg
        T, Hh, Ii, Ee, k = cfg["T"], cfg["H"], cfg["I"], cfg["E"], cfg["k"]
        seed = cfg["seed"]
        i32, bf = dict(dtype=torch.int32, device=device), dict(dtype=torch.bfloat16, device=device)
        u8, f32 = dict(dtype=torch.uint8, device=device), dict(dtype=torch.float32, device=device)
        self.fmt = {"nvfp4": moe.FMT_NVFP4, "bitplane": moe.FMT_BITPLANE8}.get(cfg.get("fmt"), moe.FMT_W4G128)
        if self.fmt == moe.FMT_NVFP4:
            mk = lambda n, kk: (torch.empty((Ee, n, kk // 2), **u8), torch.empty((Ee, n, kk // 16), **u8),
                                torch.empty((Ee,), **f32))
        elif self.fmt == moe.FMT_BITPLANE8:
            mk = lambda n, kk: (torch.empty((Ee, 8, n, kk // 32), **i32), torch.empty((Ee, n, kk // 128), **bf),
                                None)
        else:
            mk = lambda n, kk: (torch.empty((Ee, n, kk // 8), **i32), torch.empty((Ee, n, kk // 128), **bf), None)
        w13, w2 = mk(2 * Ii, Hh), mk(Hh, Ii)
        tmp = torch.empty((chunk * 2 * Ii * Hh,), **bf)
        for (n, kk, tag, st) in ((2 * Ii, Hh, synth.SEED_W13, w13), (Hh, Ii, synth.SEED_W2, w2)):
            for e0 in range(0, Ee, chunk):
                ne = min(chunk, Ee - e0)
                t = tmp[:ne * n * kk].view(ne, n, kk)
                moe.moe_synth_normal_bf16(t, seed + tag, 0.02, start=e0 * n * kk)
                if self.fmt == moe.FMT_NVFP4:
                    moe.moe_quantize_nvfp4(t, st[0][e0:e0 + ne], st[1][e0:e0 + ne], st[2][e0:e0 + ne])
                elif self.fmt == moe.FMT_BITPLANE8:
                    moe.moe_pack_bitplanes(t, st[0][e0:e0 + ne], st[1][e0:e0 + ne])
                else:
                    moe.moe_quantize_w4g128(t, st[0][e0:e0 + ne], st[1][e0:e0 + ne])
        del tmp
        self.experts = moe.Experts(self.fmt, w13[0], w13[1], w2[0], w2[1], w13[2], w2[2])
        self.wr = torch.empty((Ee, Hh), **bf)
        if cfg["router"] == "uniform":
            moe.moe_synth_uniform_bf16(self.wr, seed + synth.SEED_WR, -0.02, 0.02)
        else:
            moe.moe_synth_normal_bf16(self.wr, seed + synth.SEED_WR, 0.02)
        self.bias = torch.from_numpy(synth.zipf_rank_bias(seed + synth.SEED_BIAS, Ee)).to(device) \
            if cfg["zipf"] else None
        self.routing = moe.Routing.empty(T, Ee, k, device)
        self.route_ws = moe.moe_route_workspace(T, Ee, k, device)
        self.w4a4 = cfg.get("act") == "nvfp4"
        ws_bytes = (moe.moe_ffn_w4a4_workspace_bytes(T, Hh, Ii, Ee, k) if self.w4a4
                    else moe.moe_ffn_workspace_bytes(T, Hh, Ii, Ee, k, self.fmt))
        self.ffn_ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=device)
        self.y_rows = torch.empty((T * k, Hh), **bf)
        self.x = torch.empty((T, Hh), **bf)
        self.out = torch.empty((T, Hh), **bf)
        self.ffn_events = None
        self.bits_e = self.bits = None
        self.n_active = torch.zeros((1,), **i32)
        if self.fmt == moe.FMT_BITPLANE8:
            self.bits = torch.empty((T * k,), **u8)
        # copies of the weights to rotate over: a step of the bitplane layer reads ~160 MB of
        # planes, the H2048 W4 layer ~180 MB of its 207 MB, near the 126 MB L2; 4 * L2 bytes
        # in rotation make sure no step finds the previous steps' weights in L2
        total = Ee * expert_bytes(cfg)
        n_copies = 4 if self.fmt == moe.FMT_BITPLANE8 else max(1, min(4, -(-4 * L2_BYTES // total)))
        self.copies = [self.experts]
        g = lambda t: None if t is None else t.clone()
        for _ in range(n_copies - 1):
            self.copies.append(moe.Experts(self.fmt, w13[0].clone(), w13[1].clone(), w2[0].clone(), w2[1].clone(),
                                           g(w13[2]), g(w2[2])))
        if self.w4a4:  # the weight scales in tensor-core order: part of the weights, made untimed
            for ex in self.copies:
                ex.w4a4_tiles = moe.moe_w4a4_prepare(ex, Hh, Ii, Ee)

    def allocate_widths(self, torch, device, seed):
        """Per-expert widths for the bitplane experts under the read budget: the distortion
        tensor of the gate/up matrices (offline), the activation moments of a profiling
        batch of the workload, the routing counts of that batch, then the allocation.
        Each of the three kernels is timed with CUDA events (median of 5)."""
        import synth
        moe, c = self.moe, self.cfg
        xp = torch.empty((c["profile_tokens"], c["H"]), dtype=torch.bfloat16, device=device)
        moe.moe_synth_normal_bf16(xp, seed + synth.SEED_X + 0x51, 1.0)
        rp = moe.moe_route_topk(xp, self.wr, self.bias, c["k"])
        delta = torch.empty((c["E"], 8, c["H"]), dtype=torch.float64, device=device)
        m = torch.empty((c["H"],), dtype=torch.float64, device=device)
        lam = torch.zeros((), dtype=torch.float64, device=device)
        self.bits_e = torch.empty((c["E"],), dtype=torch.uint8, device=device)
        times = {"distortion": [], "moments": [], "allocate": []}
        for _ in range(5):
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            ev[0].record()
            moe.moe_bitplane_distortion(self.experts.w13, self.experts.w13_scale, delta=delta)
            ev[1].record()
            moe.moe_activation_moments(xp, m=m)
            ev[2].record()
            moe.moe_allocate_bits(delta, m, rp.expert_offsets, c["budget"], choices=c["choices"],
                                  bits_e=self.bits_e, lam=lam)
            ev[3].record()
            torch.cuda.synchronize()
            for i, key in enumerate(times):
                times[key].append(ev[i].elapsed_time(ev[i + 1]) * 1e3)
        moe.moe_check_device_errors()
        counts = torch.diff(rp.expert_offsets.to(torch.int64)).cpu()
        be = self.bits_e.cpu().to(torch.int64)
        hist = {str(b): int((be == b).sum()) for b in c["choices"]}
        return {"budget_bits_per_weight": c["budget"], "choices": list(c["choices"]),
                "profile_tokens": c["profile_tokens"], "widths_histogram": hist,
                "profile_read_rate": round(float((counts * be).sum()) / float(counts.sum()), 4),
                "resident_rate_mean_width": round(float(be.double().mean()), 4), "lambda": lam.item(),
                "kernel_us": {key: round(statistics.median(v), 1) for key, v in times.items()}}

    def step(self, copy: int = 0, log_active: bool = False):
        moe, c = self.moe, self.cfg
        moe.moe_route_topk(self.x, self.wr, self.bias, c["k"], out=self.routing, workspace=self.route_ws)
        if self.bits is not None:
            if c["bits"] == "rule":  # b from the routing weights by thresholds (0.05, 0.15, 0.3)
                moe.moe_select_bits(self.routing.topk_w, c["k"], bits=self.bits)
            else:  # per-expert widths of the budgeted allocation
                moe.moe_expand_bits(self.routing.topk_ids, self.bits_e, c["k"], bits=self.bits)
        if self.ffn_events is not None:
            self.ffn_events[0].record()
        if self.w4a4:
            moe.moe_grouped_ffn_w4a4(self.x, self.routing, self.copies[copy], c["I"], c["E"], c["k"],
                                     y_rows=self.y_rows, workspace=self.ffn_ws)
        else:
            moe.moe_grouped_ffn(self.x, self.routing, self.copies[copy], c["I"], c["E"], c["k"], y_rows=self.y_rows,
                                workspace=self.ffn_ws, bits=self.bits)
        if self.ffn_events is not None:
            self.ffn_events[1].record()
        moe.moe_combine(self.y_rows, self.routing, c["T"], c["k"], residual=self.x, out=self.out)
        if log_active:
            self.n_active.copy_(self.routing.expert_list[:1])

    @property
    def kernels_per_step(self):
        c = self.cfg
        route = 1 if fused_router(c["T"], c["H"]) else 3  # logits + top-k + permutation otherwise
        widths = 1 if self.bits is not None else 0        # select_bits / expand_bits
        if self.w4a4:  # row-tile prefix; x: amax, codes, routed codes + tiled scales; gate/up; h: codes,
            ffn = 8        # tiled scales; down
        else:
            # GEMM batches: gather, gate/up GEMM + GEMV pass over the small experts, down likewise
            ffn = 5 if gemm_path(c) else W4_GEMV_LAUNCHES if self.fmt == self.moe.FMT_W4G128 else 2
        return route + widths + ffn + 1                   # + combine


def run_prefill(args, rank, world, local):
    """A single-layer workload as the line's main measurement (`--workload`)."""
    import torch
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist(world, "nccl")
    import bit_mixed_precision_router_b200 as moe
    moe.load()
    cfg = LAYER_WORKLOADS[args.workload]
    if args.experts:
        cfg = dict(cfg, E=args.experts, T=max(1, cfg["T"] * args.experts // cfg["E"]),
                   desc=cfg["desc"] + " -- profiling scale: %d experts, tokens scaled to keep the rows per expert"
                        % args.experts)
    rec = bench_layer(moe, torch, device, cfg, args.steps, max(args.warmup, 3), rank,
                      world, local, e2e=not args.no_e2e)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return None
    return line_from_record(rec, world)


def line_from_record(rec, world):
    """The contract's JSON line from a workload record."""
    out = {"metric": METRIC, "value": rec["value"], "unit": "tokens/s", "n_gpus": world, "steps": rec["steps"],
           "warmup": rec["warmup"], "ms_per_step": rec["ms_per_step"], "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None}
    out.update({k: v for k, v in rec.items() if k not in out and k != "name"})
    return out


def bench_layer(moe, torch, device, cfg, K, W, rank, world, local, e2e=True):
    """Times one single-layer workload: K graph replays (W warm-up), each a step on fresh
    tokens resident in HBM; then the same through pinned host buffers (e2e); then the
    dominant op's roofline from CUDA events around moe_grouped_ffn inside a graph."""
    import synth
    T, Hh, Ii, Ee, k = cfg["T"], cfg["H"], cfg["I"], cfg["E"], cfg["k"]
    layer = PrefillLayer(moe, torch, device, cfg)
    allocation = layer.allocate_widths(torch, device, rank_seed(cfg["seed"], rank)) \
        if cfg.get("bits") == "allocated" else None
    inputs = torch.empty((W + K, T, Hh), dtype=torch.bfloat16, device=device)
    moe.moe_synth_normal_bf16(inputs, rank_seed(cfg["seed"], rank) + synth.SEED_X, 1.0)
    torch.cuda.synchronize()
    layer.x.copy_(inputs[0])
    layer.step()  # eager first call: device symbols and kernel attributes before capture
    torch.cuda.synchronize()
    moe.moe_check_device_errors()
    nc = len(layer.copies)
    graphs = [torch.cuda.CUDAGraph() for _ in range(nc)]
    cap = torch.cuda.Stream(device)
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap):
        for c_, graph in enumerate(graphs):
            with torch.cuda.graph(graph, stream=cap):
                layer.step(c_)
    torch.cuda.current_stream().wait_stream(cap)
    for s in range(W):
        layer.x.copy_(inputs[s])
        graphs[s % nc].replay()
    torch.cuda.synchronize()
    barrier(world)
    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    for s in range(W, W + K):
        layer.x.copy_(inputs[s])
        graphs[s % nc].replay()
    ev1.record()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    moe.moe_check_device_errors()
    ms = max_over_ranks(ev0.elapsed_time(ev1), world, device)
    tokens = T * K * world
    value = tokens / (ms / 1e3)

    e2e_rec = None
    if e2e:
        host_in = inputs[W:W + K].cpu().pin_memory()
        host_out = torch.empty((K, T, Hh), dtype=torch.bfloat16).pin_memory()
        barrier(world)
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        for s in range(K):
            layer.x.copy_(host_in[s], non_blocking=True)
            graphs[s % nc].replay()
            host_out[s].copy_(layer.out, non_blocking=True)
        t1.record()
        torch.cuda.synchronize()
        barrier(world)
        e2e_ms = max_over_ranks(t0.elapsed_time(t1), world, device)
        e2e_rec = {"value": round(tokens / (e2e_ms / 1e3), 1), "unit": "tokens/s", "h2d_bytes_per_step": T * Hh * 2,
                   "d2h_bytes_per_step": T * Hh * 2}

    # roofline of the dominant op: one moe_grouped_ffn call (the row gather + two tcgen05
    # GEMMs, or the two GEMV launches), CUDA events recorded on its stream inside a graph
    layer.ffn_events = (torch.cuda.Event(enable_timing=True, external=True),
                        torch.cuda.Event(enable_timing=True, external=True))
    g2s = [torch.cuda.CUDAGraph() for _ in range(nc)]
    with torch.cuda.stream(cap):
        for c_, g2 in enumerate(g2s):
            with torch.cuda.graph(g2, stream=cap):
                layer.step(c_, log_active=True)
    torch.cuda.current_stream().wait_stream(cap)
    ffn_ms, ffn_bytes = [], []
    bitplane = layer.bits is not None
    gemm = gemm_path(cfg)
    act_bytes = T * Hh * 2 + T * k * Ii * 2 * 2 + T * k * Hh * 2  # x, h (written and read), y_rows
    n_meas = min(K, 10 if gemm else 64)
    for s in range(W, W + n_meas):
        layer.x.copy_(inputs[s])
        g2s[s % nc].replay()
        torch.cuda.synchronize()
        ffn_ms.append(layer.ffn_events[0].elapsed_time(layer.ffn_events[1]))
        if bitplane:
            # the weight stream of this step: each routed expert's prefix of b_max planes (the
            # widest of its pairs), once, with its scales
            offs = layer.routing.expert_offsets.cpu().tolist()
            sp = layer.routing.sorted_pair.cpu().tolist()
            bits = layer.bits.cpu().tolist()
            nbytes = 0
            for e in range(Ee):
                if offs[e + 1] > offs[e]:
                    bmax = max(bits[sp[r]] for r in range(offs[e], offs[e + 1]))
                    nbytes += bmax * BP_PLANE_BYTES + BP_SCALE_BYTES
            ffn_bytes.append(nbytes + act_bytes)
        else:
            ffn_bytes.append(int(layer.n_active.item()) * expert_bytes(cfg) + act_bytes)
    layer.ffn_events = None
    hbm, bf16_peak, peak_kind = measured_peaks()
    avg_s = statistics.mean(ffn_ms) / 1e3
    if gemm and cfg.get("act"):
        # W4A4 on the FP4 tensor cores: 2 P 3 H I flops against 4x the bf16 peak (the nominal
        # fp4 : bf16 ratio) take less time than its bytes at the HBM peak, so HBM bounds it.
        # Algorithmic bytes: the routed experts' codes and scales, x (bf16), y_rows (bf16),
        # and h as NVFP4 written and read.
        flops = 2.0 * T * k * 3 * Hh * Ii
        nbytes = (statistics.mean(ffn_bytes) - act_bytes + T * Hh * 2 + T * k * Hh * 2
                  + 2 * T * k * Ii * 9 / 16)
        achieved = nbytes / avg_s / 1e9
        fp4_peak = 4.0 * bf16_peak
        roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                    "frac": round(achieved / hbm, 4), "peak_kind": peak_kind + " HBM copy", "traffic": None,
                    "kernel": ("k_ffn_fp4 gate/up + down (block-scaled tcgen05 FP4 MMA) with the activation "
                               "quantisers (one moe_grouped_ffn_w4a4 call)"),
                    "algorithmic_bytes_per_call": round(nbytes), "avg_call_us": round(avg_s * 1e6, 1),
                    "tensor": {"achieved": round(flops / avg_s / 1e12, 1), "peak": round(fp4_peak, 1),
                               "unit": "TFLOP/s", "frac": round(flops / avg_s / 1e12 / fp4_peak, 4),
                               "peak_kind": peak_kind + " bf16 burst x 4 (nominal fp4 : bf16 dense ratio)"}}
    elif gemm:
        flops = 2.0 * T * k * 3 * Hh * Ii
        achieved = flops / avg_s / 1e12
        roofline = {"bound": "tensor", "achieved": round(achieved, 1), "peak": bf16_peak, "unit": "TFLOP/s",
                    "frac": round(achieved / bf16_peak, 4),
                    "peak_kind": peak_kind + " bf16 burst (the fp16 MMAs of this path have the same dense peak)",
                    "traffic": None,
                    "kernel": "k_ffn_umma gate/up + down with the row gather and the GEMV pass over small experts "
                              "(one moe_grouped_ffn call)",
                    "algorithmic_flops_per_call": flops, "avg_call_us": round(avg_s * 1e6, 1)}
    else:
        achieved = sum(ffn_bytes) / (sum(ffn_ms) / 1e3) / 1e9
        traffic = None
        if allocation is not None:
            tr = committed_traffic("traffic_bitplane.json")
            traffic = tr["dram_bytes_per_call"] if tr else None  # all 64 experts at 3 planes, as allocated
        fmt_name = {"nvfp4": "NVFP4", "bitplane": "bitplane"}.get(cfg.get("fmt"), "W4")
        roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                    "frac": round(achieved / hbm, 4), "peak_kind": peak_kind + " HBM copy", "traffic": traffic,
                    "kernel": f"k_ffn_gemv<{fmt_name}> gate/up + down (one moe_grouped_ffn call)",
                    "algorithmic_bytes_per_call": round(statistics.mean(ffn_bytes)),
                    "avg_call_us": round(avg_s * 1e6, 1)}
    fmt = cfg.get("fmt")
    if bitplane:
        l2 = ("no flush: each step reads about %.0f MB of expert planes and scales, and steps rotate over %d "
              "device copies of the weights (> 4 x 126 MB L2 between reuses)" % (statistics.mean(ffn_bytes) / 1e6, nc))
    elif nc > 1:
        l2 = ("no flush: steps rotate over %d device copies of the %.0f MB of expert weights (> 4 x 126 MB L2 "
              "between reuses)" % (nc, Ee * expert_bytes(cfg) / 1e6))
    else:
        l2 = "no flush: the %.1f GB of expert weights exceed 4 x the 126 MB L2" % (Ee * expert_bytes(cfg) / 1e9)
    rec = {"value": round(value, 1), "unit": "tokens/s", "steps": K, "warmup": W, "ms_per_step": round(ms / K, 4),
           "dtype": ("e2m1" if cfg.get("act") else "fp16") if fmt == "nvfp4" and gemm else "bf16",
           "data": "synthetic (seeded Irwin-Hall N(0,1) activations, N(0,0.02) bf16 weights quantised to "
                   + {"nvfp4": "NVFP4", "bitplane": "8 bitplanes"}.get(fmt, "W4A16 g128") + ")",
           "config": {"workload": cfg["desc"], "tokens": T, "hidden": Hh, "intermediate": Ii, "experts": Ee,
                      "top_k": k, "path": "tcgen05 grouped GEMM" if gemm else "grouped GEMV",
                      "parallelism": f"dp{world} (independent replicas)", "l2": l2},
           "gpu_launches": layer.kernels_per_step * K, "clocks": clk, "roofline": roofline, "e2e": e2e_rec}
    if allocation is not None:
        rec["config"]["allocation"] = allocation
    del graphs, g2s, layer, inputs
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return rec


def oracle_prefill_sample(cfg, tokens: int, seed: int):
    """Times the CPU oracle on `tokens` tokens of one prefill layer (routing, the routed
    experts' dequantisation and SwiGLU, combine); the experts' weights are generated and
    quantised untimed.  Returns (tokens/s, seconds timed, threads)."""
    import numpy as np

    import synth
    from oracle.alloc import expand_bits
    from oracle.ffn import FMT_BITPLANE8, FMT_NVFP4, FMT_W4G128, Experts, combine, grouped_ffn, moe_layer, route
    from oracle.quant import pack_bitplanes, quantize_nvfp4, quantize_w4g128
    from oracle.routing import router_logits, topk_softmax
    T, Hh, Ii, Ee, k = cfg["T"], cfg["H"], cfg["I"], cfg["E"], cfg["k"]
    nvfp4 = cfg.get("fmt") == "nvfp4"
    bitplane = cfg.get("fmt") == "bitplane"
    x = synth.normal_bf16(seed + synth.SEED_X, tokens * Hh, 1.0).reshape(tokens, Hh)
    if cfg["router"] == "uniform":
        wr = synth.uniform_bf16(cfg["seed"] + synth.SEED_WR, Ee * Hh, -0.02, 0.02).reshape(Ee, Hh)
    else:
        wr = synth.normal_bf16(cfg["seed"] + synth.SEED_WR, Ee * Hh, 0.02).reshape(Ee, Hh)
    bias = synth.zipf_rank_bias(cfg["seed"] + synth.SEED_BIAS, Ee) if cfg["zipf"] else None
    ids, _ = topk_softmax(router_logits(x, wr, bias), k)
    if nvfp4:
        w13q, w13s = np.zeros((Ee, 2 * Ii, Hh // 2), np.uint8), np.zeros((Ee, 2 * Ii, Hh // 16), np.uint8)
        w2q, w2s = np.zeros((Ee, Hh, Ii // 2), np.uint8), np.zeros((Ee, Hh, Ii // 16), np.uint8)
        w13g, w2g = np.zeros(Ee, np.float32), np.zeros(Ee, np.float32)
    elif bitplane:
        w13q, w13s = np.zeros((Ee, 8, 2 * Ii, Hh // 32), np.uint32), np.zeros((Ee, 2 * Ii, Hh // 128), np.uint16)
        w2q, w2s = np.zeros((Ee, 8, Hh, Ii // 32), np.uint32), np.zeros((Ee, Hh, Ii // 128), np.uint16)
    else:
        w13q, w13s = np.zeros((Ee, 2 * Ii, Hh // 8), np.uint32), np.zeros((Ee, 2 * Ii, Hh // 128), np.uint16)
        w2q, w2s = np.zeros((Ee, Hh, Ii // 8), np.uint32), np.zeros((Ee, Hh, Ii // 128), np.uint16)
    for e in sorted(set(ids.reshape(-1).tolist())):
        r13 = synth.normal_rows_bf16(cfg["seed"] + synth.SEED_W13, (2 * Ii, Hh), 0.02, e, 1)
        r2 = synth.normal_rows_bf16(cfg["seed"] + synth.SEED_W2, (Hh, Ii), 0.02, e, 1)
        if nvfp4:
            a, b = quantize_nvfp4(r13), quantize_nvfp4(r2)
            w13q[e], w13s[e], w13g[e], w2q[e], w2s[e], w2g[e] = a[0][0], a[1][0], a[2][0], b[0][0], b[1][0], b[2][0]
        elif bitplane:
            a, b = pack_bitplanes(r13), pack_bitplanes(r2)
            w13q[e], w13s[e], w2q[e], w2s[e] = a[0][0], a[1][0], b[0][0], b[1][0]
        else:
            a, b = quantize_w4g128(r13), quantize_w4g128(r2)
            w13q[e], w13s[e], w2q[e], w2s[e] = a[0][0], a[1][0], b[0][0], b[1][0]
    if nvfp4:
        ex = Experts(FMT_NVFP4, w13q, w13s, w2q, w2s, w13g, w2g)
    else:
        ex = Experts(FMT_BITPLANE8 if bitplane else FMT_W4G128, w13q, w13s, w2q, w2s)
    t0 = time.perf_counter()
    if cfg.get("act") == "nvfp4":
        from oracle.w4a4 import w4a4_grouped_ffn
        r = route(x, wr, bias, k, Ee)
        combine(w4a4_grouped_ffn(x, r.offsets, r.sorted_pair, k, ex), r.weights, r.pair_to_row, x)
    elif bitplane and cfg.get("bits") == "allocated":
        # the same per-step path at per-expert widths (every expert at 3 planes, the budget's mean)
        r = route(x, wr, bias, k, Ee)
        y = grouped_ffn(x, r.offsets, r.sorted_pair, k, ex, expand_bits(r.ids, np.full(Ee, 3, np.uint8)))
        combine(y, r.weights, r.pair_to_row, x)
    else:
        moe_layer(x, wr, bias, ex, k, residual_bits=x)
    secs = time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info
        threads = max([d.get("num_threads", 1) for d in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count() or 1
    return tokens / secs, secs, threads


# ---------------------------------------------------------------- the oracle (CPU) arm
def oracle_sample(batch: int, layers_timed: int, seed: int):
    """Times the CPU oracle on a bounded sample of the decode stack: `layers_timed`
    consecutive layers of one step (weights prepared untimed).  Returns
    (tokens/s through the 16-layer stack, seconds timed, threads used)."""
    import numpy as np

    import synth
    from oracle.ffn import FMT_W4G128, Experts, stack_layer_step
    from oracle.quant import quantize_w4g128
    from oracle.routing import router_logits, topk_softmax
    x = synth.normal_bf16(seed + synth.SEED_X, batch * H, 1.0).reshape(batch, H)
    timed = 0.0
    for l in range(layers_timed):
        ls = seed + 0x100 * (l + 1)
        wr = synth.normal_bf16(ls + synth.SEED_WR, E * H, 0.02).reshape(E, H)
        ids, _ = topk_softmax(router_logits(x, wr), K_TOP)
        # quantise only the experts this layer routes to (offline work, untimed)
        w13q = np.zeros((E, 2 * I, H // 8), np.uint32)
        w13s = np.zeros((E, 2 * I, H // 128), np.uint16)
        w2q = np.zeros((E, H, I // 8), np.uint32)
        w2s = np.zeros((E, H, I // 128), np.uint16)
        for e in sorted(set(ids.reshape(-1).tolist())):
            a = quantize_w4g128(synth.normal_rows_bf16(ls + synth.SEED_W13, (2 * I, H), 0.02, e, 1))
            b = quantize_w4g128(synth.normal_rows_bf16(ls + synth.SEED_W2, (H, I), 0.02, e, 1))
            w13q[e], w13s[e], w2q[e], w2s[e] = a[0][0], a[1][0], b[0][0], b[1][0]
        ex = Experts(FMT_W4G128, w13q, w13s, w2q, w2s)
        t0 = time.perf_counter()
        x, _ = stack_layer_step(x, wr, ex, K_TOP)
        timed += time.perf_counter() - t0
    per_step = timed * LAYERS / layers_timed
    try:
        from threadpoolctl import threadpool_info
        threads = max([d.get("num_threads", 1) for d in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count() or 1
    return batch / per_step, timed, threads


def prefill_sample_tokens(cfg) -> int:
    # bounded: a few to about 30 s of oracle work (the NVFP4 oracle decodes element by element)
    if cfg.get("fmt") == "nvfp4":
        return 1
    if cfg.get("fmt") == "bitplane":
        return 16
    return 2 if cfg["H"] > 4096 else min(cfg["T"], 32)


def _threads():
    try:
        from threadpoolctl import threadpool_info
        return max([d.get("num_threads", 1) for d in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count() or 1


def _one_thread(fn):
    """fn() with every BLAS / OpenMP pool limited to one thread."""
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=1):
        return fn()


def cpu_baseline_prefill(cfg, seed: int, one_thread: bool = False):
    n = prefill_sample_tokens(cfg)
    v, secs, thr = oracle_prefill_sample(cfg, n, seed)
    out = {"value": round(v, 3), "unit": "tokens/s", "cores": thr, "host_threads": os.cpu_count(), "kind": "oracle",
           "sample": f"{n} tokens through the layer ({secs:.1f} s of CPU work: routing, dequantisation of "
                     f"their experts" + (" at 3 planes each" if cfg.get("bits") == "allocated" else
                                         " at the thresholds' widths" if cfg.get("fmt") == "bitplane" else "")
                     + ", SwiGLU, combine); weights generated and quantised untimed"}
    if one_thread:
        v1, secs1, _ = _one_thread(lambda: oracle_prefill_sample(cfg, n, seed))
        out["value_1thread"] = round(v1, 3)
    return out


def cpu_baseline(batch: int, seed: int, one_thread: bool = False):
    layers_timed = 2
    v, secs, thr = oracle_sample(batch, layers_timed, seed)
    out = {"value": round(v, 3), "unit": "tokens/s", "cores": thr, "host_threads": os.cpu_count(), "kind": "oracle",
           "sample": f"{layers_timed} of the 16 layers of one decode step at batch {batch} "
                     f"({secs:.1f} s of CPU work), scaled to the full step"}
    if one_thread:
        v1, secs1, _ = _one_thread(lambda: oracle_sample(batch, layers_timed, seed))
        out["value_1thread"] = round(v1, 3)
        out["sample"] += f"; the same sample on one thread took {secs1:.1f} s"
    return out


def cpu_baselines_for(records) -> None:
    """Adds the oracle's CPU baseline to each workload record.  The single-layer workloads
    of one layer shape and format share one oracle measurement (tokens/s per token of that
    layer, the same at every batch size: the oracle evaluates token by token)."""
    shared = {}
    for r in records:
        if "error" in r:
            continue
        name = r["name"]
        if name == "decode-b1":
            r["cpu_baseline"] = cpu_baseline(1, SEED_BASE)
            continue
        cfg = LAYER_WORKLOADS[name]
        key = (cfg["H"], cfg["I"], cfg["E"], cfg.get("fmt"), cfg.get("bits"), cfg.get("act"), cfg["zipf"], cfg["router"])
        if key not in shared:
            shared[key] = cpu_baseline_prefill(cfg, cfg["seed"])
            shared[key]["measured_on"] = name
        r["cpu_baseline"] = dict(shared[key])


def run_reference(args, rank, world):
    """The reference arm: the CPU oracle as it stands, on this workload's config."""
    if rank != 0:
        return None
    if args.workload != "decode":
        cfg = PREFILL[args.workload]
        n = prefill_sample_tokens(cfg)
        v, secs, thr = oracle_prefill_sample(cfg, n, cfg["seed"])
        return {"metric": METRIC, "value": round(v, 3), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": round(cfg["T"] / v * 1e3, 3), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
                "config": {"workload": cfg["desc"], "tokens": cfg["T"]},
                "cpu_baseline": {"value": round(v, 3), "unit": "tokens/s", "cores": thr, "kind": "oracle",
                                 "sample": f"{n} tokens through the layer ({secs:.1f} s), scaled per token"},
                "e2e": {"value": round(v, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
    B = args.batch
    K, W = args.steps, args.warmup
    # each step: a bounded sample (2 layers of the stack), W + K of them kept short
    n = max(1, min(K, 3))
    vals = []
    for s in range(n):
        v, secs, thr = oracle_sample(B, 1, SEED_BASE + s)
        vals.append(v)
    value = statistics.mean(vals)
    return {"metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": round(B / value * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": "decode stack: 16 chained OLMoE-like MoE FFN layers (H2048 I1024 E64 top-8, "
                                   "W4A16 g128 experts, bf16 router), residual add, batch %d tokens/step" % B,
                       "layers": LAYERS, "batch": B},
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": thr, "kind": "oracle",
                             "sample": f"{n} sampled steps, each 1 of the 16 layers of a decode step, "
                                       f"scaled to the full step"},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main(argv=None):
    args = parse_args(argv)
    rank, world, local = dist_env()
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return 0
    if args.workload != "decode":
        res = run_prefill(args, rank, world, local)
        if rank == 0 and res is not None and world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline_prefill(LAYER_WORKLOADS[args.workload],
                                                       LAYER_WORKLOADS[args.workload]["seed"])
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
        return 0
    res = run_gpu(args, rank, world, local)
    if rank == 0 and res is not None:
        if world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(args.batch, SEED_BASE, one_thread=True)
            cpu_baselines_for(res.get("workloads", []))
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
