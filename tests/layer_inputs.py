"""Seeded inputs of one MoE layer, made once on the host (numpy, module `synth`)
and handed to both sides: the oracle gets the numpy arrays, the CUDA path gets
device copies of the same bytes.  Also the tolerance check shared by the tests."""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

import synth
from oracle.ffn import FMT_BITPLANE8, FMT_NVFP4, FMT_W4G128, Experts
from oracle.quant import pack_bitplanes, quantize_nvfp4, quantize_w4g128

# Output tolerance of the FFN / combine against the float64 oracle.
ATOL = 2e-2
REL_L2 = 1e-2


def dev_bf16(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(torch.bfloat16)


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def as_u32(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().numpy().view(np.uint32)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


@dataclass
class LayerInputs:
    T: int
    H: int
    I: int
    E: int
    k: int
    x: np.ndarray        # bf16 bits [T][H]
    wr: np.ndarray       # bf16 bits [E][H]
    bias: np.ndarray | None
    w13: np.ndarray      # bf16 bits [E][2I][H]
    w2: np.ndarray       # bf16 bits [E][H][I]


def make_layer(seed: int, T: int, H: int, I: int, E: int, k: int, router: str = "normal",
               zipf: bool = False, wstd: float = 0.02, with_experts: bool = True) -> LayerInputs:
    x = synth.normal_bf16(seed + synth.SEED_X, T * H, 1.0).reshape(T, H)
    if router == "uniform":
        wr = synth.uniform_bf16(seed + synth.SEED_WR, E * H, -0.02, 0.02).reshape(E, H)
    else:
        wr = synth.normal_bf16(seed + synth.SEED_WR, E * H, 0.02).reshape(E, H)
    bias = synth.zipf_rank_bias(seed + synth.SEED_BIAS, E) if zipf else None
    w13 = w2 = None
    if with_experts:
        w13 = synth.normal_bf16(seed + synth.SEED_W13, E * 2 * I * H, wstd).reshape(E, 2 * I, H)
        w2 = synth.normal_bf16(seed + synth.SEED_W2, E * H * I, wstd).reshape(E, H, I)
    return LayerInputs(T, H, I, E, k, x, wr, bias, w13, w2)


def oracle_experts(fmt: int, w13: np.ndarray, w2: np.ndarray) -> Experts:
    if fmt == FMT_W4G128:
        a, b = quantize_w4g128(w13), quantize_w4g128(w2)
        return Experts(fmt, a[0], a[1], b[0], b[1])
    if fmt == FMT_BITPLANE8:
        a, b = pack_bitplanes(w13), pack_bitplanes(w2)
        return Experts(fmt, a[0], a[1], b[0], b[1])
    a, b = quantize_nvfp4(w13), quantize_nvfp4(w2)
    return Experts(fmt, a[0], a[1], b[0], b[1], a[2], b[2])


def bf16_half_ulp(v: np.ndarray) -> np.ndarray:
    """Half the spacing of bf16 values (8 significant bits) at |v|: the rounding error of
    storing v in bf16 (0 below the normal range, which these outputs never reach)."""
    a = np.abs(np.asarray(v, dtype=np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.exp2(e - 8), 0.0)


def check_close(got: np.ndarray, ref: np.ndarray, what: str, atol=ATOL, rel_l2=REL_L2, stored_bf16=True):
    """The FFN tolerance against the float64 oracle: max |err| <= atol and relative L2 <= rel_l2.
    Outputs the API stores in bf16 (y_rows, the layer output) cannot be closer to the exact
    value than bf16's own rounding, so their bound per element is atol plus bf16's half
    spacing at the reference value (up to 2^-9 relative: 0.0039 at |ref| = 1, 0.031 from 8)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    bound = atol + (bf16_half_ulp(ref) if stored_bf16 else 0.0)
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    worst = int(np.argmax(err - bound))
    assert np.all(err <= bound), (f"{what}: abs err {err.flat[worst]:.3e} > {np.broadcast_to(bound, err.shape).flat[worst]:.3e} "
                                  f"at |ref| = {abs(ref.flat[worst]):.3e}")
    assert rel <= rel_l2, f"{what}: rel L2 err {rel:.3e} > {rel_l2}"
    return float(err.max()), float(rel)


def sentinel_routing(moe, T: int, E: int, k: int):
    """Routing buffers pre-filled with values no call writes (-7, NaN), so that an output
    a kernel failed to write fails the comparison."""
    r = moe.Routing.empty(T, E, k)
    for t in (r.topk_ids, r.expert_offsets, r.sorted_pair, r.pair_to_row, r.expert_list):
        t.fill_(-7)
    r.topk_w.fill_(float("nan"))
    return r


def oracle_routing(L: LayerInputs, k: int):
    """(ids, w, offsets, sorted_pair, pair_to_row) of the oracle for a layer's inputs."""
    from oracle.routing import permute, router_logits, topk_softmax
    ids, w = topk_softmax(router_logits(L.x, L.wr, L.bias), k)
    offsets, sp, p2r = permute(ids, L.E)
    return ids, w, offsets, sp, p2r


def assert_routing_equals_oracle(r, L: LayerInputs, k: int, what: str = ""):
    """Ids, offsets, sorted_pair, pair_to_row and the active-expert list bit-exact;
    weights within 1e-6 (CPU exp against the GPU's expf)."""
    T, E = L.T, L.E
    ids, w, offsets, sp, p2r = oracle_routing(L, k)
    P = T * k
    assert np.array_equal(r.topk_ids.cpu().numpy()[:P].reshape(T, k), ids), f"{what}: topk_ids"
    got_w = r.topk_w.cpu().numpy()[:P].reshape(T, k)
    assert np.all(np.isfinite(got_w)) and np.abs(got_w - w).max() <= 1e-6, f"{what}: topk_w"
    assert np.array_equal(r.expert_offsets.cpu().numpy()[:E + 1], offsets), f"{what}: expert_offsets"
    assert np.array_equal(r.sorted_pair.cpu().numpy()[:P], sp), f"{what}: sorted_pair"
    assert np.array_equal(r.pair_to_row.cpu().numpy()[:P], p2r), f"{what}: pair_to_row"
    el = r.expert_list.cpu().numpy()
    act = np.nonzero(np.diff(offsets) > 0)[0]
    assert el[0] == act.size and np.array_equal(el[1:1 + act.size], act), f"{what}: expert_list"
