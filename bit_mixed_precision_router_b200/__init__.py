"""Python binding of libmoe.so, the C ABI of the low-bit routed-expert MoE FFN
layer (include/moe.h, include/moe_synth.h).

Argument marshalling only: each function takes torch CUDA tensors, passes their
device pointers and the current CUDA stream to the C entry point of the same
name, and raises MoeError on a non-zero status.  Every computation runs in the
library's CUDA kernels; there is no CPU or PyTorch fallback, and importing the
binding without the built library raises at ``load()``.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

FMT_W4G128, FMT_BITPLANE8, FMT_NVFP4 = 0, 1, 2
MAX_EXPERTS, MAX_TOPK = 1024, 32

STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED_SHAPE", 3: "MOE_ERR_WORKSPACE",
          4: "MOE_ERR_CUDA", 5: "MOE_ERR_MISALIGNED", 6: "MOE_ERR_DEVICE_TIMEOUT"}


class MoeError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {STATUS.get(status, status)}")
        self.status = status


class RoutingT(ctypes.Structure):
    _fields_ = [("topk_ids", ctypes.c_void_p), ("topk_w", ctypes.c_void_p), ("expert_offsets", ctypes.c_void_p),
                ("sorted_pair", ctypes.c_void_p), ("pair_to_row", ctypes.c_void_p),
                ("expert_list", ctypes.c_void_p)]


class ExpertsT(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int), ("w13", ctypes.c_void_p), ("w13_scale", ctypes.c_void_p),
                ("w2", ctypes.c_void_p), ("w2_scale", ctypes.c_void_p), ("w13_gscale", ctypes.c_void_p),
                ("w2_gscale", ctypes.c_void_p)]


class CachePlanT(ctypes.Structure):
    _fields_ = [("served_expert", ctypes.c_void_p), ("served_slot", ctypes.c_void_p), ("fetch_lo", ctypes.c_void_p),
                ("fetch_hi", ctypes.c_void_p), ("nserved", ctypes.c_void_p), ("overflow", ctypes.c_void_p)]


_lib = None
_vp, _i64, _sz, _u64, _d = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_uint64, ctypes.c_double

_SIGS = {
    "moe_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "moe_abi_version": ([], ctypes.c_int),
    "moe_quantize_w4g128": ([_vp, _i64, _i64, _i64, _vp, _vp, _vp], ctypes.c_int),
    "moe_pack_bitplanes": ([_vp, _i64, _i64, _i64, _vp, _vp, _vp], ctypes.c_int),
    "moe_quantize_nvfp4": ([_vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp], ctypes.c_int),
    "moe_quantize_nvfp4_f32": ([_vp, _i64, _i64, _vp, _vp, _vp, _vp], ctypes.c_int),
    "moe_route_workspace_bytes": ([_i64, _i64, _i64], _sz),
    "moe_route_topk": ([_vp, _vp, _vp, _i64, _i64, _i64, _i64, ctypes.POINTER(RoutingT), _vp, _sz, _vp],
                       ctypes.c_int),
    "moe_route_topk_noalloc": ([_vp, _vp, _vp, _i64, _i64, _i64, _i64, ctypes.POINTER(RoutingT), _vp],
                               ctypes.c_int),
    "moe_select_bits": ([_vp, _i64, _i64, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_uint8), _vp,
                         _vp], ctypes.c_int),
    "moe_bitplane_distortion": ([_vp, _vp, _i64, _i64, _i64, _vp, _vp], ctypes.c_int),
    "moe_activation_moments": ([_vp, _i64, _i64, _vp, _vp], ctypes.c_int),
    "moe_allocate_bits": ([_vp, _vp, _vp, _i64, _i64, ctypes.POINTER(ctypes.c_uint8), _i64, _d, _vp, _vp, _vp],
                          ctypes.c_int),
    "moe_expand_bits": ([_vp, _vp, _i64, _i64, _vp, _vp], ctypes.c_int),
    "moe_cache_state_bytes": ([_i64, _i64], _sz),
    "moe_cache_init": ([_vp, _sz, _i64, _i64, _i64], ctypes.c_int),
    "moe_cache_plan": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(ctypes.c_int32)], ctypes.c_int),
    "moe_cache_slots": ([_vp, _vp, _vp], ctypes.c_int),
    "moe_cache_step": ([_vp, _i64, _i64, ctypes.POINTER(RoutingT), _vp, _i64, _i64, _vp, ctypes.POINTER(CachePlanT),
                        _vp], ctypes.c_int),
    "moe_cache_fetch": ([ctypes.POINTER(CachePlanT), _i64, ctypes.POINTER(ExpertsT), ctypes.POINTER(ExpertsT), _i64,
                         _i64, _vp], ctypes.c_int),
    "moe_permute": ([_vp, _i64, _i64, _i64, ctypes.POINTER(RoutingT), _vp], ctypes.c_int),
    "moe_ffn_workspace_bytes": ([_i64, _i64, _i64, _i64, _i64, ctypes.c_int], _sz),
    "moe_grouped_ffn": ([_vp, ctypes.POINTER(RoutingT), ctypes.POINTER(ExpertsT), _vp, _i64, _i64, _i64, _i64,
                         _i64, _vp, _vp, _sz, _vp], ctypes.c_int),
    "moe_w4a4_scale_tiles_bytes": ([_i64, _i64, _i64], _sz),
    "moe_w4a4_prepare": ([ctypes.POINTER(ExpertsT), _i64, _i64, _i64, _vp, _sz, _vp], ctypes.c_int),
    "moe_ffn_w4a4_workspace_bytes": ([_i64, _i64, _i64, _i64, _i64], _sz),
    "moe_grouped_ffn_w4a4": ([_vp, ctypes.POINTER(RoutingT), ctypes.POINTER(ExpertsT), _vp, _i64, _i64, _i64, _i64,
                              _i64, _vp, _vp, _sz, _vp], ctypes.c_int),
    "moe_combine": ([_vp, ctypes.POINTER(RoutingT), _vp, _i64, _i64, _i64, _vp, _vp], ctypes.c_int),
    "moe_gather_rows": ([_vp, _vp, _i64, _i64, _i64, _vp, _vp], ctypes.c_int),
    "moe_ids_from_counts": ([_vp, _i64, _i64, _vp, _vp], ctypes.c_int),
    "moe_check_device_errors": ([_vp], ctypes.c_int),
    "moe_synth_normal_bf16": ([_vp, _i64, _i64, _u64, _d, _vp], ctypes.c_int),
    "moe_synth_uniform_bf16": ([_vp, _i64, _i64, _u64, _d, _d, _vp], ctypes.c_int),
}


def load(path: str = LIB_PATH):
    """Load libmoe.so (built by ``python -m bit_mixed_precision_router_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m bit_mixed_precision_router_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (args, res) in _SIGS.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def exported_symbols() -> list[str]:
    return list(_SIGS)


def _call(name: str, *args) -> None:
    st = getattr(load(), name)(*args)
    if st != 0:
        raise MoeError(name, st)


def _stream(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _p(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _check(t: torch.Tensor | None, what: str, dtype=None, numel: int | None = None) -> None:
    """Caller-provided buffers: the C entry points take plain pointers and cannot check
    sizes, so the binding checks element type and element count before passing them."""
    if t is None:
        return
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise TypeError(f"{what}: expected {dtype}, got {t.dtype}")
    if numel is not None and t.numel() < numel:
        raise ValueError(f"{what}: needs at least {numel} elements, has {t.numel()}")


_BF16 = (torch.bfloat16, torch.int16, torch.uint16)


def _bits(t: torch.Tensor) -> torch.Tensor:
    """bf16 tensors travel as their 16-bit patterns."""
    if t.dtype == torch.bfloat16:
        return t
    if t.dtype in (torch.int16, torch.uint16):
        return t
    raise TypeError(f"expected bf16 data, got {t.dtype}")


# ---------------------------------------------------------------- offline quantisers
def moe_quantize_w4g128(w: torch.Tensor, packed: torch.Tensor | None = None, scales: torch.Tensor | None = None,
                        stream=None):
    """bf16 [E][N][K] -> (packed int32 [E][N][K/8] holding uint32 words, scales bf16 [E][N][K/128])."""
    E, N, K = w.shape
    packed = torch.empty((E, N, K // 8), dtype=torch.int32, device=w.device) if packed is None else packed
    scales = torch.empty((E, N, K // 128), dtype=torch.bfloat16, device=w.device) if scales is None else scales
    _check(packed, "packed", (torch.int32, torch.uint32), E * N * (K // 8))
    _check(scales, "scales", _BF16, E * N * (K // 128))
    _call("moe_quantize_w4g128", _p(_bits(w)), E, N, K, _p(packed), _p(scales), _stream(stream))
    return packed, scales


def moe_pack_bitplanes(w: torch.Tensor, planes: torch.Tensor | None = None, scales: torch.Tensor | None = None,
                       stream=None):
    """bf16 [E][N][K] -> (planes int32 [E][8][N][K/32], scales bf16 [E][N][K/128])."""
    E, N, K = w.shape
    planes = torch.empty((E, 8, N, K // 32), dtype=torch.int32, device=w.device) if planes is None else planes
    scales = torch.empty((E, N, K // 128), dtype=torch.bfloat16, device=w.device) if scales is None else scales
    _check(planes, "planes", (torch.int32, torch.uint32), E * 8 * N * (K // 32))
    _check(scales, "scales", _BF16, E * N * (K // 128))
    _call("moe_pack_bitplanes", _p(_bits(w)), E, N, K, _p(planes), _p(scales), _stream(stream))
    return planes, scales


def moe_quantize_nvfp4(w: torch.Tensor, codes=None, block_scales=None, gscale=None, stream=None):
    """bf16 [E][N][K] -> (codes uint8 [E][N][K/2], block_scales uint8 [E][N][K/16], gscale fp32 [E])."""
    E, N, K = w.shape
    codes = torch.empty((E, N, K // 2), dtype=torch.uint8, device=w.device) if codes is None else codes
    block_scales = (torch.empty((E, N, K // 16), dtype=torch.uint8, device=w.device)
                    if block_scales is None else block_scales)
    gscale = torch.empty((E,), dtype=torch.float32, device=w.device) if gscale is None else gscale
    _check(codes, "codes", torch.uint8, E * N * (K // 2))
    _check(block_scales, "block_scales", torch.uint8, E * N * (K // 16))
    _check(gscale, "gscale", torch.float32, E)
    _call("moe_quantize_nvfp4", _p(_bits(w)), E, N, K, _p(codes), _p(block_scales), _p(gscale), _stream(stream))
    return codes, block_scales, gscale


def moe_quantize_nvfp4_f32(a: torch.Tensor, codes=None, block_scales=None, gscale=None, stream=None):
    """fp32 [R][C] as one NVFP4 tensor -> (codes uint8 [R][C/2], block_scales uint8 [R][C/16], gscale fp32 [1])."""
    R, C = a.shape
    codes = torch.empty((R, C // 2), dtype=torch.uint8, device=a.device) if codes is None else codes
    block_scales = (torch.empty((R, C // 16), dtype=torch.uint8, device=a.device)
                    if block_scales is None else block_scales)
    gscale = torch.empty((1,), dtype=torch.float32, device=a.device) if gscale is None else gscale
    _check(a, "a", torch.float32, R * C)
    _check(codes, "codes", torch.uint8, R * C // 2)
    _check(block_scales, "block_scales", torch.uint8, R * C // 16)
    _check(gscale, "gscale", torch.float32, 1)
    _call("moe_quantize_nvfp4_f32", _p(a), R, C, _p(codes), _p(block_scales), _p(gscale), _stream(stream))
    return codes, block_scales, gscale


# ---------------------------------------------------------------- routing
@dataclass
class Routing:
    """Device buffers of one routing (moe_routing_t)."""
    topk_ids: torch.Tensor
    topk_w: torch.Tensor
    expert_offsets: torch.Tensor
    sorted_pair: torch.Tensor
    pair_to_row: torch.Tensor
    expert_list: torch.Tensor

    @staticmethod
    def empty(T: int, E: int, k: int, device="cuda") -> "Routing":
        P = max(T * k, 1)
        i32 = dict(dtype=torch.int32, device=device)
        return Routing(torch.empty(P, **i32), torch.empty(P, dtype=torch.float32, device=device),
                       torch.empty(E + 1, **i32), torch.empty(P, **i32), torch.empty(P, **i32),
                       torch.empty(E + 1, **i32))

    def c(self) -> RoutingT:
        return RoutingT(_p(self.topk_ids), _p(self.topk_w), _p(self.expert_offsets), _p(self.sorted_pair),
                        _p(self.pair_to_row), _p(self.expert_list))

    def check(self, T: int, E: int, k: int) -> "Routing":
        """Raises unless the buffers hold a routing of T tokens, E experts, top-k."""
        P = T * k
        _check(self.topk_ids, "topk_ids", torch.int32, P)
        _check(self.topk_w, "topk_w", torch.float32, P)
        _check(self.expert_offsets, "expert_offsets", torch.int32, E + 1)
        _check(self.sorted_pair, "sorted_pair", torch.int32, P)
        _check(self.pair_to_row, "pair_to_row", torch.int32, P)
        _check(self.expert_list, "expert_list", torch.int32, E + 1)
        return self


def moe_route_workspace_bytes(T: int, E: int, k: int) -> int:
    return int(load().moe_route_workspace_bytes(T, E, k))


def moe_route_workspace(T: int, E: int, k: int, device) -> torch.Tensor:
    """A zero-filled router workspace for up to (T, E, k): it serves any later call with
    T' <= T and E' <= E, in any order (the completion counter sits in its first 256
    bytes whatever the shape, and each call leaves it at zero)."""
    return torch.zeros(max(moe_route_workspace_bytes(T, E, k), 16), dtype=torch.uint8, device=device)


def moe_route_topk(x: torch.Tensor, w_router: torch.Tensor, bias: torch.Tensor | None, k: int,
                   out: Routing | None = None, workspace: torch.Tensor | None = None, stream=None) -> Routing:
    T, H = x.shape
    E = w_router.shape[0]
    out = (Routing.empty(T, E, k, x.device) if out is None else out).check(T, E, k)
    _check(w_router, "w_router", _BF16, E * H)
    _check(bias, "bias", torch.float32, E)
    if workspace is None:
        workspace = moe_route_workspace(T, E, k, x.device)
    rc = out.c()
    _call("moe_route_topk", _p(_bits(x)), _p(_bits(w_router)), _p(bias), T, H, E, k, ctypes.byref(rc),
          _p(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    return out


def moe_route_topk_noalloc(x: torch.Tensor, w_router: torch.Tensor, bias: torch.Tensor | None, k: int,
                           out: Routing | None = None, stream=None) -> Routing:
    """moe_route_topk for callers that cannot provide device workspace: the logits
    scratch is the library's fixed device array (T * E <= 65536); nothing is allocated
    by the library.  Calls that overlap on one GPU race on that array."""
    T, H = x.shape
    E = w_router.shape[0]
    out = (Routing.empty(T, E, k, x.device) if out is None else out).check(T, E, k)
    _check(w_router, "w_router", _BF16, E * H)
    _check(bias, "bias", torch.float32, E)
    rc = out.c()
    _call("moe_route_topk_noalloc", _p(_bits(x)), _p(_bits(w_router)), _p(bias), T, H, E, k, ctypes.byref(rc),
          _stream(stream))
    return out


def moe_select_bits(topk_w: torch.Tensor, k: int, thresholds=(0.05, 0.15, 0.30), choices=(2, 3, 4, 8),
                    bits: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    n = topk_w.numel()
    T = n // k
    bits = torch.empty(max(n, 1), dtype=torch.uint8, device=topk_w.device) if bits is None else bits
    _check(topk_w, "topk_w", torch.float32)
    _check(bits, "bits", torch.uint8, n)
    thr = (ctypes.c_float * 3)(*thresholds)
    ch = (ctypes.c_uint8 * 4)(*choices)
    _call("moe_select_bits", _p(topk_w), T, k, thr, ch, _p(bits), _stream(stream))
    return bits


# ---------------------------------------------------------------- budgeted bit allocation
def moe_bitplane_distortion(planes: torch.Tensor, scales: torch.Tensor, delta: torch.Tensor | None = None,
                            stream=None) -> torch.Tensor:
    """delta fp64 [E][8][K] of a bitplane matrix planes [E][8][N][K/32], scales [E][N][K/128]."""
    E, _, N, K32 = planes.shape
    K = K32 * 32
    delta = torch.empty((E, 8, K), dtype=torch.float64, device=planes.device) if delta is None else delta
    _check(planes, "planes", (torch.int32, torch.uint32))
    _check(scales, "scales", _BF16, E * N * (K // 128))
    _check(delta, "delta", torch.float64, E * 8 * K)
    _call("moe_bitplane_distortion", _p(planes), _p(_bits(scales)), E, N, K, _p(delta), _stream(stream))
    return delta


def moe_activation_moments(x: torch.Tensor, m: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """m fp64 [H]: mean over the T tokens of x [T][H] (bf16) squared."""
    T, H = x.shape
    m = torch.empty(H, dtype=torch.float64, device=x.device) if m is None else m
    _check(m, "m", torch.float64, H)
    _call("moe_activation_moments", _p(_bits(x)), T, H, _p(m), _stream(stream))
    return m


def moe_allocate_bits(delta: torch.Tensor, m: torch.Tensor, expert_offsets: torch.Tensor, budget: float,
                      choices=(2, 3, 4, 8), bits_e: torch.Tensor | None = None, lam: torch.Tensor | None = None,
                      stream=None) -> torch.Tensor:
    """uint8 [E] per-expert widths under a read budget (bits per weight); the final
    multiplier is written to ``lam`` (fp64 scalar tensor) when given."""
    E, _, K = delta.shape
    bits_e = torch.empty(E, dtype=torch.uint8, device=delta.device) if bits_e is None else bits_e
    _check(delta, "delta", torch.float64)
    _check(m, "m", torch.float64, K)
    _check(expert_offsets, "expert_offsets", torch.int32, E + 1)
    _check(bits_e, "bits_e", torch.uint8, E)
    _check(lam, "lam", torch.float64, 1)
    ch = (ctypes.c_uint8 * len(choices))(*choices)
    _call("moe_allocate_bits", _p(delta), _p(m), _p(expert_offsets), E, K, ch, len(choices), float(budget),
          _p(bits_e), _p(lam), _stream(stream))
    return bits_e


def moe_expand_bits(topk_ids: torch.Tensor, bits_e: torch.Tensor, k: int, bits: torch.Tensor | None = None,
                    stream=None) -> torch.Tensor:
    """Per-pair widths bits[p] = bits_e[topk_ids[p]] for moe_grouped_ffn."""
    n = topk_ids.numel()
    bits = torch.empty(max(n, 1), dtype=torch.uint8, device=topk_ids.device) if bits is None else bits
    _check(topk_ids, "topk_ids", torch.int32)
    _check(bits_e, "bits_e", torch.uint8)
    _check(bits, "bits", torch.uint8, n)
    _call("moe_expand_bits", _p(topk_ids), _p(bits_e), n // k, k, _p(bits), _stream(stream))
    return bits


# ---------------------------------------------------------------- expert slot cache (host planning)
def _hp(a) -> int:
    """Address of a C-contiguous host numpy array (the cache entry points take host memory)."""
    import numpy as np
    if not isinstance(a, np.ndarray) or not a.flags["C_CONTIGUOUS"]:
        raise ValueError("expected a C-contiguous numpy array")
    return a.ctypes.data


def moe_cache_state_bytes(E: int, S: int) -> int:
    return int(load().moe_cache_state_bytes(E, S))


def moe_cache_init(E: int, S: int, planes: int):
    """A fresh cache state (host numpy buffer) of S slots over E experts."""
    import numpy as np
    nbytes = moe_cache_state_bytes(E, S)
    if nbytes == 0:
        raise MoeError("moe_cache_state_bytes", 1)
    state = np.zeros((nbytes + 7) // 8, dtype=np.int64)
    _call("moe_cache_init", _hp(state), state.nbytes, E, S, planes)
    return state


def moe_cache_plan(state, need):
    """Plan one step: returns (served_expert, served_slot, fetch_lo, fetch_hi, round_start)
    as numpy arrays, round_start of length R + 1."""
    import numpy as np
    need = np.ascontiguousarray(need, dtype=np.uint8)
    E = need.size
    if state.nbytes < 16 or int(np.asarray(state).view(np.int32)[1]) != E:
        raise ValueError("need: one entry per expert of the cache state")
    se, ss = np.zeros(E, np.int32), np.zeros(E, np.int32)
    lo, hi = np.zeros(E, np.uint8), np.zeros(E, np.uint8)
    rs = np.zeros(E + 1, np.int32)
    nr = ctypes.c_int32(0)
    _call("moe_cache_plan", _hp(state), _hp(need), _hp(se), _hp(ss), _hp(lo), _hp(hi), _hp(rs), ctypes.byref(nr))
    n = int(rs[nr.value])
    return se[:n], ss[:n], lo[:n], hi[:n], rs[:nr.value + 1]


def moe_cache_slots(state, S: int):
    """(expert_of int32 [S], planes uint8 [S]) of a cache state."""
    import numpy as np
    if state.nbytes < 16 or int(np.asarray(state).view(np.int32)[2]) != S:
        raise ValueError("S: the cache state's slot count")
    eo, pl = np.zeros(S, np.int32), np.zeros(S, np.uint8)
    _call("moe_cache_slots", _hp(state), _hp(eo), _hp(pl))
    return eo, pl


# ---------------------------------------------------------------- FFN and combine
@dataclass
class Experts:
    """Device buffers of quantised experts (moe_experts_t)."""
    fmt: int
    w13: torch.Tensor
    w13_scale: torch.Tensor
    w2: torch.Tensor
    w2_scale: torch.Tensor
    w13_gscale: torch.Tensor | None = None
    w2_gscale: torch.Tensor | None = None
    # NVFP4: the weight-scale tiles of the W4A4 path (moe_w4a4_prepare), made on first use
    w4a4_tiles: torch.Tensor | None = field(default=None, repr=False)

    def c(self) -> ExpertsT:
        return ExpertsT(self.fmt, _p(self.w13), _p(self.w13_scale), _p(self.w2), _p(self.w2_scale),
                        _p(self.w13_gscale), _p(self.w2_gscale))

    def check(self, H: int, I: int, E: int) -> "Experts":
        """Raises unless the buffers hold E experts of this format for hidden H and
        intermediate I (sizes as the quantisers write them)."""
        n13, n2 = 2 * I * H, H * I  # weights per matrix of one expert
        if self.fmt == FMT_W4G128:
            sizes = ((self.w13, n13 // 8, (torch.int32, torch.uint32)), (self.w2, n2 // 8, (torch.int32, torch.uint32)),
                     (self.w13_scale, n13 // 128, _BF16), (self.w2_scale, n2 // 128, _BF16))
        elif self.fmt == FMT_BITPLANE8:
            sizes = ((self.w13, n13 // 4, (torch.int32, torch.uint32)), (self.w2, n2 // 4, (torch.int32, torch.uint32)),
                     (self.w13_scale, n13 // 128, _BF16), (self.w2_scale, n2 // 128, _BF16))
        elif self.fmt == FMT_NVFP4:
            sizes = ((self.w13, n13 // 2, torch.uint8), (self.w2, n2 // 2, torch.uint8),
                     (self.w13_scale, n13 // 16, torch.uint8), (self.w2_scale, n2 // 16, torch.uint8),
                     (self.w13_gscale, 1, torch.float32), (self.w2_gscale, 1, torch.float32))
            if self.w13_gscale is None or self.w2_gscale is None:
                raise ValueError("NVFP4 experts need their per-expert scales")
        else:
            raise ValueError(f"unknown format {self.fmt}")
        for i, (t, per_expert, dt) in enumerate(sizes):
            _check(t, f"experts buffer {i}", dt, per_expert * E)
        return self

    def c_host(self) -> ExpertsT:
        """The same struct over page-locked host tensors (a slot cache's expert store)."""
        return ExpertsT(self.fmt, _pinned(self.w13), _pinned(self.w13_scale), _pinned(self.w2),
                        _pinned(self.w2_scale), _pinned(self.w13_gscale), _pinned(self.w2_gscale))


def _pinned(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    if t.is_cuda or not t.is_pinned() or not t.is_contiguous():
        raise ValueError("expected a contiguous page-locked host tensor")
    return t.data_ptr()


# ---------------------------------------------------------------- expert slot cache (device)
@dataclass
class CachePlan:
    """Device buffers of one step's cache plan (moe_cache_plan_t)."""
    served_expert: torch.Tensor
    served_slot: torch.Tensor
    fetch_lo: torch.Tensor
    fetch_hi: torch.Tensor
    nserved: torch.Tensor
    overflow: torch.Tensor

    @staticmethod
    def empty(E: int, device="cuda") -> "CachePlan":
        i32, u8 = dict(dtype=torch.int32, device=device), dict(dtype=torch.uint8, device=device)
        return CachePlan(torch.empty(E, **i32), torch.empty(E, **i32), torch.empty(E, **u8), torch.empty(E, **u8),
                         torch.zeros(1, **i32), torch.zeros(1, **i32))

    def c(self) -> CachePlanT:
        return CachePlanT(_p(self.served_expert), _p(self.served_slot), _p(self.fetch_lo), _p(self.fetch_hi),
                          _p(self.nserved), _p(self.overflow))


def moe_cache_state_device(E: int, S: int, planes: int, device="cuda") -> torch.Tensor:
    """A fresh cache state (moe_cache_init on the host) copied to device memory."""
    host = moe_cache_init(E, S, planes)
    return torch.from_numpy(host.view("uint8")).to(device)


def moe_cache_step(state: torch.Tensor, E: int, S: int, routing: Routing, T: int, k: int,
                   bits: torch.Tensor | None = None, slot_ids: torch.Tensor | None = None,
                   plan: CachePlan | None = None, stream=None):
    """One step's plan on the device; returns (slot_ids int32 [T*k], plan)."""
    slot_ids = torch.empty(max(T * k, 1), dtype=torch.int32, device=state.device) if slot_ids is None else slot_ids
    plan = CachePlan.empty(E, state.device) if plan is None else plan
    routing.check(T, E, k)
    _check(bits, "bits", torch.uint8, T * k)
    _check(slot_ids, "slot_ids", torch.int32, T * k)
    for name in ("served_expert", "served_slot", "fetch_lo", "fetch_hi"):
        _check(getattr(plan, name), name, None, E)
    _check(state, "state", torch.uint8, moe_cache_state_bytes(E, S))
    rc, pc = routing.c(), plan.c()
    _call("moe_cache_step", _p(state), E, S, ctypes.byref(rc), _p(bits), T, k, _p(slot_ids), ctypes.byref(pc),
          _stream(stream))
    return slot_ids, plan


def moe_cache_fetch(plan: CachePlan, E: int, host_store: "Experts", slots: "Experts", H: int, I: int, stream=None):
    host_store.check(H, I, E)
    slots.check(H, I, int(slots.w13.shape[0]))
    pc, hc, sc = plan.c(), host_store.c_host(), slots.c()
    _call("moe_cache_fetch", ctypes.byref(pc), E, ctypes.byref(hc), ctypes.byref(sc), H, I, _stream(stream))


def moe_permute(ids: torch.Tensor, T: int, k: int, E: int, out: Routing | None = None, stream=None) -> Routing:
    """The permutation alone; out.topk_ids and out.topk_w are the caller's (not written)."""
    out = (Routing.empty(T, E, k, ids.device) if out is None else out).check(T, E, k)
    _check(ids, "ids", torch.int32, T * k)
    rc = out.c()
    _call("moe_permute", _p(ids), T, k, E, ctypes.byref(rc), _stream(stream))
    return out


def quantize_experts(fmt: int, w13: torch.Tensor, w2: torch.Tensor, stream=None) -> Experts:
    """Quantise bf16 w13 [E][2I][H] and w2 [E][H][I] into one of the three formats."""
    if fmt == FMT_W4G128:
        a, b = moe_quantize_w4g128(w13, stream=stream), moe_quantize_w4g128(w2, stream=stream)
        return Experts(fmt, a[0], a[1], b[0], b[1])
    if fmt == FMT_BITPLANE8:
        a, b = moe_pack_bitplanes(w13, stream=stream), moe_pack_bitplanes(w2, stream=stream)
        return Experts(fmt, a[0], a[1], b[0], b[1])
    if fmt == FMT_NVFP4:
        a, b = moe_quantize_nvfp4(w13, stream=stream), moe_quantize_nvfp4(w2, stream=stream)
        return Experts(fmt, a[0], a[1], b[0], b[1], a[2], b[2])
    raise ValueError(fmt)


def moe_ffn_workspace_bytes(T: int, H: int, I: int, E: int, k: int, fmt: int) -> int:
    return int(load().moe_ffn_workspace_bytes(T, H, I, E, k, fmt))


def moe_grouped_ffn(x: torch.Tensor, routing: Routing, experts: Experts, I: int, E: int, k: int,
                    bits: torch.Tensor | None = None, y_rows: torch.Tensor | None = None,
                    workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    T, H = x.shape
    y_rows = torch.empty((max(T * k, 1), H), dtype=torch.bfloat16, device=x.device) if y_rows is None else y_rows
    routing.check(T, E, k)
    experts.check(H, I, E)
    _check(bits, "bits", torch.uint8, T * k)
    _check(y_rows, "y_rows", _BF16, T * k * H)
    need = moe_ffn_workspace_bytes(T, H, I, E, k, experts.fmt)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=x.device)
    rc, ec = routing.c(), experts.c()
    _call("moe_grouped_ffn", _p(_bits(x)), ctypes.byref(rc), ctypes.byref(ec), _p(bits), T, H, I, E, k,
          _p(y_rows), _p(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    return y_rows


def moe_w4a4_scale_tiles_bytes(H: int, I: int, E: int) -> int:
    return int(load().moe_w4a4_scale_tiles_bytes(H, I, E))


def moe_w4a4_prepare(experts: Experts, H: int, I: int, E: int, out: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
    """The weight scales of NVFP4 experts in the order the FP4 tensor cores read them (once per
    set of experts; again after the weights change)."""
    experts.check(H, I, E)
    need = moe_w4a4_scale_tiles_bytes(H, I, E)
    out = torch.empty(max(need, 16), dtype=torch.uint8, device=experts.w13.device) if out is None else out
    ec = experts.c()
    _call("moe_w4a4_prepare", ctypes.byref(ec), H, I, E, _p(out), out.numel() * out.element_size(), _stream(stream))
    return out


def moe_ffn_w4a4_workspace_bytes(T: int, H: int, I: int, E: int, k: int) -> int:
    return int(load().moe_ffn_w4a4_workspace_bytes(T, H, I, E, k))


def moe_grouped_ffn_w4a4(x: torch.Tensor, routing: Routing, experts: Experts, I: int, E: int, k: int,
                         y_rows: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                         stream=None, scale_tiles: torch.Tensor | None = None) -> torch.Tensor:
    """The grouped FFN with NVFP4 weights and NVFP4 activations quantised on the fly.
    scale_tiles: moe_w4a4_prepare's output for these experts; if None, the experts' own
    (prepared on first use and kept in experts.w4a4_tiles)."""
    T, H = x.shape
    y_rows = torch.empty((max(T * k, 1), H), dtype=torch.bfloat16, device=x.device) if y_rows is None else y_rows
    routing.check(T, E, k)
    experts.check(H, I, E)
    _check(y_rows, "y_rows", _BF16, T * k * H)
    if scale_tiles is None:
        if experts.w4a4_tiles is None:
            experts.w4a4_tiles = moe_w4a4_prepare(experts, H, I, E, stream=stream)
        scale_tiles = experts.w4a4_tiles
    _check(scale_tiles, "scale_tiles", torch.uint8, moe_w4a4_scale_tiles_bytes(H, I, E))
    need = moe_ffn_w4a4_workspace_bytes(T, H, I, E, k)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=x.device)
    rc, ec = routing.c(), experts.c()
    _call("moe_grouped_ffn_w4a4", _p(_bits(x)), ctypes.byref(rc), ctypes.byref(ec), _p(scale_tiles), T, H, I, E, k,
          _p(y_rows), _p(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    return y_rows


def moe_combine(y_rows: torch.Tensor, routing: Routing, T: int, k: int, residual: torch.Tensor | None = None,
                out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    H = y_rows.shape[1]
    out = torch.empty((T, H), dtype=torch.bfloat16, device=y_rows.device) if out is None else out
    _check(y_rows, "y_rows", _BF16, T * k * H)
    _check(routing.topk_w, "topk_w", torch.float32, T * k)
    _check(routing.pair_to_row, "pair_to_row", torch.int32, T * k)
    _check(residual, "residual", _BF16, T * H)
    _check(out, "out", _BF16, T * H)
    rc = routing.c()
    _call("moe_combine", _p(y_rows), ctypes.byref(rc), _p(residual), T, H, k, _p(out), _stream(stream))
    return out


def moe_gather_rows(src: torch.Tensor, idx: torch.Tensor, div: int = 1, n: int | None = None,
                    dst: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """dst[i] = src[idx[i] // div] (bf16 rows) for the first n indices."""
    n = idx.numel() if n is None else n
    H = src.shape[1]
    dst = torch.empty((max(n, 1), H), dtype=src.dtype, device=src.device) if dst is None else dst
    _check(src, "src", _BF16)
    _check(idx, "idx", torch.int32, n)
    _check(dst, "dst", _BF16, n * H)
    _call("moe_gather_rows", _p(_bits(src)), _p(idx), n, div, H, _p(_bits(dst)), _stream(stream))
    return dst


def moe_ids_from_counts(counts: torch.Tensor, n: int, ids: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """ids int32 [n] of received rows from counts int32 [S][El] (n = counts.sum())."""
    S, El = counts.shape
    ids = torch.empty(max(n, 1), dtype=torch.int32, device=counts.device) if ids is None else ids
    _check(counts, "counts", torch.int32, S * El)
    _check(ids, "ids", torch.int32, n)
    _call("moe_ids_from_counts", _p(counts), S, El, _p(ids), _stream(stream))
    return ids


def moe_check_device_errors(stream=None) -> None:
    _call("moe_check_device_errors", _stream(stream))


# ---------------------------------------------------------------- synthetic inputs
def moe_synth_normal_bf16(out: torch.Tensor, seed: int, std: float, start: int = 0, stream=None) -> torch.Tensor:
    _call("moe_synth_normal_bf16", _p(out), out.numel(), start, seed & (2 ** 64 - 1), float(std), _stream(stream))
    return out


def moe_synth_uniform_bf16(out: torch.Tensor, seed: int, lo: float, hi: float, start: int = 0,
                           stream=None) -> torch.Tensor:
    _call("moe_synth_uniform_bf16", _p(out), out.numel(), start, seed & (2 ** 64 - 1), float(lo), float(hi),
          _stream(stream))
    return out
