"""The C ABI library on a machine without a GPU: it loads, exports every function
that include/*.h declares, and rejects invalid arguments on the host before any
CUDA call (argument validation never touches the device)."""
import ctypes
import os
import re

import pytest

import bit_mixed_precision_router_b200 as moe
from bit_mixed_precision_router_b200 import ExpertsT, RoutingT

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
OK, INVALID, SHAPE, WS, CUDA, MISALIGNED = 0, 1, 2, 3, 4, 5
A = 0x10000  # a fake, 16-byte aligned device address: validation only inspects the number


def declared_functions():
    names = set()
    for h in ("moe.h", "moe_synth.h"):
        text = open(os.path.join(ROOT, "include", h)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text))
    return names


@pytest.fixture(scope="module")
def lib():
    from bit_mixed_precision_router_b200 import build
    build.build()
    return moe.load()


def test_library_exports_every_declared_function(lib):
    names = declared_functions()
    assert len(names) >= 14
    for n in sorted(names):
        assert hasattr(lib, n), n
    assert set(moe.exported_symbols()) == names  # the binding covers the whole ABI
    assert lib.moe_abi_version() == 2
    assert lib.moe_status_string(3) == b"workspace missing or too small"
    assert lib.moe_status_string(99) == b"unknown status"


def test_quantizer_validation(lib):
    assert lib.moe_quantize_w4g128(A, 2, 4, 100, A, A, None) == SHAPE
    assert lib.moe_quantize_w4g128(None, 2, 4, 128, A, A, None) == INVALID
    assert lib.moe_quantize_w4g128(A, 0, 4, 128, A, A, None) == INVALID
    assert lib.moe_quantize_w4g128(A + 2, 2, 4, 128, A, A, None) == MISALIGNED
    assert lib.moe_pack_bitplanes(A, 2, 4, 96, A, A, None) == SHAPE
    assert lib.moe_quantize_nvfp4(A, 2, 4, 48, A, A, A, None) == SHAPE
    assert lib.moe_quantize_nvfp4(A, 2, 4, 64, A, A, None, None) == INVALID


def _routing():
    return RoutingT(A, A, A, A, A, A)


def test_route_validation(lib):
    r = _routing()
    call = lambda T, H, E, k, ws=A, wsb=1 << 30, x=A: lib.moe_route_topk(x, A, None, T, H, E, k, ctypes.byref(r),
                                                                         ws, wsb, None)
    assert call(4, 200, 8, 2) == SHAPE        # H % 256
    assert call(4, 256, 0, 1) == SHAPE        # E < 1
    assert call(4, 256, 1025, 2) == SHAPE     # E > MOE_MAX_EXPERTS
    assert call(4, 256, 8, 9) == SHAPE        # k > E
    assert call(4, 256, 64, 33) == SHAPE      # k > MOE_MAX_TOPK
    assert call(-1, 256, 8, 2) == INVALID
    assert call(4, 256, 8, 2, ws=None) == WS
    assert call(4, 256, 8, 2, wsb=16) == WS
    assert call(4, 256, 8, 2, x=None) == INVALID
    assert call(0, 256, 8, 2, ws=None, wsb=0) == OK  # no tokens: nothing to do, nothing launched
    r.sorted_pair = None
    assert call(4, 256, 8, 2) == INVALID
    r.sorted_pair = A + 4
    assert call(4, 256, 8, 2) == MISALIGNED
    assert lib.moe_route_workspace_bytes(16, 64, 8) >= 16 * 64 * 4


def test_ffn_and_combine_validation(lib):
    r = _routing()
    ex = ExpertsT(0, A, A, A, A, None, None)
    call = lambda T, H, I, E, k, bits=None, ws=A, wsb=1 << 40: lib.moe_grouped_ffn(
        A, ctypes.byref(r), ctypes.byref(ex), bits, T, H, I, E, k, A, ws, wsb, None)
    assert call(4, 2048, 1000, 64, 8) == SHAPE   # I % 128
    assert call(4, 2000, 1024, 64, 8) == SHAPE   # H % 256
    assert call(4, 2048, 1024, 64, 8, ws=None) == WS
    assert call(4, 2048, 1024, 64, 8, wsb=1024) == WS
    assert call(0, 2048, 1024, 64, 8, ws=None, wsb=0) == OK
    assert call(4, 131072, 1024, 64, 8) == SHAPE  # larger than the supported hidden size
    ex.fmt = 1
    assert call(4, 2048, 1024, 64, 8) == INVALID  # bitplanes need the bits array
    ex.fmt = 2
    assert call(4, 2048, 1024, 64, 8) == INVALID  # NVFP4 needs the per-expert scales
    ex.fmt = 7
    assert call(4, 2048, 1024, 64, 8) == INVALID
    assert lib.moe_ffn_workspace_bytes(16, 2048, 1024, 64, 8, 0) >= 16 * 8 * 1024 * 2
    # tensor-core path (T*k >= 32*E): h plus the token rows gathered into routed order
    P = 2048 * 8
    for fmt in (0, 2):
        assert lib.moe_ffn_workspace_bytes(2048, 2048, 768, 128, 8, fmt) >= P * 768 * 2 + P * 2048 * 2
    c = lambda T, H, k, res=None: lib.moe_combine(A, ctypes.byref(r), res, T, H, k, A, None)
    assert c(4, 2044, 8) == SHAPE
    assert c(4, 2048, 0) == INVALID
    assert c(4, 2048, 8, res=A + 8) == MISALIGNED
    assert c(0, 2048, 8) == OK


def test_w4a4_validation(lib):
    r = _routing()
    ex = ExpertsT(2, A, A, A, A, A, A)
    H, I, E, k = 2048, 1024, 64, 8
    need = lib.moe_ffn_w4a4_workspace_bytes(4, H, I, E, k)
    tiles = lib.moe_w4a4_scale_tiles_bytes(H, I, E)
    assert tiles == E * 3 * H * I // 16  # one E4M3 scale per 16 weights, re-laid out
    call = lambda T, H, I, E, k, st=A, ws=A, wsb=need: lib.moe_grouped_ffn_w4a4(
        A, ctypes.byref(r), ctypes.byref(ex), st, T, H, I, E, k, A, ws, wsb, None)
    assert call(4, H, 1000, E, k) == SHAPE      # I % 128
    assert call(4, 2176, I, E, k) == SHAPE      # H % 256
    assert call(4, H, I, E, k, st=None) == INVALID  # the prepared weight-scale tiles are required
    assert call(4, H, I, E, k, st=A + 8) == MISALIGNED
    assert call(4, H, I, E, k, ws=None) == WS
    assert call(4, H, I, E, k, wsb=need - 1) == WS
    assert call(0, H, I, E, k, st=None, ws=None, wsb=0) == OK
    ex.fmt = 0
    assert call(4, H, I, E, k) == INVALID       # NVFP4 experts only
    ex.fmt = 2
    ex.w2_gscale = None
    assert call(4, H, I, E, k) == INVALID       # per-expert scales required
    prep = lambda H, I, E, out=A, nb=tiles: lib.moe_w4a4_prepare(ctypes.byref(ex), H, I, E, out, nb, None)
    assert prep(H, I, E) == INVALID
    ex.w2_gscale = A
    assert prep(H, 1000, E) == SHAPE
    assert prep(H, I, E, out=None) == INVALID
    assert prep(H, I, E, nb=tiles - 1) == WS
    assert prep(H, I, 2000) == SHAPE
    # workspace: x and h quantised, routed x codes, h in fp32, tile-ordered activation scales
    P = 4096 * 8
    assert lib.moe_ffn_w4a4_workspace_bytes(4096, 7168, 2048, 256, 8) >= P * 2048 * 4 + P * 7168 // 2


def test_select_bits_validation(lib):
    thr = (ctypes.c_float * 3)(0.05, 0.15, 0.3)
    bad_thr = (ctypes.c_float * 3)(0.3, 0.15, 0.05)
    ch = (ctypes.c_uint8 * 4)(2, 3, 4, 8)
    bad_ch = (ctypes.c_uint8 * 4)(0, 3, 4, 8)
    assert lib.moe_select_bits(A, 4, 8, bad_thr, ch, A, None) == INVALID
    assert lib.moe_select_bits(A, 4, 8, thr, bad_ch, A, None) == INVALID
    assert lib.moe_select_bits(A, 0, 8, thr, ch, A, None) == OK
    assert lib.moe_synth_normal_bf16(None, 4, 0, 1, 1.0, None) == INVALID
    assert lib.moe_synth_normal_bf16(A, 0, 0, 1, 1.0, None) == OK


def test_allocation_validation(lib):
    nan, inf = float("nan"), float("inf")
    d = lambda E, N, K, planes=A, delta=A: lib.moe_bitplane_distortion(planes, A, E, N, K, delta, None)
    assert d(4, 8, 2048, planes=None) == INVALID
    assert d(0, 8, 2048) == INVALID
    assert d(4, 0, 2048) == INVALID
    assert d(4, 8, 2000) == SHAPE
    assert d(4, 8, 2048, planes=A + 4) == MISALIGNED
    assert d(4, 8, 2048, delta=A + 4) == MISALIGNED
    m = lambda T, H, x=A, out=A: lib.moe_activation_moments(x, T, H, out, None)
    assert m(0, 2048) == INVALID
    assert m(4, 0) == INVALID
    assert m(4, 2048, x=None) == INVALID
    assert m(4, 2048, x=A + 1) == MISALIGNED
    assert m(4, 2048, out=A + 4) == MISALIGNED

    def alloc(E, K, choices, budget, offs=A, lam=None):
        ch = (ctypes.c_uint8 * max(len(choices), 1))(*choices)
        return lib.moe_allocate_bits(A, A, offs, E, K, ch, len(choices), budget, A, lam, None)
    assert alloc(64, 2048, (2, 3, 4, 8), nan) == INVALID
    assert alloc(64, 2048, (2, 3, 4, 8), -0.5) == INVALID
    assert alloc(64, 2048, (2, 3, 4, 8), inf) == INVALID
    assert alloc(64, 2048, (), 4.0) == INVALID
    assert alloc(64, 2048, (1, 2, 3, 4, 5, 6, 7, 8, 8), 4.0) == INVALID
    assert alloc(64, 2048, (2, 3, 3), 4.0) == INVALID
    assert alloc(64, 2048, (0, 3), 4.0) == INVALID
    assert alloc(64, 2048, (2, 9), 4.0) == INVALID
    assert alloc(0, 2048, (2, 8), 4.0) == SHAPE
    assert alloc(1025, 2048, (2, 8), 4.0) == SHAPE
    assert alloc(64, 0, (2, 8), 4.0) == SHAPE
    assert alloc(64, 2048, (2, 8), 4.0, offs=A + 2) == MISALIGNED
    assert alloc(64, 2048, (2, 8), 4.0, lam=A + 4) == MISALIGNED
    assert lib.moe_allocate_bits(None, A, A, 64, 2048, (ctypes.c_uint8 * 2)(2, 8), 2, 4.0, A, None, None) == INVALID
    e = lambda T, k, ids=A: lib.moe_expand_bits(ids, A, T, k, A, None)
    assert e(-1, 8) == INVALID
    assert e(4, 0, ) == INVALID
    assert e(4, 33) == INVALID
    assert e(4, 8, ids=None) == INVALID
    assert e(4, 8, ids=A + 2) == MISALIGNED
    assert e(0, 8, ids=None) == OK


def test_device_cache_validation(lib):
    plan = moe.CachePlanT(A, A, A, A, A, A)
    r = RoutingT(A, A, A, A, A, A)

    def step(E, S, T, k, state=A):
        return lib.moe_cache_step(state, E, S, ctypes.byref(r), None, T, k, A, ctypes.byref(plan), None)
    assert step(64, 16, 2, 8, state=None) == INVALID
    assert step(64, 0, 2, 8) == INVALID
    assert step(64, 65, 2, 8) == INVALID
    assert step(64, 16, 4, 8) == SHAPE        # 32 pairs may route to 32 experts: more than 16 slots
    assert step(64, 16, 2, 8, state=A + 4) == MISALIGNED
    assert step(64, 16, 0, 8) == OK
    ex = ExpertsT(0, A, A, A, A, None, None)

    def fetch(E, H, I, e1=ex, e2=ex):
        return lib.moe_cache_fetch(ctypes.byref(plan), E, ctypes.byref(e1), ctypes.byref(e2), H, I, None)
    assert fetch(64, 2048, 1000) == SHAPE
    assert fetch(64, 2000, 1024) == SHAPE
    assert fetch(64, 2048, 1024, e2=ExpertsT(1, A, A, A, A, None, None)) == INVALID   # formats differ
    nv = ExpertsT(2, A, A, A, A, None, None)
    assert fetch(64, 2048, 1024, e1=nv, e2=nv) == INVALID                            # NVFP4 needs its scales
    assert fetch(64, 2048, 1024, e1=ExpertsT(0, A + 8, A, A, A, None, None)) == MISALIGNED

    def perm(T, k, E, ids=A):
        return lib.moe_permute(ids, T, k, E, ctypes.byref(r), None)
    assert perm(4, 0, 8) == SHAPE
    assert perm(4, 2, 8, ids=None) == INVALID
    assert perm(4, 2, 8, ids=A + 4) == MISALIGNED
    assert perm(0, 2, 8) == OK


def test_remaining_entry_points_validation(lib):
    # activation quantiser (fp32 rows, NVFP4 codes): 16-wide blocks, every pointer required
    q = lambda R, C, a=A, sc=A: lib.moe_quantize_nvfp4_f32(a, R, C, A, sc, A, None)
    assert q(4, 40) == SHAPE
    assert q(0, 64) == INVALID
    assert q(4, 64, a=None) == INVALID
    assert q(4, 64, sc=None) == INVALID
    assert q(4, 64, a=A + 4) == MISALIGNED
    # the no-alloc router: shape limits of its fixed array, then pointers
    r = _routing()
    na = lambda T, H, E, k, x=A: lib.moe_route_topk_noalloc(x, A, None, T, H, E, k, ctypes.byref(r), None)
    assert na(-1, 256, 8, 2) == INVALID
    assert na(4, 200, 8, 2) == SHAPE
    assert na(4, 256, 8, 9) == SHAPE
    assert na(65536 // 64 + 1, 256, 64, 8) == SHAPE   # T * E above MOE_NOALLOC_MAX_LOGITS
    assert na(0, 256, 8, 2, x=None) == OK             # no tokens: nothing to do, nothing looked up
    assert na(4, 256, 8, 2, x=None) == INVALID
    r.expert_list = None
    assert na(4, 256, 8, 2) == INVALID
    r.expert_list = A + 8
    assert na(4, 256, 8, 2) == MISALIGNED
    r.expert_list = A
    assert na(4, 256, 8, 2, x=A + 2) == MISALIGNED
    # expert parallelism: row gather and local ids from the exchanged counts
    g = lambda n, div, H, src=A, idx=A: lib.moe_gather_rows(src, idx, n, div, H, A, None)
    assert g(-1, 1, 2048) == INVALID
    assert g(4, 0, 2048) == INVALID
    assert g(4, 1, 2044) == SHAPE
    assert g(0, 1, 2048, src=None) == OK
    assert g(4, 1, 2048, idx=None) == INVALID
    assert g(4, 1, 2048, src=A + 8) == MISALIGNED
    assert g(4, 1, 2048, idx=A + 2) == MISALIGNED
    c = lambda S, El, counts=A: lib.moe_ids_from_counts(counts, S, El, A, None)
    assert c(0, 8) == INVALID
    assert c(2, 0) == INVALID
    assert c(2, 8, counts=None) == INVALID
    assert c(1 << 11, 1 << 10) == SHAPE
    assert c(2, 8, counts=A + 2) == MISALIGNED
    # seeded generator
    assert lib.moe_synth_uniform_bf16(None, 4, 0, 1, -1.0, 1.0, None) == INVALID
    assert lib.moe_synth_uniform_bf16(A, 4, -1, 1, -1.0, 1.0, None) == INVALID
    assert lib.moe_synth_uniform_bf16(A, 0, 0, 1, -1.0, 1.0, None) == OK
