"""The library's slot-cache planner (host entry points, no GPU) against the oracle:
every step's service order, slots, fetched plane ranges and rounds, and the slots'
contents after it, on seeded routing sequences; plus argument validation."""
import ctypes

import numpy as np
import pytest

import bit_mixed_precision_router_b200 as moe
from oracle.cache import SlotCache, need_from_routing
from oracle.routing import permute


@pytest.fixture(scope="module")
def lib():
    from bit_mixed_precision_router_b200 import build
    build.build()
    return moe.load()


def _oracle_flat(rounds):
    se = [sv.expert for r in rounds for sv in r]
    ss = [sv.slot for r in rounds for sv in r]
    lo = [sv.lo for r in rounds for sv in r]
    hi = [sv.hi for r in rounds for sv in r]
    rs = [0]
    for r in rounds:
        rs.append(rs[-1] + len(r))
    return se, ss, lo, hi, rs


@pytest.mark.parametrize("E,S,P,density", [(64, 16, 1, 0.15), (64, 64, 8, 0.6), (128, 24, 8, 0.3),
                                           (8, 1, 8, 0.5), (1024, 200, 8, 0.25), (5, 2, 1, 0.9)])
def test_planner_matches_oracle(lib, E, S, P, density):
    rng = np.random.default_rng(E + S + P)
    state = moe.moe_cache_init(E, S, P)
    ref = SlotCache(E=E, S=S, P=P)
    for step in range(120):
        need = (rng.integers(1, P + 1, size=E) * (rng.random(E) < density)).astype(np.uint8)
        got = moe.moe_cache_plan(state, need)
        want = _oracle_flat(ref.plan(need.tolist()))
        for g, w, name in zip(got, want, ("served_expert", "served_slot", "fetch_lo", "fetch_hi", "round_start")):
            assert g.tolist() == list(w), (step, name)
        eo, pl = moe.moe_cache_slots(state, S)
        assert eo.tolist() == ref.expert_of and pl.tolist() == ref.planes


def test_planner_on_routed_decode_steps(lib):
    # demand from real routing (top-8 of 64 experts, 8 tokens) with per-pair widths
    rng = np.random.default_rng(7)
    E, S, k, T = 64, 16, 8, 8
    state = moe.moe_cache_init(E, S, 8)
    ref = SlotCache(E=E, S=S, P=8)
    for step in range(40):
        ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
        offsets, sp, _ = permute(ids, E)
        bits = rng.choice(np.array([2, 3, 4, 8], np.uint8), size=T * k)
        need = np.array(need_from_routing(offsets, sp, bits, planes=8), np.uint8)
        got = moe.moe_cache_plan(state, need)
        want = _oracle_flat(ref.plan(need.tolist()))
        assert [g.tolist() for g in got] == [list(w) for w in want]


def test_cache_validation(lib):
    assert lib.moe_cache_state_bytes(0, 1) == 0
    assert lib.moe_cache_state_bytes(8, 9) == 0
    assert lib.moe_cache_state_bytes(1025, 4) == 0
    assert lib.moe_cache_state_bytes(64, 16) > 0
    buf = np.zeros(64, np.int64)
    assert lib.moe_cache_init(buf.ctypes.data, buf.nbytes, 64, 16, 9) == 1
    assert lib.moe_cache_init(buf.ctypes.data, buf.nbytes, 64, 16, 8) == 3  # too small
    assert lib.moe_cache_init(buf.ctypes.data + 4, buf.nbytes, 4, 2, 8) == 5
    state = moe.moe_cache_init(4, 2, 3)
    with pytest.raises(moe.MoeError):
        moe.moe_cache_plan(state, np.array([4, 0, 0, 0], np.uint8))  # above the planes
    eo, pl = moe.moe_cache_slots(state, 2)
    assert eo.tolist() == [-1, -1] and pl.tolist() == [0, 0]        # untouched by the rejected call
    raw = np.zeros(8, np.int64)  # not an initialised state: the library rejects it
    outs = [np.zeros(4, np.int32), np.zeros(4, np.int32), np.zeros(4, np.uint8), np.zeros(4, np.uint8),
            np.zeros(5, np.int32)]
    nr = ctypes.c_int32(0)
    assert lib.moe_cache_plan(raw.ctypes.data, np.zeros(4, np.uint8).ctypes.data,
                              *[o.ctypes.data for o in outs], ctypes.byref(nr)) == 1
    with pytest.raises(ValueError):  # the binding checks need against the state's expert count
        moe.moe_cache_plan(state, np.zeros(5, np.uint8))
    with pytest.raises(ValueError):
        moe.moe_cache_slots(state, 3)
