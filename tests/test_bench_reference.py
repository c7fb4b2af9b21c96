"""bench.py's reference arm (the CPU oracle, no GPU) keeps the JSON line contract: the
keys the driver reads, the reference-arm fields, and consistent values."""
import json

import pytest

import bench

KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
        "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"}


def _check(res, steps, warmup):
    assert KEYS <= set(res)
    json.dumps(res)  # one JSON line
    assert res["impl"] == "reference" and res["metric"] == bench.METRIC
    assert res["unit"] == "tokens/s" and res["higher_is_better"] is True and res["scaling"] == "weak"
    assert res["steps"] == steps and res["warmup"] == warmup and res["n_gpus"] == 1
    assert res["value"] > 0 and res["ms_per_step"] > 0 and res["vs_baseline"] is None
    assert isinstance(res["config"]["workload"], str) and res["config"]["workload"]
    cb = res["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == res["value"] and cb["cores"] >= 1 and cb["sample"]
    e2e = res["e2e"]
    assert e2e["value"] == res["value"] and e2e["unit"] == res["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_decode_batch1():
    args = bench.parse_args(["--impl", "reference", "--batch", "1", "--steps", "1", "--warmup", "0"])
    _check(bench.run_reference(args, 0, 1), 1, 0)


def test_reference_arm_other_ranks_do_no_work():
    args = bench.parse_args(["--impl", "reference", "--steps", "1", "--warmup", "0"])
    assert bench.run_reference(args, 1, 2) is None


@pytest.mark.parametrize("workload,steps", [("decode", 512), ("bitplane-h2048-e64", 512),
                                            ("prefill-h2048-e128", 20), ("prefill-h7168-e256", 20)])
def test_default_steps_per_workload(workload, steps):
    assert bench.parse_args(["--workload", workload]).steps == steps
