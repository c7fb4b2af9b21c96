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
                                            ("prefill-h2048-e128", 20), ("prefill-h7168-e256", 20),
                                            ("layer-h7168-e256-t64-nvfp4", 200), ("layer-h2048-e64-t16", 200)])
def test_default_steps_per_workload(workload, steps):
    assert bench.parse_args(["--workload", workload]).steps == steps


def test_every_extra_workload_is_defined():
    # one record per benchmark configuration besides the headline decode stack at batch 8
    for name in bench.EXTRA_WORKLOADS:
        assert name == "decode-b1" or name in bench.LAYER_WORKLOADS
    shapes = {(c["H"], c["I"], c["E"], c.get("fmt", "w4"), c["T"]) for c in bench.LAYER_WORKLOADS.values()}
    for want in [(2048, 1024, 64, "w4", 16), (2048, 768, 128, "w4", 2048), (2048, 1024, 64, "bitplane", 64),
                 (7168, 2048, 256, "w4", 1), (7168, 2048, 256, "w4", 64), (7168, 2048, 256, "w4", 4096),
                 (7168, 2048, 256, "nvfp4", 1), (7168, 2048, 256, "nvfp4", 64), (7168, 2048, 256, "nvfp4", 4096)]:
        assert want in shapes


def test_path_and_bytes_per_workload():
    c = bench.LAYER_WORKLOADS
    assert not bench.gemm_path(c["layer-h7168-e256-t64"]) and bench.gemm_path(c["prefill-h7168-e256"])
    assert bench.gemm_path(c["prefill-h2048-e128"]) and not bench.gemm_path(c["bitplane-h2048-e64"])
    # W4 g128: half a byte per weight + one bf16 scale per 128 weights (the OLMoE-like expert: 3.244 MB)
    assert bench.expert_bytes(c["layer-h2048-e64-t16"]) == bench.W4_EXPERT_BYTES == 3244032
    # NVFP4: half a byte + one E4M3 byte per 16 weights + two fp32 per-tensor scales
    n = 3 * 7168 * 2048
    assert bench.expert_bytes(c["layer-h7168-e256-t1-nvfp4"]) == n // 2 + n // 16 + 8


def test_w4a4_workload():
    # NVFP4 weights and activations at the DeepSeek-like prefill shape: always the GEMM path,
    # one record of its own in the default run
    c = bench.LAYER_WORKLOADS["prefill-h7168-e256-w4a4"]
    assert c.get("act") == "nvfp4" and c.get("fmt") == "nvfp4" and (c["H"], c["I"], c["E"], c["T"]) == (7168, 2048, 256, 4096)
    assert bench.gemm_path(c) and "prefill-h7168-e256-w4a4" in bench.EXTRA_WORKLOADS


def test_profile_commands_run_the_current_bench():
    # every bench.py command line quoted in profiles/ parses with the current flags, so each
    # committed summary can be re-made from committed files
    import glob
    import os
    import re
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    n = 0
    for f in sorted(glob.glob(os.path.join(root, "profiles", "*.md"))):
        text = open(f).read().replace("\\\n", " ")
        assert "--clock-control none" in text, f
        for m in re.finditer(r"python bench\.py([^>&\n`'\";|]*)", text):
            bench.parse_args(m.group(1).split())
            n += 1
    assert n >= 8
