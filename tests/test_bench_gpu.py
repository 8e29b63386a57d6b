"""bench.py end to end on the GPU for every workload: one timed step after three warm-ups, and
the JSON line carries the contract's keys. Guards the benchmark itself (its workloads, e2e leg and
roofline fields) against breaking when the library grows."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
        "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches",
        "clocks"}


RECORD_KEYS = {"value", "unit", "ms_per_step", "scaling", "dtype", "config", "per_rows",
               "roofline", "e2e", "graph", "torch_mm", "gpu_launches", "clocks"}
FP32_LOGITS = {"decode", "spec_verify", "prefill", "decode_f16_bias"}


def check_record(rec: dict, name: str):
    assert rec["value"] > 0 and rec["gpu_launches"] >= 1
    assert {"bound", "achieved", "peak", "unit", "frac", "traffic"} <= set(rec["roofline"])
    assert {"value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"} <= set(rec["e2e"])
    assert {"workload", "parallelism", "calls_per_step", "rows_per_call"} <= set(rec["config"])
    for r in rec["per_rows"].values():
        assert 0 < r["us_min_block"] <= r["us_median_block"]
    if name == "vocab_parallel_logprobs":
        assert "skipped" in rec["graph"]
    else:
        assert rec["graph"]["value"] > 0
    if name in FP32_LOGITS:
        assert rec["torch_mm"]["value"] > 0 and rec["torch_mm"]["ours_speedup"] > 0
    else:
        assert "skipped" in rec["torch_mm"]


@pytest.mark.parametrize("workload", ["decode", "spec_verify", "nvfp4", "decode_f16_bias",
                                      "prefill", "prefill_logprobs", "nvfp4_quantize",
                                      "vocab_parallel_logprobs"])
def test_bench_line(workload):
    """Each workload alone (--only); the default decode run also measures every other workload
    into the line's "workloads" map."""
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--workload", workload,
           "--steps", "1", "--warmup", "3", "--no-cpu-baseline"]
    if workload != "decode":
        cmd.append("--only")
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=900, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert KEYS <= set(line), KEYS - set(line)
    assert line["n_gpus"] == 1
    assert {"graph", "torch_mm", "per_rows"} <= set(line)
    check_record(line, workload)
    if workload == "decode":
        import bench
        assert set(line["workloads"]) == set(bench.SECONDARY)
        for name, rec in line["workloads"].items():
            assert RECORD_KEYS <= set(rec), (name, RECORD_KEYS - set(rec))
            check_record(rec, name)
            assert rec["config"] == bench.config_of(name, 1)
        assert line["workloads"]["prefill"]["roofline"]["bound"] == "tensor"
    else:
        assert "workloads" not in line
