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


@pytest.mark.parametrize("workload", ["decode", "spec_verify", "nvfp4", "decode_f16_bias",
                                      "prefill", "prefill_logprobs", "nvfp4_quantize",
                                      "vocab_parallel_logprobs"])
def test_bench_line(workload):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--workload", workload,
                          "--steps", "1", "--warmup", "3", "--no-cpu-baseline"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert KEYS <= set(line), KEYS - set(line)
    assert line["value"] > 0 and line["n_gpus"] == 1 and line["gpu_launches"] >= 1
    assert {"bound", "achieved", "peak", "unit", "frac", "traffic"} <= set(line["roofline"])
    assert {"value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"} <= set(line["e2e"])
