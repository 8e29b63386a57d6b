"""bench.py --traffic-from: ncu launch lists (one CSV per workload) to profiles/traffic.json.

Runs on the CPU on synthetic CSVs shaped like ncu's --csv output (its own messages first, then
one row per launch and metric), written to a temporary directory, and checks the grouping of
launches into calls, the units, the time-only case and the tie to the kernel sources."""
import csv
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
import bench  # noqa: E402

HDR = ["ID", "Process ID", "Process Name", "Host Name", "Kernel Name", "Context", "Stream",
       "Block Size", "Grid Size", "Device", "CC", "Section Name", "Metric Name", "Metric Unit",
       "Metric Value"]


def write_list(path, launches):
    """launches: [(kernel name, {metric: (unit, value)})] in launch order."""
    with open(path, "w", newline="") as f:
        f.write("==PROF== Connected to process 1 (python)\n")
        f.write("==WARNING== Note: Running with unmodified GPU clocks.\n")
        w = csv.writer(f, quoting=csv.QUOTE_ALL)
        w.writerow(HDR)
        for i, (name, metrics) in enumerate(launches):
            for metric, (unit, value) in metrics.items():
                w.writerow([i, 1, "python", "h", name, 1, 7, "(320, 1, 1)", "(148, 1, 1)", 0,
                            "10.0", "Command line profiler metrics", metric, unit, value])


def full(ns, rd, wr, rd_unit="byte", wr_unit="byte", t_unit="nsecond"):
    return {"gpu__time_duration.sum": (t_unit, ns), "dram__bytes_read.sum": (rd_unit, rd),
            "dram__bytes_write.sum": (wr_unit, wr)}


def test_calls_units_and_time_only_lists(tmp_path):
    # decode: 7 calls of one kernel each, units as ncu prints them
    write_list(tmp_path / "decode.csv",
               [("void lmhead_bf16_f32_kernel<4, 0>(...)", full(95000 + i, 622412288, 4100000))
                for i in range(6)]
               + [("void lmhead_bf16_f32_kernel<2, 0>(...)",
                   full("102.5", "645.0", "1,000", rd_unit="Mbyte", wr_unit="Kbyte",
                        t_unit="usecond"))])
    # the quantiser: two kernels per call
    write_list(tmp_path / "nvfp4_quantize.csv",
               [("nvfp4_absmax_kernel", full(92700, 622000000, 3900000)),
                ("nvfp4_encode_kernel", full(155700, 622000000, 117200000))])
    # prefill: the time only
    write_list(tmp_path / "prefill.csv",
               [("void lmhead_bf16_f32_kernel<1, 1>(...)",
                 {"gpu__time_duration.sum": ("msecond", "6.7815")})])
    out = tmp_path / "traffic.json"
    res = bench.write_traffic(str(tmp_path), str(out))
    assert json.loads(out.read_text()) == res
    h = bench.kernel_source_hash()

    dec = res["lmhead_bf16_f32_kernel"]["decode"]
    assert dec["calls"] == 7 and dec["kernels_per_call"] == 1 and dec["source_hash"] == h
    assert dec["per_call_bytes"][:6] == [622412288 + 4100000] * 6
    assert dec["per_call_bytes"][6] == 645_000_000 + 1_000_000
    assert dec["per_call_ns_under_ncu"][6] == pytest.approx(102500.0)
    assert dec["bytes_per_launch"] == int(sum(dec["per_call_bytes"]) / 7)

    q = res["nvfp4_encode_kernel + nvfp4_absmax_kernel"]["nvfp4_quantize"]
    assert q["calls"] == 1 and q["kernels_per_call"] == 2
    assert q["bytes_per_launch"] == 622000000 + 3900000 + 622000000 + 117200000
    assert q["per_call_ns_under_ncu"] == [pytest.approx(92700 + 155700)]

    pf = res["lmhead_bf16_f32_kernel"]["prefill"]
    assert pf["bytes_per_launch"] is None and "note" in pf
    assert pf["per_call_ns_under_ncu"] == [pytest.approx(6.7815e6)]
    assert "nvfp4" not in res.get("lmhead_w4a16_nvfp4_kernel", {})   # no CSV, no entry


def test_recorded_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    """bench reports a recorded figure only while its source hash is the current one."""
    rec = {"lmhead_bf16_f32_kernel": {"decode": {"bytes_per_launch": 123,
                                                 "source_hash": bench.kernel_source_hash()}},
           "lmhead_w4a16_nvfp4_kernel": {"nvfp4": {"bytes_per_launch": 456,
                                                   "source_hash": "0000000000000000"}}}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "_ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: rec["lmhead_bf16_f32_kernel"]
                        ["decode"]["source_hash"])
    assert bench.recorded_traffic("lmhead_bf16_f32_kernel", "decode") == 123
    assert bench.recorded_traffic("lmhead_w4a16_nvfp4_kernel", "nvfp4") is None
    assert bench.recorded_traffic("lmhead_bf16_f32_kernel", "prefill") is None


def test_a_list_shorter_than_one_call_is_an_error(tmp_path):
    write_list(tmp_path / "nvfp4_quantize.csv",
               [("nvfp4_absmax_kernel", full(92700, 622000000, 3900000))])
    with pytest.raises(ValueError):
        bench.write_traffic(str(tmp_path), str(tmp_path / "t.json"))


def test_kernels_per_call_matches_the_workloads():
    assert bench.kernels_per_call("decode") == 1
    assert bench.kernels_per_call("prefill_logprobs") == 2
    assert bench.kernels_per_call("nvfp4_quantize") == 2
    assert bench.kernels_per_call("vocab_parallel_logprobs") == 3
    assert bench.roofline_kernel("nvfp4") == "lmhead_w4a16_nvfp4_kernel"
