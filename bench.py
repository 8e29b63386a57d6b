"""Benchmark of the LM-head library on B200: one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Workloads (seeded synthetic inputs from tests/synth.py; the pages use no dataset):
  decode       (default) rows in {1,2,4,8,16,32,64}, H = 2048, V = 151936, bf16 -> fp32,
               alpha = 1/8. One step = one call per row count (7 calls).
  spec_verify  rows in {128, 97, 32}, H = 4096, V = 128256, alpha = 1/16 (3 calls per step).
  prefill      rows = 8192, H = 4096, V = 151936, alpha = 1/8 (1 call per step).
  nvfp4        W4A16 NVFP4 head, rows in {1, 16, 64, 65, 256}, H = 2048, V = 151936, bf16 out.
  decode_f16_bias   the decode shape with fp16 operands and an fp16 embedding bias.
  prefill_logprobs  the prefill shape, log-probabilities of one target per row, no logits out.
  vocab_parallel_logprobs  the same with W's rows split over the GPUs (see below).
  nvfp4_quantize    the NVFP4 quantiser of a bf16 W [151936, 2048].
  prefill_2048      the prefill kernel on 2048 rows (a small case for profiling).
  prefill_4608      the same on 4608 rows: two row-tile groups, as at 8192 (profiling).
Metric: microseconds per LM-head call (lower is better) and the fraction of the roofline the
kernel reaches. Every call reads a weight matrix larger than L2 (126 MB); two copies of it are
alternated so no call starts with its weights cached by the previous one.

Multi-GPU: the head does not shard across the replicas (one process per GPU runs the same
workload on its own GPU, no collective in the data path); timing is the max over ranks and
`value` is the job's time per call: max elapsed / (calls per rank * N). The exception is
vocab_parallel_logprobs (the prefill log-probabilities with W's rows split over the N GPUs, one
all-gather of 12 bytes per row and GPU per call): there the N ranks make each call together, so
`value` = max elapsed / calls, and the scaling is strong.

--impl reference times the CPU oracle (the reference arm of this build) on a bounded sample of
the same workload, scaled to the same metric; only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

_ROOT = os.path.dirname(os.path.abspath(__file__))
for _p in (_ROOT, os.path.join(_ROOT, "tests")):   # tests/ holds the seeded input generator
    if _p not in sys.path:
        sys.path.insert(0, _p)

METRIC = "LM-head µs/call and achieved % of roofline (HBM GB/s decode, TFLOP/s prefill)"
UNIT = "us/call"

WORKLOAD_TEXT = {
    "decode": "decode LM head: rows {1,2,4,8,16,32,64}, H=2048, V=151936, bf16 hidden/W, fp32 "
              "accumulate and logits, alpha=1/8",
    "spec_verify": "speculative-verify LM head: rows {128,97,32}, H=4096, V=128256, bf16 in, "
                   "fp32 out, alpha=1/16",
    "prefill": "prefill LM head: rows=8192, H=4096, V=151936, bf16 in, fp32 out, alpha=1/8",
    "nvfp4": "NVFP4 W4A16 head: rows {1,16,64,65,256}, H=2048, V=151936, E2M1 + E4M3/16 + fp32 "
             "scale, bf16 hidden and logits, alpha=1/8",
    "prefill_2048": "prefill kernel on 2048 rows (profiling case): H=4096, V=151936, bf16 in, "
                    "fp32 out, alpha=1/8",
    "prefill_4608": "prefill kernel on 4608 rows (profiling case, two row-tile groups): H=4096, "
                    "V=151936, bf16 in, fp32 out, alpha=1/8",
    "prefill_logprobs_2048": "log-prob mode of the prefill kernel on 2048 rows (profiling case): "
                             "H=4096, V=151936, bf16 in, alpha=1/8, no logits written",
    "prefill_logprobs": "prefill LM head computing log-probabilities of one target token per row "
                        "(log-softmax in the epilogue, no logits written): rows=8192, H=4096, "
                        "V=151936, bf16 in, fp32 out, alpha=1/8",
    "vocab_parallel_logprobs": "vocab-parallel prefill log-probabilities: W[151936, 4096] split "
                               "in contiguous row slices over the GPUs; per GPU the slice's "
                               "(max, sum, target logit) for rows=8192, an all-gather of 12 B "
                               "per row, the merge; bf16 in, fp32 out, alpha=1/8",
    "nvfp4_quantize": "NVFP4 quantiser (absmax pass, then encode pass) of a bf16 W[151936, 2048] "
                      "into E2M1 codes, E4M3 block scales and an fp32 global scale",
    "decode_f16_bias": "decode LM head with fp16 operands and an fp16 embedding bias: rows "
                       "{1,2,4,8,16,32,64}, H=2048, V=151936, fp32 accumulate and logits, "
                       "alpha=1/8",
}


def kernel_source_hash() -> str:
    """sha256 over the CUDA sources and the public header (what a traffic figure is tied to)."""
    import glob
    import hashlib
    h = hashlib.sha256()
    files = sorted(glob.glob(os.path.join(_ROOT, "fp32_accumulate_lm_b200", "csrc", "*")) +
                   glob.glob(os.path.join(_ROOT, "include", "*.h")))
    for f in files:
        with open(f, "rb") as fh:
            h.update(os.path.basename(f).encode())
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch (read + write) from profiles/traffic.json, if it was captured from
    the current kernel sources; None otherwise."""
    try:
        with open(os.path.join(_ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)
    except Exception:
        return None
    ent = rec.get(kernel, {}).get(workload)
    if not ent or ent.get("source_hash") != kernel_source_hash():
        return None
    return ent.get("bytes_per_launch")


def roofline_kernel(name: str) -> str:
    """The kernel (or kernel pair) a workload's roofline and traffic figures belong to."""
    return ("nvfp4_encode_kernel + nvfp4_absmax_kernel" if name == "nvfp4_quantize" else
            "lmhead_w4a16_nvfp4_kernel" if name == "nvfp4" else "lmhead_bf16_f32_kernel")


def kernels_per_call(name: str) -> int:
    """Launches of this library's kernels per call of a workload."""
    if name == "vocab_parallel_logprobs":
        return 3            # slice stats, combine, merge
    if name in ("nvfp4_quantize", "prefill_logprobs", "prefill_logprobs_2048"):
        return 2            # absmax + encode; log-prob epilogue + combine
    return 1


TRAFFIC_ABOUT = (
    "DRAM bytes per call (dram__bytes_read.sum + dram__bytes_write.sum, summed over the call's "
    "kernels), mean over the calls of one timed bench step, from one ncu capture per workload "
    "(1 pass, --clock-control none): python bench.py --workload W --only --steps 1 --warmup 3 "
    "--no-cpu-baseline under ncu --metrics gpu__time_duration.sum,dram__bytes_read.sum,"
    "dram__bytes_write.sum -k 'regex:(lmhead|nvfp4)' -s <warm-up launches> -c <one step's "
    "launches> --csv --log-file DIR/W.csv; written by python bench.py --traffic-from DIR; valid "
    "only while source_hash matches bench.kernel_source_hash().")

_NCU_UNITS = {"byte": 1, "B": 1, "Kbyte": 1e3, "KB": 1e3, "Mbyte": 1e6, "MB": 1e6, "Gbyte": 1e9,
              "GB": 1e9, "nsecond": 1, "ns": 1, "usecond": 1e3, "us": 1e3, "msecond": 1e6,
              "ms": 1e6}


def read_ncu_launches(path: str) -> list:
    """An ncu --csv launch list as one dict per launch, in launch order: the kernel name, "ns"
    (gpu__time_duration.sum) and the dram__bytes_* counters in bytes, when captured."""
    import csv
    launches, hdr = {}, None
    with open(path, newline="") as f:
        for row in csv.reader(f):
            if row and row[0] == "ID":
                hdr = row
                continue
            if hdr is None or len(row) != len(hdr):
                continue              # ncu's own messages before the table
            d = dict(zip(hdr, row))
            e = launches.setdefault(int(d["ID"]), {"name": d["Kernel Name"]})
            v = float(d["Metric Value"].replace(",", "")) * _NCU_UNITS[d["Metric Unit"]]
            if d["Metric Name"] == "gpu__time_duration.sum":
                e["ns"] = v
            elif d["Metric Name"].startswith("dram__bytes"):
                e[d["Metric Name"]] = v
    return [launches[k] for k in sorted(launches)]


def write_traffic(csv_dir: str, out_path: str | None = None) -> dict:
    """profiles/traffic.json from the launch lists DIR/<workload>.csv (one timed step of each
    workload, captured as TRAFFIC_ABOUT says), tied to the current kernel sources."""
    h = kernel_source_hash()
    res = {"_about": TRAFFIC_ABOUT}
    for name in sorted(WORKLOAD_TEXT):
        path = os.path.join(csv_dir, name + ".csv")
        if not os.path.exists(path):
            continue
        launches = read_ncu_launches(path)
        kpc = kernels_per_call(name)
        calls = len(launches) // kpc
        if calls == 0:
            raise ValueError(f"{path}: {len(launches)} launches, fewer than one call's {kpc}")
        groups = [launches[c * kpc:(c + 1) * kpc] for c in range(calls)]
        ent = {"calls": calls, "kernels_per_call": kpc,
               "per_call_ns_under_ncu": [sum(k["ns"] for k in g) for g in groups],
               "source_hash": h}
        if all("dram__bytes_read.sum" in k and "dram__bytes_write.sum" in k for k in launches):
            per_call = [int(sum(k["dram__bytes_read.sum"] + k["dram__bytes_write.sum"] for k in g))
                        for g in groups]
            ent["bytes_per_launch"] = int(sum(per_call) / calls)
            ent["per_call_bytes"] = per_call
        else:
            ent["bytes_per_launch"] = None
            ent["note"] = ("launch list only (gpu__time_duration.sum); DRAM bytes not captured "
                           "at this size")
        res.setdefault(roofline_kernel(name), {})[name] = ent
    out_path = out_path or os.path.join(_ROOT, "profiles", "traffic.json")
    with open(out_path, "w") as f:
        json.dump(res, f, indent=1)
        f.write("\n")
    return res


def load_peaks() -> dict:
    path = os.path.join(_ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d["bf16_tflops_sustained"]), "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# ---------------------------------------------------------------- clocks sampler (NVML)

class ClockSampler:
    """Samples SM clock and throttle reasons of one GPU every ~20 ms on a thread."""

    REASONS = {
        "hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
        "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, index: int):
        self.index = index
        self.samples: list[int] = []
        self.reasons: set[str] = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for name, bit in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.02)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self) -> dict:
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        self._stop.set()
        self._t.join()
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ---------------------------------------------------------------- workloads on the GPU

class Workload:
    """Device-resident inputs and outputs of one workload, and one step = its list of calls."""

    def __init__(self, name: str, device, world: int = 1, rank: int = 0):
        import torch
        import synth
        self.name = name
        rows_list, H, V, std, alpha = synth.WORKLOADS[name]
        self.rows_list, self.H, self.V, self.alpha = rows_list, H, V, alpha
        seed = {"decode": synth.SEED_DECODE, "spec_verify": synth.SEED_SPEC,
                "prefill": synth.SEED_PREFILL, "nvfp4": synth.SEED_NVFP4,
                "prefill_2048": synth.SEED_PREFILL, "prefill_4608": synth.SEED_PREFILL,
                "decode_f16_bias": synth.SEED_F16,
                "nvfp4_quantize": synth.SEED_NVFP4, "prefill_logprobs": synth.SEED_PREFILL,
                "prefill_logprobs_2048": synth.SEED_PREFILL,
                "vocab_parallel_logprobs": synth.SEED_PREFILL}[name]
        rmax = max(rows_list)
        self.quantize = name == "nvfp4_quantize"
        self.vocab_parallel = name == "vocab_parallel_logprobs"
        self.world = world
        if self.quantize:
            # one call quantises all V rows of a bf16 W; two copies alternate (each > L2)
            import fp32_accumulate_lm_b200 as lm
            self.dtype = torch.bfloat16
            self.bias = None
            self.nvfp4 = False
            self.logprobs = False
            self.vocab_parallel = False
            self.weights = [synth.weight(V, H, std, seed + i, device=device) for i in (0, 1)]
            self.hidden = self.weights[0]
            self.hid = {V: self.weights[0]}
            self.outs = {V: torch.empty((V, H // 2), dtype=torch.uint8, device=device)}
            self.q_scales = torch.empty((V, H // 16), dtype=torch.uint8, device=device)
            self.q_g = torch.empty((1,), dtype=torch.float32, device=device)
            self.ws = torch.empty((lm.nvfp4_quantize_workspace_bytes(),), dtype=torch.uint8,
                                  device=device)
            self.calls = 0
            return
        self.dtype = torch.float16 if name == "decode_f16_bias" else torch.bfloat16
        self.hidden = synth.hidden(rmax, H, seed, device=device, dtype=self.dtype)
        self.bias = (synth.bias(V, synth.SEED_BIAS, device=device, dtype=self.dtype)
                     if name == "decode_f16_bias" else None)
        self.nvfp4 = name == "nvfp4"
        if self.nvfp4:
            self.weights = [synth.random_nvfp4_codes(V, H, seed + i, device=device) for i in (0, 1)]
            self.g = 1.0 / 4096
            self.outs = {r: torch.empty((r, V), dtype=torch.bfloat16, device=device)
                         for r in rows_list}
        elif self.vocab_parallel:
            # this rank's contiguous slice of each of the two weight copies
            import fp32_accumulate_lm_b200 as lm
            self.v_begin, self.V_shard = lm.vocab_shard(V, world, rank)
            self.weights = []
            for i in (0, 1):
                full = synth.weight(V, H, std, seed + i, device=device, dtype=self.dtype)
                self.weights.append(full if world == 1 else
                                    full[self.v_begin:self.v_begin + self.V_shard].clone())
                del full
        else:
            self.weights = [synth.weight(V, H, std, seed + i, device=device, dtype=self.dtype)
                            for i in (0, 1)]
            self.outs = {r: torch.empty((r, V), dtype=torch.float32, device=device)
                         for r in rows_list}
        self.hid = {r: self.hidden[:r] for r in rows_list}
        self.general = self.bias is not None or self.dtype != torch.bfloat16  # lmhead_logits_f32
        self.logprobs = name in ("prefill_logprobs", "vocab_parallel_logprobs",
                                 "prefill_logprobs_2048")
        if self.logprobs:
            import fp32_accumulate_lm_b200 as lm
            gen = torch.Generator(device="cpu")
            gen.manual_seed(seed + 700_000)
            self.targets = torch.randint(0, V, (rmax,), generator=gen, dtype=torch.int32).to(device)
            self.outs = {r: torch.empty((r,), dtype=torch.float32, device=device) for r in rows_list}
            self.lse = {r: torch.empty((r,), dtype=torch.float32, device=device) for r in rows_list}
            vw = self.V_shard if self.vocab_parallel else V
            self.ws = torch.empty((lm.logprobs_workspace_bytes(rmax, vw),), dtype=torch.uint8,
                                  device=device)
            if self.vocab_parallel:
                self.stats = {r: torch.empty((r, 3), dtype=torch.float32, device=device)
                              for r in rows_list}
        self.calls = 0

    def call(self, r: int, hidden=None, out=None, stream=None):
        import fp32_accumulate_lm_b200 as lm
        if self.quantize:
            W = self.weights[self.calls & 1] if hidden is None else hidden
            self.calls += 1
            lm.nvfp4_quantize(W, workspace=self.ws,
                              out=(self.outs[r] if out is None else out, self.q_scales, self.q_g),
                              stream=stream)
            return
        w = self.weights[self.calls & 1]
        self.calls += 1
        h = self.hid[r] if hidden is None else hidden
        o = self.outs[r] if out is None else out
        if self.nvfp4:
            lm.logits_w4a16_nvfp4(h, w[0], w[1], self.g, self.alpha, out=o, stream=stream)
        elif self.vocab_parallel:
            lm.logprobs_vocab_parallel(h, w, self.v_begin, self.targets[:r], self.alpha,
                                       workspace=self.ws, stats=self.stats[r],
                                       out=(o, self.lse[r]), stream=stream)
        elif self.logprobs:
            lm.logprobs_f32(h, w, self.targets[:r], self.alpha, workspace=self.ws,
                            out=(o, self.lse[r]), stream=stream)
        elif self.general:
            lm.logits_f32(h, w, self.alpha, bias=self.bias, out=o, stream=stream)
        else:
            lm.logits_bf16_f32(h, w, self.alpha, out=o, stream=stream)

    def bytes_of(self, r: int) -> int:
        H, V = self.H, self.V
        if self.quantize:  # two passes over W (absmax, then encode), codes, scales and g out
            return 2 * V * H * 2 + V * H // 2 + V * H // 16 + 4
        if self.nvfp4:
            return V * H // 2 + V * H // 16 + 4 + r * H * 2 + r * V * 2
        if self.vocab_parallel:  # this rank's slice; the stats out, gathered, read by the merge
            n = self.V_shard
            n_chunks = 4 * ((n + 127) // 128)
            return (n * H * 2 + r * H * 2 + r * 4 + 2 * r * n_chunks * 8 + r * 12
                    + 2 * self.world * r * 12 + r * 8)
        if self.logprobs:  # W, hidden, targets in; the chunk pairs out and back; lp, lse out
            n_chunks = 4 * ((V + 127) // 128)
            return V * H * 2 + r * H * 2 + r * 4 + 2 * r * n_chunks * 8 + r * 8
        return V * H * 2 + r * H * 2 + r * V * 4 + (V * 2 if self.bias is not None else 0)

    def flops_of(self, r: int) -> int:
        if self.vocab_parallel:
            return 2 * r * self.H * self.V_shard
        return 0 if self.quantize else 2 * r * self.H * self.V


def dist_setup(n_gpus: int, backend: str = "nccl"):
    """One process per GPU (torchrun env). `backend` "gloo" runs the same plumbing on CPU."""
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    elif backend == "nccl":
        torch.cuda.set_device(0)
    return world, rank, local


def _device_sync():
    import torch
    if torch.cuda.is_available() and torch.cuda.is_initialized():
        torch.cuda.synchronize()


def barrier(world: int):
    """Device idle on every rank, then a process-group barrier, then idle again."""
    import torch.distributed as dist
    _device_sync()
    if world > 1:
        dist.barrier()
    _device_sync()


def max_over_ranks(x: float, world: int) -> float:
    import torch
    import torch.distributed as dist
    if world == 1:
        return x
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_us_per_call(elapsed_ms: float, steps: int, calls_per_step: int, world: int) -> float:
    """Whole-job time per call: the slowest rank's elapsed time over every rank's calls."""
    return elapsed_ms * 1e3 / (steps * calls_per_step * world)


# The default run measures the decode head as the headline `value`, then every other workload of
# the library into the line's "workloads" map, each with its own roofline, e2e, clocks and CPU
# baseline, so one run covers the whole metric (HBM-bound decode shapes, tensor-bound prefill).
PRIMARY = "decode"
SECONDARY = ["spec_verify", "prefill", "nvfp4", "decode_f16_bias", "prefill_logprobs",
             "vocab_parallel_logprobs", "nvfp4_quantize"]
# A timed region at least this long is "a long step": the sustained bf16 peak applies.
SUSTAINED_REGION_S = 1.0
PER_ROW_IDLE_S = 1.0   # idle before each per-row-count loop (see measure)
PER_ROW_WARMUP = 20    # untimed calls of the row count before its loop
PER_ROW_MIN_CALLS = 100  # timed calls per row count at least
PER_ROW_BLOCKS = 5     # blocks of each per-row-count loop (median and minimum of their means)


def config_of(name: str, world: int) -> dict:
    """The workload's description: the same keys and values in both arms of the bench."""
    import synth
    rows_list = synth.WORKLOADS[name][0]
    vp = name == "vocab_parallel_logprobs"
    return {"workload": WORKLOAD_TEXT[name],
            "l2": "weights 2x larger than L2 per call; two weight copies alternated",
            "parallelism": (f"vocab-parallel x{world} (all-gather of the row stats)" if vp else
                            f"replicas x{world} (no data-path collective)"),
            "calls_per_step": len(rows_list),
            "rows_per_call": list(rows_list)}


def measure(name: str, args, world: int, rank: int, peaks: dict, cpu_budget_s: float) -> dict:
    """Warm-up, then a timed region of args.steps steps of workload `name`: per-launch CUDA events
    on the launching stream, barrier + synchronize on both sides, max over ranks. Returns the
    workload's record (its inputs are freed before returning)."""
    import torch
    import fp32_accumulate_lm_b200 as lm

    dev = torch.device("cuda", torch.cuda.current_device())
    wl = Workload(name, dev, world, rank)
    stream = torch.cuda.current_stream()
    rl = wl.rows_list
    calls_per_step = len(rl)

    for _ in range(args.warmup):
        for r in rl:
            wl.call(r)
    torch.cuda.synchronize()
    if lm.device_status(clear=True) != 0:
        raise RuntimeError(f"{name}: device status word set during warm-up")

    # The timed region: exactly K steps, bracketed by barrier + synchronize, one CUDA event at
    # each end on the launching stream (an event between every two calls would add about 3 us to
    # each call on these GPUs).
    n_ev = args.steps * calls_per_step
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(torch.cuda.current_device())
    barrier(world)
    sampler.start()
    e_start.record(stream)
    for _ in range(args.steps):
        for r in rl:
            wl.call(r)
    e_end.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    barrier(world)
    if lm.device_status(clear=True) != 0:
        raise RuntimeError(f"{name}: device status word set during the timed region")
    elapsed_ms = e_start.elapsed_time(e_end)
    elapsed_ms = max_over_ranks(elapsed_ms, world)

    # Per row count (the detail below the headline): each row count alone, between two events.
    # Each loop starts after PER_ROW_IDLE_S of idle, so that every row count starts from the same
    # power state (the loops follow the timed region, and after tensor-heavy calls the power cap
    # holds the SM clock down for a while), then runs PER_ROW_WARMUP untimed calls of its row
    # count so the clock is back up from idle, then times max(steps, PER_ROW_MIN_CALLS) calls.
    # The loop is cut into PER_ROW_BLOCKS blocks with an event at each boundary, so the median and
    # the minimum of the block means come with the mean.
    per_row_ms, per_row_blocks = {}, {}
    per_row_calls = max(args.steps, PER_ROW_MIN_CALLS)
    per_block = -(-per_row_calls // PER_ROW_BLOCKS)
    per_row_calls = per_block * PER_ROW_BLOCKS
    for r in rl:
        time.sleep(PER_ROW_IDLE_S)
        for _ in range(max(args.warmup, PER_ROW_WARMUP)):
            wl.call(r)
        torch.cuda.synchronize()
        barrier(world)
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(PER_ROW_BLOCKS + 1)]
        evs[0].record(stream)
        for blk in range(PER_ROW_BLOCKS):
            for _ in range(per_block):
                wl.call(r)
            evs[blk + 1].record(stream)
        torch.cuda.synchronize()
        per_row_ms[r] = evs[0].elapsed_time(evs[-1]) / per_row_calls
        per_row_blocks[r] = [evs[i].elapsed_time(evs[i + 1]) / per_block
                             for i in range(PER_ROW_BLOCKS)]
    barrier(world)

    # per row count: mean launch duration, algorithmic bytes and flops
    detail = {}
    tot_bytes = tot_flops = 0.0
    for r in rl:
        mean_ms = per_row_ms[r]
        b, fl = wl.bytes_of(r), wl.flops_of(r)
        blocks = per_row_blocks[r]
        detail[str(r)] = {"us": round(mean_ms * 1e3, 2), "calls": per_row_calls,
                          "us_median_block": round(statistics.median(blocks) * 1e3, 2),
                          "us_min_block": round(min(blocks) * 1e3, 2),
                          "GBps": round(b / (mean_ms * 1e-3) / 1e9, 1),
                          "TFLOPs": round(fl / (mean_ms * 1e-3) / 1e12, 1)}
        tot_bytes += b
        tot_flops += fl
    # the timed region's mean launch duration (one step = one launch per row count)
    tot_ms = elapsed_ms / args.steps
    # prefill, its profiling case, log-probs, vocab-parallel log-probs
    tensor_bound = name.startswith("prefill") or wl.vocab_parallel
    if tensor_bound:
        achieved = tot_flops / (tot_ms * 1e-3) / 1e12
        long_region = elapsed_ms >= SUSTAINED_REGION_S * 1e3
        peak = peaks["bf16_tflops_sustained" if long_region else "bf16_tflops"]
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4),
                "peak_kind": ("bf16 dense, sustained" if long_region else "bf16 dense, burst") +
                             f" ({peaks['source']}; timed region {elapsed_ms / 1e3:.2f} s)"}
    else:
        achieved = tot_bytes / (tot_ms * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "peak_kind": f"HBM copy ({peaks['source']})"}
    roof["kernel"] = roofline_kernel(name)
    roof["traffic"] = recorded_traffic(roof["kernel"], name)
    roof["algorithmic_bytes_per_launch"] = int(tot_bytes / calls_per_step)
    roof["source_hash"] = kernel_source_hash()

    # the same step replayed from a CUDA graph, and the pages' PyTorch call for context
    graph = run_graph(args, wl, world)
    torch_mm = run_torch_mm(args, wl, tot_ms / calls_per_step)

    # end to end through the C ABI: pinned host hidden -> device, call, outputs -> pinned host
    e2e = run_e2e(args, wl, world)

    # Replicas: every rank makes whole calls. Vocab-parallel: the ranks make each call together.
    value = job_us_per_call(elapsed_ms, args.steps, calls_per_step,
                            1 if wl.vocab_parallel else world)
    rec = {
        "value": round(value, 3), "unit": UNIT, "ms_per_step": round(elapsed_ms / args.steps, 5),
        "scaling": "strong" if wl.vocab_parallel else "weak",
        "dtype": ("f32" if wl.quantize else "e2m1xbf16" if wl.nvfp4 else
                  "f16" if wl.dtype == torch.float16 else "bf16"),
        "config": config_of(name, world),
        "per_rows": detail,
        "roofline": roof,
        "e2e": e2e,
        "graph": graph,
        "torch_mm": torch_mm,
        "gpu_launches": n_ev * kernels_per_call(name),
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and cpu_budget_s > 0:
        rec["cpu_baseline"] = cpu_baseline(name, wl, cpu_budget_s)
    del wl
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return rec


def run_ours(args) -> dict | None:
    world, rank, local = dist_setup(args.gpus)
    peaks = load_peaks()
    budget = 0.0 if args.no_cpu_baseline else 10.0
    main = measure(args.workload, args, world, rank, peaks, budget)
    line = {
        "metric": METRIC, "value": main["value"], "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": main["ms_per_step"],
        "higher_is_better": False, "scaling": main["scaling"], "vs_baseline": None,
        "dtype": main["dtype"],
        "data": "synthetic (seeded N(0,1) hidden, N(0,std) weights; no dataset on the pages)",
        "config": main["config"],
        "per_rows": main["per_rows"],
        "roofline": main["roofline"],
        "e2e": main["e2e"],
        "graph": main["graph"],
        "torch_mm": main["torch_mm"],
        "gpu_launches": main["gpu_launches"],
        "clocks": main["clocks"],
    }
    if "cpu_baseline" in main:
        line["cpu_baseline"] = main["cpu_baseline"]
    if args.workload == PRIMARY and not args.only:
        # every rank runs the same workloads in the same order (vocab-parallel has a collective)
        line["workloads"] = {name: measure(name, args, world, rank, peaks, budget / 2)
                             for name in SECONDARY}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return line if rank == 0 else None


def run_graph(args, wl, world: int) -> dict:
    """The timed region's calls replayed from a CUDA graph: two steps (an even number of calls,
    so the two weight copies keep alternating across replays) captured once through the same
    Python calls, then max(1, steps // 2) replays between two events on the launching stream.
    This leaves out the host's launch work that the main figure includes. The vocab-parallel
    workload is left out: its step holds a collective."""
    import torch
    if wl.vocab_parallel:
        return {"skipped": "the step holds an all-gather across the ranks"}
    stream = torch.cuda.current_stream()
    steps_per_graph = 2
    calls = steps_per_graph * len(wl.rows_list)
    g = torch.cuda.CUDAGraph()
    # thread_local: other threads' CUDA calls (the NCCL watchdog's under torchrun) may go on
    # during the capture; only this thread's calls are checked
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        for _ in range(steps_per_graph):
            for r in wl.rows_list:
                wl.call(r)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    reps = max(1, args.steps // steps_per_graph)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    a.record(stream)
    for _ in range(reps):
        g.replay()
    b.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    elapsed_ms = max_over_ranks(a.elapsed_time(b), world)
    del g
    import fp32_accumulate_lm_b200 as lm
    if lm.device_status(clear=True) != 0:
        raise RuntimeError(f"{wl.name}: device status word set during the graph replays")
    return {"value": round(job_us_per_call(elapsed_ms, reps, calls, world), 3), "unit": UNIT,
            "replays": reps, "calls_per_replay": calls}


def run_torch_mm(args, wl, ours_ms_per_call: float) -> dict:
    """Context only: the pages' own call, torch.mm(hidden, W.T, out_dtype=float32) (cuBLAS
    through PyTorch), then the multiply by alpha (after adding the bias, where the workload has
    one), on the same inputs, the same weight alternation and the same timed-region shape.
    Only the workloads whose product is the fp32 logits have it."""
    import torch
    if wl.quantize or wl.nvfp4 or wl.logprobs or wl.vocab_parallel:
        return {"skipped": "no fp32-logits call to compare with"}
    stream = torch.cuda.current_stream()
    k = [0]
    into = [True]  # the out= form, unless this torch refuses it with out_dtype

    def one(r):
        w = wl.weights[k[0] & 1]
        k[0] += 1
        if into[0]:
            try:
                o = torch.mm(wl.hid[r], w.t(), out_dtype=torch.float32, out=wl.outs[r])
            except (RuntimeError, TypeError):
                into[0] = False
        if not into[0]:
            o = torch.mm(wl.hid[r], w.t(), out_dtype=torch.float32)
        if wl.bias is not None:
            o.add_(wl.bias)
        o.mul_(wl.alpha)

    for _ in range(args.warmup):
        for r in wl.rows_list:
            one(r)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.steps):
        for r in wl.rows_list:
            one(r)
    b.record(stream)
    torch.cuda.synchronize()
    ms_per_call = a.elapsed_time(b) / (args.steps * len(wl.rows_list))
    return {"value": round(ms_per_call * 1e3, 3), "unit": UNIT,
            "ours_speedup": round(ms_per_call / ours_ms_per_call, 3),
            "how": ("torch.mm(hidden, W.T, out_dtype=float32, out=logits)" if into[0] else
                    "logits = torch.mm(hidden, W.T, out_dtype=float32)") +
                   (", logits.add_(bias)" if wl.bias is not None else "") +
                   ", logits.mul_(alpha); per rank, context only"}


def run_e2e(args, wl, world: int) -> dict:
    """Same metric through the public call with host buffers: every call copies its hidden rows
    from pinned host memory and its result back to pinned host memory inside the timed region,
    pipelined as a caller would: the copies run on their own streams (host-to-device and
    device-to-host, so PCIe carries both directions at once) and two sets of buffers alternate,
    so call i's result travels back while call i + 1 computes. Events order each copy after the
    work it depends on and keep a buffer from being overwritten before its copy has read it."""
    import torch
    compute = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    rl = wl.rows_list
    h_host = {r: wl.hid[r].cpu().pin_memory() for r in rl}
    h_dev = {r: [torch.empty_like(wl.hid[r]) for _ in range(2)] for r in rl}
    o_dev = {r: [wl.outs[r], torch.empty_like(wl.outs[r])] for r in rl}
    # one host buffer per row count: the downloads run in order on one stream
    o_host = {r: torch.empty(wl.outs[r].shape, dtype=wl.outs[r].dtype).pin_memory() for r in rl}
    ev = lambda: torch.cuda.Event()
    uploaded = [ev(), ev()]     # hidden rows of the slot are on the device
    computed = [ev(), ev()]     # the slot's call is done (its hidden rows may be overwritten)
    downloaded = [ev(), ev()]   # the slot's result is on the host (its buffer may be reused)
    for e in computed + downloaded:
        e.record(compute)
    calls = [0]

    def one_call(r):
        s = calls[0] & 1
        calls[0] += 1
        up.wait_event(computed[s])
        with torch.cuda.stream(up):
            h_dev[r][s].copy_(h_host[r], non_blocking=True)
        uploaded[s].record(up)
        compute.wait_event(uploaded[s])
        compute.wait_event(downloaded[s])
        wl.call(r, hidden=h_dev[r][s], out=o_dev[r][s], stream=compute)
        computed[s].record(compute)
        down.wait_event(computed[s])
        with torch.cuda.stream(down):
            o_host[r].copy_(o_dev[r][s], non_blocking=True)
        downloaded[s].record(down)

    steps = max(1, min(args.steps, 50))
    for _ in range(2):
        for r in rl:
            one_call(r)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(compute)
    up.wait_event(e0)
    down.wait_event(e0)
    for _ in range(steps):
        for r in rl:
            one_call(r)
    compute.wait_stream(up)
    compute.wait_stream(down)
    e1.record(compute)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    h2d = sum(h_host[r].numel() * h_host[r].element_size() for r in rl)
    d2h = sum(o_host[r].numel() * o_host[r].element_size() for r in rl)
    share = 1 if wl.vocab_parallel else world   # calls made together count once
    return {"value": round(ms * 1e3 / (steps * len(rl) * share), 3), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "pipelining": "copies on two streams, two buffer sets alternated"}


# ---------------------------------------------------------------- CPU oracle (baseline arm)
#
# Both CPU legs -- the repo arm's cpu_baseline and the reference arm -- time the oracle the same
# way: the step's first n distinct hidden rows (n <= 64) against the first `vslice` rows of W,
# scaled by V / vslice and by the step's total rows / n, per call. The oracle decodes W once per
# call, so timing the distinct rows together amortises that decode as a real call would.

ORACLE_MAX_ROWS = 64


def _oracle_inputs(name: str, n_rows: int, vslice: int, wl=None) -> dict:
    """numpy inputs for the oracle: hidden rows [n_rows, H] and the first vslice rows of the
    weights (NVFP4 codes and scales for the NVFP4 head), from the GPU workload's own tensors
    when `wl` is given, else regenerated on the host with the workload's seeds."""
    import numpy as np
    import torch
    import synth
    rows_list, H, V, std, alpha = synth.WORKLOADS[name]
    seed = {"decode": synth.SEED_DECODE, "spec_verify": synth.SEED_SPEC,
            "nvfp4": synth.SEED_NVFP4, "decode_f16_bias": synth.SEED_F16,
            "nvfp4_quantize": synth.SEED_NVFP4}.get(name, synth.SEED_PREFILL)
    f16 = name == "decode_f16_bias"
    dt = torch.float16 if f16 else torch.bfloat16
    bits = lambda t: t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    d = {"name": name, "H": H, "V": V, "alpha": alpha, "f16": f16}
    if name == "nvfp4_quantize":
        d["w"] = (bits(wl.weights[0][:vslice]) if wl is not None
                  else synth.weight(vslice, H, std, seed, dtype=dt))
        return d
    d["h"] = (bits(wl.hidden[:n_rows]) if wl is not None
              else synth.hidden(n_rows, H, seed, dtype=dt))
    if name == "nvfp4":
        if wl is not None:
            d["packed"] = wl.weights[0][0][:vslice].cpu().numpy()
            d["scales"] = wl.weights[0][1][:vslice].cpu().numpy()
            d["g"] = wl.g
        else:
            d["packed"], d["scales"] = synth.random_nvfp4_codes(vslice, H, seed)
            d["g"] = 1.0 / 4096
        return d
    d["w"] = bits(wl.weights[0][:vslice]) if wl is not None else synth.weight(vslice, H, std,
                                                                               seed, dtype=dt)
    d["b"] = ((bits(wl.bias[:vslice]) if wl is not None else synth.bias(vslice, synth.SEED_BIAS,
                                                                        dtype=dt))
              if f16 else None)
    if name in ("prefill_logprobs", "vocab_parallel_logprobs", "prefill_logprobs_2048"):
        gen = torch.Generator(device="cpu")
        gen.manual_seed(seed + 700_000)
        d["t"] = torch.randint(0, vslice, (n_rows,), generator=gen, dtype=torch.int32).numpy()
    return d


def _oracle_run(d: dict) -> float:
    """Seconds of one oracle call on the prepared inputs."""
    import oracle
    t0 = time.perf_counter()
    if d["name"] == "nvfp4_quantize":
        oracle.nvfp4_quantize(d["w"])
    elif d["name"] == "nvfp4":
        oracle.logits_w4a16_nvfp4(d["h"], d["packed"], d["scales"], d["g"], d["alpha"])
    elif "t" in d:
        oracle.logprobs_f32(d["h"], d["w"], d["alpha"], d["t"])
    else:
        oracle.logits_f32(d["h"], d["w"], d["alpha"], bias_bits=d["b"],
                          dtype="f16" if d["f16"] else "bf16")
    return time.perf_counter() - t0


def _oracle_plan(name: str, budget_s: float, wl=None):
    """(n_rows, vslice, per-call scale) for oracle calls of about budget_s seconds each: the
    step's distinct rows (at most 64), and as much of the vocabulary as the budget allows."""
    import synth
    rows_list, H, V, _, _ = synth.WORKLOADS[name]
    if name == "nvfp4_quantize":
        probe = 1024
        t = _oracle_run(_oracle_inputs(name, 0, probe, wl))
        vslice = int(max(probe, min(V, probe * budget_s / max(t, 1e-6))))
        return 0, vslice, V / vslice
    n_rows = min(max(rows_list), ORACLE_MAX_ROWS)
    probe = min(V, 2048)
    t = _oracle_run(_oracle_inputs(name, n_rows, probe, wl))
    vslice = int(max(probe, min(V, probe * budget_s / max(t, 1e-6))))
    scale = (V / vslice) * (sum(rows_list) / n_rows) / len(rows_list)
    return n_rows, vslice, scale


def _oracle_sample_text(name: str, n_rows: int, vslice: int, secs: float) -> str:
    import synth
    rows_list, H, V, _, _ = synth.WORKLOADS[name]
    if name == "nvfp4_quantize":
        return (f"{vslice} of W's {V} rows x H={H} ({secs:.1f} s per sample), scaled by rows to "
                "one call")
    return (f"the step's first {n_rows} distinct rows (of {sum(rows_list)} rows in "
            f"{len(rows_list)} calls) x {vslice} of V={V} vocab rows x H={H} ({secs:.1f} s per "
            "sample), scaled by V and by rows, per call")


def host_cpu() -> dict:
    """The host's CPU model and logical core count, for the CPU-baseline records."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu_model": model, "nproc": os.cpu_count()}


def cpu_baseline(name: str, wl, budget_s: float = 10.0) -> dict:
    """The oracle as it stands, on the host cores, on the bench's own inputs (rank 0, N = 1)."""
    import oracle
    n_rows, vslice, scale = _oracle_plan(name, budget_s, wl)
    d = _oracle_inputs(name, n_rows, vslice, wl)
    secs = _oracle_run(d)
    cores = 1 if name == "nvfp4_quantize" else oracle.default_threads()
    return {"value": round(1e6 * secs * scale, 1), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": _oracle_sample_text(name, n_rows, vslice, secs), **host_cpu()}


def run_reference(args) -> dict | None:
    """The reference arm: the CPU oracle (this build has no installable reference; the pages hold
    no code) timed as cpu_baseline times it, each step one bounded sample of the workload."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", str(args.gpus)))
    if rank != 0:
        return None
    import oracle
    name = args.workload
    per_step_s = min(10.0, 90.0 / max(1, args.steps + args.warmup))
    n_rows, vslice, scale = _oracle_plan(name, per_step_s)
    d = _oracle_inputs(name, n_rows, vslice)
    for _ in range(args.warmup):
        _oracle_run(d)
    times = [_oracle_run(d) for _ in range(args.steps)]
    total = sum(times)
    us_per_call = 1e6 * (total / args.steps) * scale
    cores = 1 if name == "nvfp4_quantize" else oracle.default_threads()
    sample = "per step: " + _oracle_sample_text(name, n_rows, vslice, total / args.steps)
    return {
        "metric": METRIC, "value": round(us_per_call, 1), "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * total / args.steps, 3), "higher_is_better": False,
        "scaling": "strong" if name == "vocab_parallel_logprobs" else "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(name, world),
        "impl": "reference",
        "cpu_baseline": {"value": round(us_per_call, 1), "unit": UNIT, "cores": cores,
                         "kind": "oracle", "sample": sample, **host_cpu()},
        "e2e": {"value": round(us_per_call, 1), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="decode", choices=sorted(WORKLOAD_TEXT))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", action="store_true",
                    help="measure only --workload (the default run adds every other workload)")
    ap.add_argument("--traffic-from", metavar="DIR",
                    help="write profiles/traffic.json from the ncu launch lists DIR/<workload>.csv "
                         "and exit (no GPU needed)")
    args = ap.parse_args()
    if args.traffic_from:
        res = write_traffic(args.traffic_from)
        for kern, ents in res.items():
            if kern != "_about":
                for name, e in ents.items():
                    print(f"{name}: {kern}, {e['calls']} calls, bytes per call "
                          f"{e['bytes_per_launch']}")
        print("source_hash", kernel_source_hash())
        return
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    line = run_reference(args) if args.impl == "reference" else run_ours(args)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
