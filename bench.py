"""Benchmark of the LM-head library on B200: one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Workloads (seeded synthetic inputs from fp32_accumulate_lm_b200.synth; the pages use no dataset):
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
if _ROOT not in sys.path:
    sys.path.insert(0, _ROOT)

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
        from fp32_accumulate_lm_b200 import synth
        self.name = name
        rows_list, H, V, std, alpha = synth.WORKLOADS[name]
        self.rows_list, self.H, self.V, self.alpha = rows_list, H, V, alpha
        seed = {"decode": synth.SEED_DECODE, "spec_verify": synth.SEED_SPEC,
                "prefill": synth.SEED_PREFILL, "nvfp4": synth.SEED_NVFP4,
                "prefill_2048": synth.SEED_PREFILL, "decode_f16_bias": synth.SEED_F16,
                "nvfp4_quantize": synth.SEED_NVFP4, "prefill_logprobs": synth.SEED_PREFILL,
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
        self.logprobs = name in ("prefill_logprobs", "vocab_parallel_logprobs")
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


def run_ours(args) -> dict | None:
    import torch
    import fp32_accumulate_lm_b200 as lm

    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks = load_peaks()
    wl = Workload(args.workload, dev, world, rank)
    stream = torch.cuda.current_stream()
    rl = wl.rows_list
    calls_per_step = len(rl)

    for _ in range(args.warmup):
        for r in rl:
            wl.call(r)
    torch.cuda.synchronize()
    if lm.device_status(clear=True) != 0:
        raise RuntimeError("device status word set during warm-up")

    # ---- timed region: K steps, per-launch events on the launching stream
    n_ev = args.steps * calls_per_step
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev + 1)]
    sampler = ClockSampler(torch.cuda.current_device())
    barrier(world)
    sampler.start()
    ev[0].record(stream)
    i = 0
    for _ in range(args.steps):
        for r in rl:
            wl.call(r)
            i += 1
            ev[i].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    barrier(world)
    if lm.device_status(clear=True) != 0:
        raise RuntimeError("device status word set during the timed region")
    elapsed_ms = ev[0].elapsed_time(ev[n_ev])
    per_call_ms = [ev[j].elapsed_time(ev[j + 1]) for j in range(n_ev)]
    elapsed_ms = max_over_ranks(elapsed_ms, world)

    # per row count: mean launch duration, algorithmic bytes and flops
    detail = {}
    tot_bytes = tot_flops = tot_ms = 0.0
    for k, r in enumerate(rl):
        ms = per_call_ms[k::calls_per_step]
        mean_ms = sum(ms) / len(ms)
        b, fl = wl.bytes_of(r), wl.flops_of(r)
        detail[str(r)] = {"us": round(mean_ms * 1e3, 2), "us_min": round(min(ms) * 1e3, 2),
                          "GBps": round(b / (mean_ms * 1e-3) / 1e9, 1),
                          "TFLOPs": round(fl / (mean_ms * 1e-3) / 1e12, 1)}
        tot_bytes += b
        tot_flops += fl
        tot_ms += mean_ms
    # prefill, its profiling case, log-probs, vocab-parallel log-probs
    tensor_bound = args.workload.startswith("prefill") or wl.vocab_parallel
    if tensor_bound:
        achieved = tot_flops / (tot_ms * 1e-3) / 1e12
        peak = peaks["bf16_tflops_sustained"]
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4),
                "peak_kind": f"bf16 dense, sustained ({peaks['source']})"}
    else:
        achieved = tot_bytes / (tot_ms * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "peak_kind": f"HBM copy ({peaks['source']})"}
    roof["kernel"] = ("nvfp4_encode_kernel + nvfp4_absmax_kernel" if wl.quantize else
                      "lmhead_w4a16_nvfp4_kernel" if wl.nvfp4 else "lmhead_bf16_f32_kernel")
    roof["traffic"] = recorded_traffic(roof["kernel"], args.workload)
    roof["algorithmic_bytes_per_launch"] = int(tot_bytes / calls_per_step)
    roof["source_hash"] = kernel_source_hash()

    # ---- end to end through the C ABI: pinned host hidden -> device, call, logits -> pinned host
    e2e = run_e2e(args, wl, world)

    # Replicas: every rank makes whole calls. Vocab-parallel: the ranks make each call together.
    value = job_us_per_call(elapsed_ms, args.steps, calls_per_step,
                            1 if wl.vocab_parallel else world)
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(elapsed_ms / args.steps, 5), "higher_is_better": False,
        "scaling": "strong" if wl.vocab_parallel else "weak", "vs_baseline": None,
        "dtype": ("f32" if wl.quantize else "e2m1xbf16" if wl.nvfp4 else
                  "f16" if wl.dtype == torch.float16 else "bf16"),
        "data": "synthetic (seeded N(0,1) hidden, N(0,std) weights; no dataset on the pages)",
        "config": {"workload": WORKLOAD_TEXT[args.workload],
                   "l2": "weights 2x larger than L2 per call; two weight copies alternated",
                   "parallelism": (f"vocab-parallel x{world} (all-gather of the row stats)"
                                   if wl.vocab_parallel else
                                   f"replicas x{world} (no data-path collective)"),
                   "calls_per_step": calls_per_step, "per_rows": detail},
        "roofline": roof,
        "e2e": e2e,
        "gpu_launches": n_ev * (3 if wl.vocab_parallel else
                                2 if (wl.quantize or wl.logprobs) else 1),
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.workload, wl)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return line if rank == 0 else None


def run_e2e(args, wl, world: int) -> dict:
    """Same metric through the public call with host buffers: every call copies its hidden rows
    from pinned host memory and its logits back to pinned host memory inside the timed region."""
    import torch
    stream = torch.cuda.current_stream()
    rl = wl.rows_list
    h_host = {r: wl.hid[r].cpu().pin_memory() for r in rl}
    h_dev = {r: torch.empty_like(wl.hid[r]) for r in rl}
    o_host = {r: torch.empty(wl.outs[r].shape, dtype=wl.outs[r].dtype).pin_memory() for r in rl}
    steps = max(1, min(args.steps, 50))
    for _ in range(2):
        for r in rl:
            h_dev[r].copy_(h_host[r], non_blocking=True)
            wl.call(r, hidden=h_dev[r])
            o_host[r].copy_(wl.outs[r], non_blocking=True)
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        for r in rl:
            h_dev[r].copy_(h_host[r], non_blocking=True)
            wl.call(r, hidden=h_dev[r])
            o_host[r].copy_(wl.outs[r], non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    h2d = sum(h_host[r].numel() * h_host[r].element_size() for r in rl)
    d2h = sum(o_host[r].numel() * o_host[r].element_size() for r in rl)
    share = 1 if wl.vocab_parallel else world   # calls made together count once
    return {"value": round(ms * 1e3 / (steps * len(rl) * share), 3), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps}


# ---------------------------------------------------------------- CPU oracle (baseline arm)

_SAMPLES: dict = {}


def _oracle_sample(workload: str, rows: int, vocab_slice: int, wl=None):
    """Time the oracle on `rows` rows against the first `vocab_slice` weight rows; returns
    (seconds, multiply-adds done). Inputs are generated once and reused; only the oracle call is
    timed."""
    import oracle
    from fp32_accumulate_lm_b200 import synth
    rows_list, H, V, std, alpha = synth.WORKLOADS[workload]
    key = (workload, rows, vocab_slice)
    f16 = workload == "decode_f16_bias"
    if key not in _SAMPLES:
        import torch
        dt = torch.float16 if f16 else torch.bfloat16
        h = synth.hidden(rows, H, 7, dtype=dt)
        if workload == "nvfp4":
            _SAMPLES[key] = (h, synth.nvfp4_weights(vocab_slice, H, std, 7))
        else:
            _SAMPLES[key] = (h, (synth.weight(vocab_slice, H, std, 7, dtype=dt),
                                 synth.bias(vocab_slice, 7, dtype=dt) if f16 else None))
    h, w = _SAMPLES[key]
    t0 = time.perf_counter()
    if workload == "nvfp4":
        packed, scales, g = w
        oracle.logits_w4a16_nvfp4(h, packed, scales, g, alpha)
    else:
        oracle.logits_f32(h, w[0], alpha, bias_bits=w[1], dtype="f16" if f16 else "bf16")
    return time.perf_counter() - t0, rows * vocab_slice * H


def cpu_baseline(workload: str, wl) -> dict:
    """The oracle on the host cores, on the bench's own inputs: as many of the step's rows as fit
    in about 10 s (all of them for the decode workload), against the full vocabulary, scaled by
    rows to the step and reported per call."""
    import numpy as np
    import oracle
    import torch
    cores = oracle.default_threads()
    H, V = wl.H, wl.V
    if wl.quantize:  # the oracle quantiser is single-threaded: time a slice of W's rows
        w = wl.weights[0].view(torch.int16).cpu().numpy().view(np.uint16)
        n = 4096
        t0 = time.perf_counter()
        oracle.nvfp4_quantize(w[:n])
        secs = time.perf_counter() - t0
        return {"value": round(1e6 * secs * V / n, 1), "unit": UNIT, "cores": 1, "kind": "oracle",
                "sample": f"{n} of W's {V} rows x H={H} ({secs:.1f} s), scaled by rows"}
    rows_in_step = sum(wl.rows_list)
    h_all = wl.hidden.view(torch.int16).cpu().numpy().view(np.uint16)
    if wl.nvfp4:
        packed = wl.weights[0][0].cpu().numpy()
        scales = wl.weights[0][1].cpu().numpy()

        def run(h, vrows):
            oracle.logits_w4a16_nvfp4(h, packed[:vrows], scales[:vrows], wl.g, wl.alpha)
    else:
        w = wl.weights[0].view(torch.int16).cpu().numpy().view(np.uint16)
        b = None if wl.bias is None else wl.bias.view(torch.int16).cpu().numpy().view(np.uint16)
        dt = "f16" if wl.dtype == torch.float16 else "bf16"

        tg = wl.targets.cpu().numpy() if wl.logprobs else None

        def run(h, vrows):
            if wl.logprobs:
                oracle.logprobs_f32(h, w[:vrows], wl.alpha, np.minimum(tg[:h.shape[0]], vrows - 1),
                                    dtype=dt)
            else:
                oracle.logits_f32(h, w[:vrows], wl.alpha,
                                  bias_bits=None if b is None else b[:vrows], dtype=dt)
    probe_v = min(V, 4096)
    t0 = time.perf_counter()
    run(h_all[:1], probe_v)
    t_row = (time.perf_counter() - t0) * V / probe_v
    n_rows = int(max(1, min(rows_in_step, h_all.shape[0], 10.0 / max(t_row, 1e-9))))
    t0 = time.perf_counter()
    run(h_all[:n_rows], V)
    secs = time.perf_counter() - t0
    us_per_call = 1e6 * secs * (rows_in_step / n_rows) / len(wl.rows_list)
    return {"value": round(us_per_call, 1), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{n_rows} of the step's {rows_in_step} rows x full V={V} x H={H} "
                      f"({secs:.1f} s), scaled by rows to the step, per call"}


def _reference_quantize(args, H: int, V: int) -> dict:
    """The oracle quantiser as the reference arm: each step quantises a slice of W's rows, scaled
    by rows to one call."""
    import oracle
    from fp32_accumulate_lm_b200 import synth
    n = 2048
    w = synth.weight(n, H, 0.02, 7)
    for _ in range(args.warmup):
        oracle.nvfp4_quantize(w)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.nvfp4_quantize(w)
        times.append(time.perf_counter() - t0)
    total = sum(times)
    us = 1e6 * total / args.steps * V / n
    sample = f"per step: {n} of W's {V} rows x H={H}, scaled by rows to one call"
    return {
        "metric": METRIC, "value": round(us, 1), "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * total / args.steps, 3), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT[args.workload], "parallelism": "host core"},
        "impl": "reference",
        "cpu_baseline": {"value": round(us, 1), "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(us, 1), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def run_reference(args) -> dict | None:
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    import oracle
    from fp32_accumulate_lm_b200 import synth
    rows_list, H, V, std, alpha = synth.WORKLOADS[args.workload]
    cores = oracle.default_threads()
    if args.workload == "nvfp4_quantize":
        return _reference_quantize(args, H, V)
    mean_macs_per_call = sum(r * H * V for r in rows_list) / len(rows_list)
    # bounded per-step sample sized so warm-up + steps stay near a minute of CPU time
    vslice = 256
    t_probe, m_probe = _oracle_sample(args.workload, 1, vslice)
    budget_s = 60.0
    per_step_s = budget_s / max(1, args.steps + args.warmup)
    vslice = int(max(128, min(V, vslice * per_step_s / max(t_probe, 1e-6))))
    for _ in range(args.warmup):
        _oracle_sample(args.workload, 1, vslice)
    times = []
    macs = 0
    for _ in range(args.steps):
        s, m = _oracle_sample(args.workload, 1, vslice)
        times.append(s)
        macs = m
    total = sum(times)
    us_per_call = 1e6 * (total / (args.steps * macs)) * mean_macs_per_call
    sample = f"per step: 1 row x {vslice} vocab rows x H={H}, scaled by multiply-adds to the mean call"
    return {
        "metric": METRIC, "value": round(us_per_call, 1), "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * total / args.steps, 3), "higher_is_better": False,
        "scaling": "strong" if args.workload == "vocab_parallel_logprobs" else "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT[args.workload], "parallelism": "host cores"},
        "impl": "reference",
        "cpu_baseline": {"value": round(us_per_call, 1), "unit": UNIT, "cores": cores,
                         "kind": "oracle", "sample": sample},
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
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    line = run_reference(args) if args.impl == "reference" else run_ours(args)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
