"""The multi-process plumbing of bench.py on CPU: two gloo ranks run its barrier, its max over
ranks and its whole-job per-call figure, exactly as the GPU replicas do under torchrun."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup(world, backend="gloo")
    try:
        bench.barrier(w)
        elapsed = 100.0 + 7.0 * r          # rank 1 is the slow one
        worst = bench.max_over_ranks(elapsed, w)
        value = bench.job_us_per_call(worst, steps=10, calls_per_step=7, world=w)
        bench.barrier(w)
        q.put((r, w, worst, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_rank():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=5) for _ in range(world))
    assert [g[0] for g in got] == [0, 1]
    for _, w, worst, value in got:
        assert w == world
        assert worst == 107.0
        # 107 ms over 2 ranks x 10 steps x 7 calls
        assert value == pytest.approx(107.0e3 / 140.0)


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_us_per_call(2.0, steps=4, calls_per_step=5, world=1) == pytest.approx(100.0)
    bench.barrier(1)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")

    class Args:
        workload, steps, warmup, gpus = "decode", 3, 3, 2
    assert bench.run_reference(Args()) is None


def test_reference_arm_line_and_config_match_the_repo_arm(monkeypatch):
    """The reference arm (the CPU oracle) on a shrunken decode workload: the contract's keys,
    impl "reference", and the same config dict as the repo arm's line for the same N, so the two
    lines describe the same workload."""
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import bench
    import synth
    monkeypatch.setitem(synth.WORKLOADS, "decode", ([1, 2, 4], 256, 1024, 0.02, 1.0 / 8))
    monkeypatch.delenv("RANK", raising=False)
    monkeypatch.delenv("WORLD_SIZE", raising=False)

    class Args:
        workload, steps, warmup, gpus = "decode", 3, 3, 1
    line = bench.run_reference(Args())
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "us/call"
    assert line["config"] == bench.config_of("decode", 1)
    assert line["config"]["rows_per_call"] == [1, 2, 4]
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": "us/call", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    # the plan times the step's distinct rows (4 here) against the whole small vocabulary
    n_rows, vslice, scale = bench._oracle_plan("decode", 1.0)
    assert n_rows == 4 and vslice == 1024 and scale == pytest.approx((1 + 2 + 4) / 4 / 3)
