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
