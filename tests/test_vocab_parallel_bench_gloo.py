"""bench.py's whole-job figure for the vocab-parallel workload, on CPU with two gloo ranks: the
ranks make each call together, so the job's time per call is the slowest rank's time over the
calls (not over calls x ranks, as for replicas), and each rank's slice is the one vocab_shard
gives."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_vocab_parallel_counts_each_call_once():
    sys.path.insert(0, ROOT)
    import bench
    # 2 ranks, slowest 107 ms over 10 steps of 1 call: 10.7 ms per call for the job
    assert bench.job_us_per_call(107.0, steps=10, calls_per_step=1, world=1) == pytest.approx(
        10.7e3)
    # the replicas' figure for the same elapsed time divides by the ranks as well
    assert bench.job_us_per_call(107.0, steps=10, calls_per_step=1, world=2) == pytest.approx(
        5.35e3)


def test_gather_without_a_process_group_is_the_identity():
    sys.path.insert(0, ROOT)
    import torch
    import fp32_accumulate_lm_b200 as lm
    s = torch.arange(12, dtype=torch.float32).view(4, 3)
    g = lm.gather_shard_stats(s)
    assert tuple(g.shape) == (1, 4, 3) and torch.equal(g[0], s)
