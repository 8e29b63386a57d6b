"""The exchange of the vocab-parallel log-probabilities on CPU: two and three gloo ranks each hold
one vocab slice (vocab_shard), compute that slice's stats (here with the oracle, standing in for
the GPU half), and gather_shard_stats brings every rank the stats of all slices in rank order,
from which the merge gives the log-softmax of the whole row. The GPU halves are covered by
test_vocab_parallel.py on one device."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    rng = np.random.default_rng(106)
    rows, H, V = 7, 64, 1001
    h = rng.normal(0, 1, (rows, H)).astype(np.float32)
    w = rng.normal(0, 0.3, (V, H)).astype(np.float32)
    to_bits = lambda x: (x.view(np.uint32) >> 16).astype(np.uint16)  # exact: truncation to bf16
    t = np.array([0, 333, 334, 500, 667, 1000, 1001], np.int32)      # last one held by no slice
    return to_bits(h), to_bits(w), t


def _rank_main(rank: int, world: int, port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch
    import torch.distributed as dist
    import oracle
    import fp32_accumulate_lm_b200 as lm
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        h, w, t = _inputs()
        V = w.shape[0]
        b, n = lm.vocab_shard(V, world, rank)
        mine = oracle.logprob_shard_stats(h, w[b:b + n], b, 0.5, t)
        got = lm.gather_shard_stats(torch.from_numpy(mine)).numpy()
        want = np.stack([oracle.logprob_shard_stats(h, w[bb:bb + nn], bb, 0.5, t)
                         for bb, nn in (lm.vocab_shard(V, world, r) for r in range(world))])
        same = bool(np.array_equal(got, want, equal_nan=True))
        lp, lse = oracle.logprob_merge_shards(got)
        lp1, lse1 = oracle.logprobs_f32(h, w, 0.5, t)
        q.put((rank, same, lp.tolist(), lse.tolist(), lp1.tolist(), lse1.tolist()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gathered_stats_merge_to_the_whole_row(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=5) for _ in range(world))
    for rank, same, lp, lse, lp1, lse1 in res:
        assert same, rank                     # rank r's slot holds slice r's stats
        lp, lse, lp1, lse1 = map(np.array, (lp, lse, lp1, lse1))
        # the merged double sums round to the same fp32 as the whole-row oracle, up to one ulp
        assert np.allclose(lse, lse1, rtol=2.4e-7, atol=0)
        assert np.allclose(lp[:-1], lp1[:-1], rtol=2.4e-7, atol=1e-7)
        assert np.isnan(lp[-1]) and np.isnan(lp1[-1])
    # every rank ends with the same result
    assert all(np.array_equal(np.array(r[2]), np.array(res[0][2]), equal_nan=True) for r in res)
