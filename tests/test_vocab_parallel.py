"""GPU parity of the vocab-parallel log-probabilities (lmhead_logprobs_shard_stats_f32, then
lmhead_logprobs_merge_shards): every vocab slice runs on this one device in turn, as the g GPUs of
a split would, and their stats are stacked in slice order -- the array the all-gather delivers.

"FP32 LM head skip FP32 cast" (key source excerpt, _compute_lm_head) takes the head as a
VocabParallelEmbedding; the log-softmax is over the whole row:
    lse[r] = log sum_v exp(z[r, v]),  logprob[r] = z[r, t_r] - lse[r].
Checks: a slice's max and target logit are those of lmhead_logits_f32 on the slice, bit for bit
(one accumulator chain per logit, whichever call computes it); one slice is the one-GPU entry bit
for bit; any split agrees with numpy's float64 log-sum-exp of the whole row's logits within the
fused reduction's bound plus one rounding per merged slice, and with the CPU oracle within the
logits' fp32 bound on top of that.
"""
import numpy as np
import pytest
import torch

import oracle
import fp32_accumulate_lm_b200 as lm
import synth
from gpu_helpers import check_status
from tolerance import fp32_bound

pytestmark = pytest.mark.gpu

TDT = {"bf16": torch.bfloat16, "f16": torch.float16}


def lse64(z: np.ndarray) -> np.ndarray:
    z = z.astype(np.float64)
    m = z.max(axis=1, keepdims=True)
    return (m + np.log(np.exp(z - m).sum(axis=1, keepdims=True)))[:, 0]


def merged_bound(lse: np.ndarray, V_shard_max: int, shards: int) -> np.ndarray:
    """The one-GPU reduction's bound for the largest slice, (n + 37) * 2^-23 with n =
    ceil(n_chunks / 32) and n_chunks = 4 * ceil(V / 128), plus 2^-23 for each slice merged in
    (one rounding of the running sum and one of its exp), plus the roundings of lse and of the
    final subtraction."""
    n = -(-(4 * (-(-V_shard_max // 128))) // 32)
    return (n + 37 + shards) * 2.0 ** -23 + 4e-7 * np.abs(lse) + 1e-6


def slices(V, g):
    return [lm.vocab_shard(V, g, r) for r in range(g)]


def make(rows, H, V, seed, dtype="bf16", with_bias=False, std=0.05):
    h = synth.hidden(rows, H, seed, dtype=TDT[dtype])
    w = synth.weight(V, H, std, seed, dtype=TDT[dtype])
    b = synth.bias(V, seed, dtype=TDT[dtype]) if with_bias else None
    t = np.random.default_rng(seed).integers(0, V, rows).astype(np.int32)
    dev = lambda x: None if x is None else synth.bits_to_torch(x, TDT[dtype], "cuda")
    return (h, w, b, t), (dev(h), dev(w), dev(b), torch.from_numpy(t).cuda())


def split_run(hd, wd, bd, td, alpha, g):
    stats = torch.stack([
        lm.logprobs_shard_stats_f32(hd, wd[b0:b0 + n], b0, td, alpha,
                                    None if bd is None else bd[b0:b0 + n])
        for b0, n in slices(wd.shape[0], g)])
    lp, lse = lm.logprobs_merge_shards(stats.contiguous())
    check_status()
    return stats.cpu().numpy(), lp.cpu().numpy(), lse.cpu().numpy()


@pytest.mark.parametrize("dtype,with_bias", [("bf16", False), ("bf16", True), ("f16", True)])
def test_slice_stats_are_the_slice_logits(dtype, with_bias):
    rows, H, V = 37, 256, 1000
    _, (hd, wd, bd, td) = make(rows, H, V, 41, dtype, with_bias)
    t = td.cpu().numpy()
    stats, _, _ = split_run(hd, wd, bd, td, 0.7, 3)
    for i, (b0, n) in enumerate(slices(V, 3)):
        z = lm.logits_f32(hd, wd[b0:b0 + n].contiguous(), 0.7,
                          bias=None if bd is None else bd[b0:b0 + n].contiguous()).cpu().numpy()
        m, s, zt = stats[i, :, 0], stats[i, :, 1], stats[i, :, 2]
        assert np.array_equal(m, z.max(axis=1)), i
        held = (t >= b0) & (t < b0 + n)
        assert np.array_equal(zt[held], z[np.nonzero(held)[0], t[held] - b0]), i
        assert np.isnan(zt[~held]).all(), i
        s64 = np.exp(z.astype(np.float64) - m[:, None].astype(np.float64)).sum(axis=1)
        nb = -(-(4 * (-(-n // 128))) // 32)
        assert np.all(np.abs(s - s64) <= (nb + 37) * 2.0 ** -23 * s64), i


@pytest.mark.parametrize("dtype,with_bias", [("bf16", False), ("bf16", True), ("f16", False)])
def test_one_slice_is_the_one_gpu_entry_bit_for_bit(dtype, with_bias):
    for rows, H, V, seed in [(4, 256, 1024, 42), (65, 320, 300, 43), (3, 2048, 151936, 44)]:
        _, (hd, wd, bd, td) = make(rows, H, V, seed, dtype, with_bias)
        _, lp, lse = split_run(hd, wd, bd, td, 0.125, 1)
        lp1, lse1 = lm.logprobs_f32(hd, wd, td, 0.125, bias=bd)
        assert np.array_equal(lp, lp1.cpu().numpy()) and np.array_equal(lse, lse1.cpu().numpy())


@pytest.mark.parametrize("g", [2, 3, 8])
def test_splits_match_the_whole_row_and_the_oracle(g):
    for rows, H, V, seed, with_bias in [(17, 136, 1001, 45, True), (64, 512, 40000, 46, False)]:
        (h, w, b, t), (hd, wd, bd, td) = make(rows, H, V, seed, "bf16", with_bias)
        stats, lp, lse = split_run(hd, wd, bd, td, 0.25, g)
        z = lm.logits_f32(hd, wd, 0.25, bias=bd).cpu().numpy()
        want_lse = lse64(z)
        vmax = max(n for _, n in slices(V, g))
        bound = merged_bound(want_lse, vmax, g)
        assert np.all(np.abs(lse - want_lse) <= bound), (g, V)
        want_lp = z[np.arange(rows), t].astype(np.float64) - want_lse
        assert np.all(np.abs(lp - want_lp) <= bound), (g, V)
        ref_lp, ref_lse = oracle.logprobs_f32(h, w, 0.25, t, bias_bits=b)
        _, absum = oracle.logits_f32(h, w, 0.25, bias_bits=b)
        tol = 2 * fp32_bound(absum).max(axis=1) + merged_bound(ref_lse, vmax, g)
        assert np.all(np.abs(lp - ref_lp) <= tol) and np.all(np.abs(lse - ref_lse) <= tol), (g, V)
        # the same split again gives the same bits
        _, lp2, lse2 = split_run(hd, wd, bd, td, 0.25, g)
        assert np.array_equal(lp, lp2) and np.array_equal(lse, lse2)


def test_targets_on_slice_edges_and_outside():
    rows, H, V = 8, 128, 300                      # three slices of 100
    _, (hd, wd, _, _) = make(rows, H, V, 47)
    t = np.array([0, 99, 100, 199, 200, 299, 300, -1], np.int32)
    stats, lp, lse = split_run(hd, wd, None, torch.from_numpy(t).cuda(), 0.125, 3)
    z = lm.logits_f32(hd, wd, 0.125).cpu().numpy()
    want_lse = lse64(z)
    bound = merged_bound(want_lse, 100, 3)
    for r in range(6):
        assert abs(lp[r] - (z[r, t[r]] - want_lse[r])) <= bound[r], r
        holder = t[r] // 100
        assert [not np.isnan(stats[i, r, 2]) for i in range(3)] == [i == holder for i in range(3)]
    assert np.isnan(lp[6]) and np.isnan(lp[7]) and np.isfinite(lse).all()
    assert np.isnan(stats[:, 6:, 2]).all()


def test_decode_shape_in_eight_slices_against_the_oracle():
    """H = 2048, V = 151936 (the decode head) in eight slices of 18992: 4 rows against the
    oracle."""
    rows, H, V = 4, 2048, 151936
    (h, w, b, t), (hd, wd, bd, td) = make(rows, H, V, 48, std=0.02)
    _, lp, lse = split_run(hd, wd, None, td, 1.0 / 8, 8)
    ref_lp, ref_lse = oracle.logprobs_f32(h, w, 1.0 / 8, t)
    _, absum = oracle.logits_f32(h, w, 1.0 / 8)
    tol = 2 * fp32_bound(absum).max(axis=1) + merged_bound(ref_lse, 18992, 8)
    assert np.all(np.abs(lp - ref_lp) <= tol) and np.all(np.abs(lse - ref_lse) <= tol)


def test_through_a_one_rank_nccl_group():
    """logprobs_vocab_parallel end to end (slice stats, NCCL all-gather, merge) in a process
    group of one rank: the all-gather is the identity and the result is the one-GPU entry's."""
    import socket
    from datetime import timedelta
    import torch.distributed as dist
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        _, (hd, wd, bd, td) = make(33, 512, 5000, 49, "bf16", True)
        b0, n = lm.vocab_shard(5000, 1, 0)
        lp, lse = lm.logprobs_vocab_parallel(hd, wd[b0:b0 + n], b0, td, 0.5, bd[b0:b0 + n])
        torch.cuda.synchronize()
        lp1, lse1 = lm.logprobs_f32(hd, wd, td, 0.5, bias=bd)
        assert torch.equal(lp, lp1) and torch.equal(lse, lse1)
        check_status()
    finally:
        dist.destroy_process_group()


def test_rows_past_the_first_row_tile():
    """300 rows span two 256-row tiles: every row's slice max and target logit are the slice
    logits' bits, and the merged result agrees with the one-GPU entry."""
    rows, H, V = 300, 256, 5000
    _, (hd, wd, bd, td) = make(rows, H, V, 50, "bf16", True)
    t = td.cpu().numpy()
    stats, lp, lse = split_run(hd, wd, bd, td, 0.5, 3)
    for i, (b0, n) in enumerate(slices(V, 3)):
        z = lm.logits_f32(hd, wd[b0:b0 + n].contiguous(), 0.5,
                          bias=bd[b0:b0 + n].contiguous()).cpu().numpy()
        assert np.array_equal(stats[i, :, 0], z.max(axis=1)), i
        held = (t >= b0) & (t < b0 + n)
        assert np.array_equal(stats[i, held, 2], z[np.nonzero(held)[0], t[held] - b0]), i
        assert np.isnan(stats[i, ~held, 2]).all(), i
    lp1, lse1 = lm.logprobs_f32(hd, wd, td, 0.5, bias=bd)
    bound = 2 * merged_bound(lse1.cpu().numpy().astype(np.float64), 1667, 3)
    assert np.all(np.abs(lp - lp1.cpu().numpy()) <= bound)
    assert np.all(np.abs(lse - lse1.cpu().numpy()) <= bound)


# ---------------------------------------------------------------- vocab-parallel logits

@pytest.mark.parametrize("rows,g,dtype,with_bias", [(5, 1, "bf16", False), (5, 3, "bf16", True),
                                                    (300, 4, "bf16", True), (37, 2, "f16", True),
                                                    (513, 8, "bf16", False)])
def test_slice_logits_written_into_every_buffer_make_the_whole_head(rows, g, dtype, with_bias):
    """Each vocab slice's call (one per GPU of a g-way split, here run in turn on one device)
    stores its columns into every buffer; the buffers, local here, stand for the g GPUs'
    buffers, which the kernel addresses the same way. Afterwards every buffer holds the whole
    head's logits bit for bit (lmhead_logits_f32 on all of W), and nothing outside its [rows, V]
    block was written (NaN canaries in extra rows and in columns past V)."""
    H, V = 192, 1111
    (h, w, b, _), (hd, wd, bd, _) = make(rows, H, V, 60 + g, dtype, with_bias)
    alpha = 0.3
    ld = V + 13
    bufs = [torch.full((rows + 3, ld), float("nan"), dtype=torch.float32, device="cuda")
            for _ in range(min(g, 3))]
    for b0, n in slices(V, g):
        lm.logits_vocab_slice_f32(hd, wd[b0:b0 + n].contiguous(), b0, bufs, alpha,
                                  bias_slice=None if bd is None else bd[b0:b0 + n].contiguous())
    whole = lm.logits_f32(hd, wd, alpha, bias=bd)
    check_status()
    want = whole.cpu().numpy().view(np.uint32)
    for buf in bufs:
        got = buf.cpu().numpy()
        assert np.array_equal(got[:rows, :V].view(np.uint32), want)
        assert np.isnan(got[:rows, V:]).all() and np.isnan(got[rows:]).all()


def test_vocab_parallel_logits_single_rank_and_oracle():
    """VocabParallelLogits without a process group (one rank holds the whole vocabulary): the
    one-GPU logits, and on sampled rows the CPU oracle within the fp32 bound."""
    from tolerance import assert_fp32_close
    rows, H, V = 260, 256, 3000
    (h, w, b, _), (hd, wd, bd, _) = make(rows, H, V, 71, "bf16", True)
    head = lm.VocabParallelLogits(max_rows=512, V=V)
    assert (head.v_begin, head.V_shard) == (0, V)
    got = head(hd, wd, 0.25, bias_shard=bd)
    assert tuple(got.shape) == (rows, V)
    whole = lm.logits_f32(hd, wd, 0.25, bias=bd)
    check_status()
    assert torch.equal(got.view(torch.int32), whole.view(torch.int32))
    sample = np.array([0, 1, 128, 255, 256, 259])
    ref, absum = oracle.logits_f32(h[sample], w, 0.25, bias_bits=b)
    assert_fp32_close(got.cpu().numpy()[sample], ref, absum, "vocab-parallel logits")


def test_vocab_parallel_logits_on_symmetric_memory_in_a_one_rank_group():
    """VocabParallelLogits forced onto torch's symmetric memory in a one-rank NCCL group: the
    rendezvous, the mapping of every rank's buffer and the two barriers around each call run for
    real, and the buffer holds the one-GPU entry's bits for two calls of different row counts."""
    import socket
    from datetime import timedelta
    import torch.distributed as dist
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        _, (hd, wd, bd, _) = make(300, 256, 3000, 72, "bf16", True)
        head = lm.VocabParallelLogits(max_rows=512, V=3000, symmetric=True)
        assert head._handle is not None and head.world == 1
        for rows in (300, 5):
            h = hd[:rows].contiguous()
            got = head(h, wd, 0.25, bias_shard=bd).clone()
            want = lm.logits_f32(h, wd, 0.25, bias=bd)
            check_status()
            assert torch.equal(got.view(torch.int32), want.view(torch.int32)), rows
        del head
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("rows,H", [(64, 2048), (300, 4096)])
def test_slice_logits_at_the_bench_shapes(rows, H):
    """The decode shape (64 rows, H = 2048) and a CTA-pair shape (300 rows, H = 4096) at
    V = 151936, split 8 ways into two buffers: every buffer is the whole head's logits bit for
    bit, and sampled rows agree with the CPU oracle."""
    from tolerance import assert_fp32_close
    V, g = 151936, 8
    (h, w, _, _), (hd, wd, _, _) = make(rows, H, V, 80 + rows, "bf16", False, std=0.02)
    alpha = 0.125
    bufs = [torch.empty((rows, V), dtype=torch.float32, device="cuda") for _ in range(2)]
    for b0, n in slices(V, g):
        lm.logits_vocab_slice_f32(hd, wd[b0:b0 + n], b0, bufs, alpha)
    whole = lm.logits_f32(hd, wd, alpha)
    check_status()
    for buf in bufs:
        assert torch.equal(buf.view(torch.int32), whole.view(torch.int32))
    sample = np.array([0, rows // 2, rows - 1])
    ref, absum = oracle.logits_bf16_f32(h[sample], w, alpha)
    assert_fp32_close(bufs[1].cpu().numpy()[sample], ref, absum, "slice logits, bench shape")
