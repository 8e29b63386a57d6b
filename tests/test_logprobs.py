"""GPU parity of lmhead_logprobs_f32: log-probabilities of given tokens over the fp32 logits,
computed in the head's epilogue without writing the logits.

    lse[r] = log sum_v exp(z[r, v]),  logprob[r] = z[r, t_r] - lse[r]
(the first page's "Purpose": fp32 logits for RL training-inference consistency and for the
rejection sampling of speculative decoding.)

Two checks per case:
  * against the fused path's own logits: lmhead_logits_f32 gives z bit for bit, and numpy's
    float64 log-sum-exp of that z bounds the reduction and combine error tightly;
  * against the CPU oracle end to end: the logits differ from the oracle's by at most the fp32
    bound of tolerance.fp32_bound per element, and since d logprob / d z_v sums to at most 2 in
    absolute value, |gpu - oracle| <= 2 * max_v bound_v + the reduction bound.
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


def reduction_bound(lse: np.ndarray, V: int) -> np.ndarray:
    """Worst case of the fused reduction: a row's sum is built by at most 5 merges inside a
    32-entry chunk (the epilogue's lane steps), ceil(n_chunks / 32) in order within a segment
    and 32 across segments (the combine), n_chunks = 4 * ceil(V / 128); each merge adds at most
    one rounding of the running sum (2^-24 relative, doubled for its exp), so
    |d lse| <= (n + 37) * 2^-23; plus the rounding of lse itself and of the final subtraction."""
    n_chunks = 4 * (-(-V // 128))
    n = -(-n_chunks // 32)
    return (n + 37) * 2.0 ** -23 + 4e-7 * np.abs(lse) + 1e-6


def case(rows, H, V, seed, dtype="bf16", with_bias=False, std=0.02):
    h = synth.hidden(rows, H, seed, dtype=TDT[dtype])
    w = synth.weight(V, H, std, seed, dtype=TDT[dtype])
    b = synth.bias(V, seed, dtype=TDT[dtype]) if with_bias else None
    t = np.random.default_rng(seed).integers(0, V, rows).astype(np.int32)
    return h, w, b, t


def run(h, w, b, t, alpha, dtype):
    hd = synth.bits_to_torch(h, TDT[dtype], "cuda")
    wd = synth.bits_to_torch(w, TDT[dtype], "cuda")
    bd = None if b is None else synth.bits_to_torch(b, TDT[dtype], "cuda")
    td = torch.from_numpy(t).cuda()
    lp, lse = lm.logprobs_f32(hd, wd, td, alpha, bias=bd)
    z = lm.logits_f32(hd, wd, alpha, bias=bd)
    check_status()
    return lp.cpu().numpy(), lse.cpu().numpy(), z.cpu().numpy()


@pytest.mark.parametrize("dtype,with_bias", [("bf16", False), ("bf16", True), ("f16", True)])
def test_matches_own_logits_and_oracle(dtype, with_bias):
    for rows, H, V, seed in [(4, 256, 1024, 1), (1, 64, 1, 2), (17, 136, 129, 3),
                             (65, 320, 300, 4), (3, 2048, 151936, 5)]:
        h, w, b, t = case(rows, H, V, seed, dtype, with_bias, std=0.05)
        for alpha in (1.0 / 8, 0.7):
            lp, lse, z = run(h, w, b, t, alpha, dtype)
            want_lse = lse64(z)
            assert np.all(np.abs(lse - want_lse) <= reduction_bound(want_lse, V)), (rows, V, alpha)
            want_lp = z[np.arange(rows), t].astype(np.float64) - want_lse
            assert np.all(np.abs(lp - want_lp) <= reduction_bound(want_lse, V)), (rows, V, alpha)
            ref_lp, ref_lse = oracle.logprobs_f32(h, w, alpha, t, bias_bits=b, dtype=dtype)
            _, absum = oracle.logits_f32(h, w, alpha, bias_bits=b, dtype=dtype)
            tol = 2 * fp32_bound(absum).max(axis=1) + reduction_bound(ref_lse, V)
            assert np.all(np.abs(lp - ref_lp) <= tol), (rows, V, alpha)
            assert np.all(np.abs(lse - ref_lse) <= tol), (rows, V, alpha)


def test_targets_at_the_edges_and_out_of_range():
    rows, H, V = 6, 128, 300          # last v-tile holds 44 entries
    h, w, b, _ = case(rows, H, V, 11)
    t = np.array([0, 127, 128, 255, 299, V], np.int32)
    lp, lse, z = run(h, w, None, t, 0.125, "bf16")
    want_lse = lse64(z)
    for r in range(5):
        assert abs(lp[r] - (z[r, t[r]] - want_lse[r])) <= reduction_bound(want_lse[r:r + 1], V)[0]
    assert np.isnan(lp[5]) and np.isfinite(lse[5])
    t2 = np.array([-1, 0, 0, 0, 0, 2 ** 31 - 1], np.int32)
    lp2, lse2, _ = run(h, w, None, t2, 0.125, "bf16")
    assert np.isnan(lp2[0]) and np.isnan(lp2[5])
    assert np.array_equal(lse2, lse)                       # lse does not depend on the targets
    for r in range(1, 5):
        assert abs(lp2[r] - (z[r, 0] - want_lse[r])) <= reduction_bound(want_lse[r:r + 1], V)[0]


def test_rows_are_independent_of_the_row_count_and_deterministic():
    rows, H, V = 300, 1024, 40000
    h, w, b, t = case(rows, H, V, 21, "bf16", True, std=0.05)
    hd = synth.bits_to_torch(h, torch.bfloat16, "cuda")
    wd = synth.bits_to_torch(w, torch.bfloat16, "cuda")
    bd = synth.bits_to_torch(b, torch.bfloat16, "cuda")
    td = torch.from_numpy(t).cuda()
    lp, lse = lm.logprobs_f32(hd, wd, td, 0.25, bias=bd)
    lp2, lse2 = lm.logprobs_f32(hd, wd, td, 0.25, bias=bd)
    assert torch.equal(lp, lp2) and torch.equal(lse, lse2)
    for r in (1, 2, 17, 64, 65, 256):
        a, l = lm.logprobs_f32(hd[:r].contiguous(), wd, td[:r].contiguous(), 0.25, bias=bd)
        assert torch.equal(a, lp[:r]) and torch.equal(l, lse[:r]), r
    check_status()


def test_prefill_shape_sampled_rows_against_oracle():
    """8192 x 4096 x 151936 (the prefill workload's shape): 3 sampled rows against the oracle."""
    rows_list, H, V, std, alpha = synth.WORKLOADS["prefill"]
    R = rows_list[0]
    hd = synth.hidden(R, H, synth.SEED_PREFILL, device="cuda")
    wd = synth.weight(V, H, std, synth.SEED_PREFILL, device="cuda")
    t = np.random.default_rng(31).integers(0, V, R).astype(np.int32)
    lp, lse = lm.logprobs_f32(hd, wd, torch.from_numpy(t).cuda(), alpha)
    check_status()
    sample = [0, 4097, 8191]
    h = hd[sample].view(torch.int16).cpu().numpy().view(np.uint16)
    w = wd.view(torch.int16).cpu().numpy().view(np.uint16)
    ref_lp, ref_lse = oracle.logprobs_f32(h, w, alpha, t[sample])
    _, absum = oracle.logits_f32(h, w, alpha)
    tol = 2 * fp32_bound(absum).max(axis=1) + reduction_bound(ref_lse, V)
    got_lp = lp.cpu().numpy()[sample]
    got_lse = lse.cpu().numpy()[sample]
    assert np.all(np.abs(got_lp - ref_lp) <= tol) and np.all(np.abs(got_lse - ref_lse) <= tol)
