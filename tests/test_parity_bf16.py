"""GPU parity of the fp32-accumulate head (entry 1) against the CPU oracle, through the C ABI.

    logits = fl32(alpha * hidden @ W^T), bf16 operands, fp32 accumulation
("[Model] Honor fp32 head_dtype in Inkling muP logits (target + MTP draft)", "Purpose" and
"muP is folded into the fp32 GEMM"; "FP32 LM head skip FP32 cast", implementation breakdown).

Floating-point results are compared element by element within the bound in tolerance.py;
cases where every summation order is exact (small integers, one-hot rows, zero and identity
weights) are compared bit for bit, as are the properties the method promises exactly: the
alpha fold equals a separate fp32 multiply, and a row's logits are the same whatever the number
of rows in the call (lm_head_nvfp4_rows.rs, module doc).
"""
import numpy as np
import pytest
import torch

import oracle
import fp32_accumulate_lm_b200 as lm
import synth
from gpu_helpers import bf16_bits_of_f32, check_status, dev_bf16, f32_bits, gpu_bf16_f32
from tolerance import assert_fp32_close

pytestmark = pytest.mark.gpu


# ---------------------------------------------------------------- tiny workload (4 x 256 x 1024)

def test_tiny_matches_oracle_and_rows_are_invariant():
    rows_list, H, V, std, alpha = synth.WORKLOADS["tiny"]
    h = synth.hidden(4, H, synth.SEED_TINY)
    w = synth.weight(V, H, std, synth.SEED_TINY)
    ref, absum = oracle.logits_bf16_f32(h, w, alpha)
    got = gpu_bf16_f32(h, w, alpha)
    assert_fp32_close(got, ref, absum, "tiny")
    for r in (1, 2, 3):
        sub = gpu_bf16_f32(h[:r], w, alpha)
        assert np.array_equal(f32_bits(sub), f32_bits(got[:r])), r


def test_one_hot_rows_are_exact():
    H, V = 256, 1024
    w = synth.weight(V, H, 0.02, synth.SEED_TINY)
    ks = [0, 1, 15, 16, 63, 64, 200, 255]
    h = np.zeros((len(ks), H), np.float32)
    for i, k in enumerate(ks):
        h[i, k] = 1.0
    for alpha in (0.25, 1.0 / 3.0):
        ref, _ = oracle.logits_bf16_f32(bf16_bits_of_f32(h), w, alpha)
        got = gpu_bf16_f32(bf16_bits_of_f32(h), w, alpha)
        assert np.array_equal(f32_bits(got), f32_bits(ref))


@pytest.mark.parametrize("rows,H,V", [(37, 200, 300), (1, 8, 1), (16, 64, 128), (17, 72, 129),
                                      (256, 136, 257), (257, 64, 130), (5, 1000, 515)])
def test_integer_inputs_bit_exact_on_ragged_shapes(rows, H, V):
    """Small integers keep every partial sum exact in fp32, so any summation order gives the
    oracle's bits. Ragged rows / H / V cover the zero-filled tile edges."""
    rng = np.random.default_rng(rows * 1000 + H + V)
    hi = rng.integers(-6, 7, (rows, H)).astype(np.float32)
    wi = rng.integers(-6, 7, (V, H)).astype(np.float32)
    hb, wb = bf16_bits_of_f32(hi), bf16_bits_of_f32(wi)
    ref, _ = oracle.logits_bf16_f32(hb, wb, 1.0)
    got = gpu_bf16_f32(hb, wb, 1.0)
    assert np.array_equal(f32_bits(got), f32_bits(ref))
    got2 = gpu_bf16_f32(hb, wb, 0.5)
    assert np.array_equal(f32_bits(got2), f32_bits((ref * np.float32(0.5)).astype(np.float32)))


def test_zero_and_identity_block_weights():
    rows, H, V = 9, 128, 300
    h = synth.hidden(rows, H, 5)
    got = gpu_bf16_f32(h, np.zeros((V, H), np.uint16), 0.125)
    assert np.all(got == 0) and not np.any(np.signbit(got))
    eye = np.zeros((V, H), np.float32)
    eye[np.arange(H), np.arange(H)] = 1.0
    got = gpu_bf16_f32(h, bf16_bits_of_f32(eye), 0.125)
    want = (synth.bf16_bits_to_f32(h) * np.float32(0.125)).astype(np.float32)
    assert np.array_equal(f32_bits(got[:, :H]), f32_bits(want))
    assert np.all(got[:, H:] == 0)


def test_alpha_fold_equals_separate_fp32_multiply():
    """Page 1: folding alpha into the GEMM is bit-identical to the projection followed by an
    fp32 multiply. Non-power-of-two alphas make the check non-trivial."""
    rows, H, V = 33, 512, 1000
    h = synth.hidden(rows, H, 11)
    w = synth.weight(V, H, 0.02, 11)
    base = gpu_bf16_f32(h, w, 1.0)
    for alpha in (1.0 / 3.0, 1.0 / 6.0, 0.7, 1.0 / 8.0, -0.5, 1e-30):
        fused = gpu_bf16_f32(h, w, alpha)
        with np.errstate(under="ignore"):
            sep = (base * np.float32(alpha)).astype(np.float32)
        assert np.array_equal(f32_bits(fused), f32_bits(sep)), alpha


def test_tiny_magnitudes_match_oracle():
    """Values near the bottom of the fp32 range (no flush to zero in the epilogue)."""
    rows, H, V = 4, 64, 256
    h = (synth.bf16_bits_to_f32(synth.hidden(rows, H, 3)) * np.float32(2.0 ** -60)).astype(np.float32)
    w = (synth.bf16_bits_to_f32(synth.weight(V, H, 1.0, 3)) * np.float32(2.0 ** -60)).astype(np.float32)
    hb, wb = bf16_bits_of_f32(h), bf16_bits_of_f32(w)
    ref, absum = oracle.logits_bf16_f32(hb, wb, 0.25)
    got = gpu_bf16_f32(hb, wb, 0.25)
    assert_fp32_close(got, ref, absum, "tiny magnitudes")


def test_row_count_and_position_invariance():
    """A row's logits are the same bits at every row count (1..513 crosses the 16-row padding
    steps and the 256-row tiles) and at every position in the call."""
    H, V = 320, 700
    hmax = synth.hidden(513, H, 21)
    w = synth.weight(V, H, 0.02, 21)
    alpha = 1.0 / 8
    full = gpu_bf16_f32(hmax, w, alpha)
    ref, absum = oracle.logits_bf16_f32(hmax[:40], w, alpha)
    assert_fp32_close(full[:40], ref, absum, "prefix rows")
    for r in list(range(1, 18)) + [31, 32, 33, 64, 100, 255, 256, 257, 300, 512]:
        sub = gpu_bf16_f32(hmax[:r], w, alpha)
        assert np.array_equal(f32_bits(sub), f32_bits(full[:r])), r
    perm = np.random.default_rng(0).permutation(513)
    shuffled = gpu_bf16_f32(hmax[perm], w, alpha)
    assert np.array_equal(f32_bits(shuffled), f32_bits(full[perm]))


def test_vocab_position_invariance():
    """A vocab row's logits do not depend on where it sits in W (which TMEM lane of which tile,
    full or partial): rolling W by rows that are not multiples of 16 or 128 rolls the logits."""
    rows, H, V = 5, 192, 1000
    h = synth.hidden(rows, H, 41)
    w = synth.weight(V, H, 0.02, 41)
    base = gpu_bf16_f32(h, w, 0.125)
    for shift in (1, 37, 128 + 5, 500):
        rolled = gpu_bf16_f32(h, np.roll(w, shift, axis=0), 0.125)
        assert np.array_equal(f32_bits(rolled), f32_bits(np.roll(base, shift, axis=1))), shift
    # the same rows inside a 300-row call (round-robin tiles) and a 5-row call (strips)
    many = gpu_bf16_f32(np.concatenate([h, synth.hidden(295, H, 42)]), w, 0.125)
    assert np.array_equal(f32_bits(many[:rows]), f32_bits(base))


def test_deterministic_and_no_writes_outside_logits():
    rows, H, V = 70, 256, 333
    h = dev_bf16(synth.hidden(rows, H, 8))
    w = dev_bf16(synth.weight(V, H, 0.02, 8))
    pad = 4096
    buf = torch.full((rows * V + 2 * pad,), float("nan"), dtype=torch.float32, device="cuda")
    out = buf[pad:pad + rows * V].view(rows, V)
    lm.logits_bf16_f32(h, w, 0.25, out=out)
    check_status()
    first = out.clone()
    lm.logits_bf16_f32(h, w, 0.25, out=out)
    check_status()
    assert torch.equal(first.view(torch.int32), out.view(torch.int32))
    assert torch.isnan(buf[:pad]).all() and torch.isnan(buf[pad + rows * V:]).all()


def test_side_stream_and_empty_call():
    rows, H, V = 8, 128, 256
    h = dev_bf16(synth.hidden(rows, H, 9))
    w = dev_bf16(synth.weight(V, H, 0.02, 9))
    ref = lm.logits_bf16_f32(h, w, 0.5)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out = lm.logits_bf16_f32(h, w, 0.5)
    s.synchronize()
    check_status()
    assert torch.equal(out.view(torch.int32), ref.view(torch.int32))
    empty = lm.logits_bf16_f32(h[:0], w, 0.5)
    assert empty.shape == (0, V)


# ---------------------------------------------------------------- full-size workloads

@pytest.fixture(scope="module")
def decode_inputs():
    rows_list, H, V, std, alpha = synth.WORKLOADS["decode"]
    h = synth.hidden(max(rows_list), H, synth.SEED_DECODE)
    w = synth.weight(V, H, std, synth.SEED_DECODE)
    return h, w, dev_bf16(w), rows_list, alpha


def test_decode_workload_matches_oracle(decode_inputs):
    """rows in {1..64}, H = 2048, V = 151936, alpha = 1/8: every element of the 64-row call
    against the oracle, every smaller call bitwise against its prefix."""
    h, w, wd, rows_list, alpha = decode_inputs
    full = gpu_bf16_f32(h, wd, alpha)
    ref, absum = oracle.logits_bf16_f32(h, w, alpha)
    assert_fp32_close(full, ref, absum, "decode R=64")
    for r in rows_list:
        sub = gpu_bf16_f32(h[:r], wd, alpha)
        assert np.array_equal(f32_bits(sub), f32_bits(full[:r])), r


def test_spec_verify_workload():
    """32 sequences x (1 target + 3 draft) rows = 128, ragged 97, and the 32-row draft-head call
    (rows 4s): H = 4096, V = 128256, alpha = 1/16. Shared rows must be bit-identical between
    the target and draft calls (page 1 requires draft and target logits to agree)."""
    rows_list, H, V, std, alpha = synth.WORKLOADS["spec_verify"]
    h = synth.hidden(128, H, synth.SEED_SPEC)
    w = synth.weight(V, H, std, synth.SEED_SPEC)
    wd = dev_bf16(w)
    full = gpu_bf16_f32(h, wd, alpha)
    sample = np.random.default_rng(synth.SEED_SPEC).choice(128, 16, replace=False)
    ref, absum = oracle.logits_bf16_f32(h[sample], w, alpha)
    assert_fp32_close(full[sample], ref, absum, "spec-verify sampled rows")
    ragged = gpu_bf16_f32(h[:97], wd, alpha)
    assert np.array_equal(f32_bits(ragged), f32_bits(full[:97]))
    draft_rows = np.arange(0, 128, 4)
    draft = gpu_bf16_f32(h[draft_rows], wd, alpha)
    assert np.array_equal(f32_bits(draft), f32_bits(full[draft_rows]))


def test_prefill_workload_sampled_rows():
    """rows = 8192, H = 4096, V = 151936, alpha = 1/8 in the launch configuration the benchmark
    times; 64 seeded sampled rows against the oracle and bitwise against a 64-row call."""
    rows_list, H, V, std, alpha = synth.WORKLOADS["prefill"]
    R = rows_list[0]
    hd = synth.hidden(R, H, synth.SEED_PREFILL, device="cuda")
    wd = synth.weight(V, H, std, synth.SEED_PREFILL, device="cuda")
    out = lm.logits_bf16_f32(hd, wd, alpha)
    check_status()
    sample = np.sort(np.random.default_rng(synth.SEED_PREFILL_SAMPLE).choice(R, 64, replace=False))
    idx = torch.from_numpy(sample).cuda()
    got = out[idx].cpu().numpy()
    del out
    h_s = hd[idx].contiguous()
    small = lm.logits_bf16_f32(h_s, wd, alpha)
    check_status()
    assert np.array_equal(f32_bits(small.cpu().numpy()), f32_bits(got))
    h_bits = h_s.view(torch.int16).cpu().numpy().view(np.uint16)
    w_bits = wd.view(torch.int16).cpu().numpy().view(np.uint16)
    ref, absum = oracle.logits_bf16_f32(h_bits, w_bits, alpha)
    assert_fp32_close(got, ref, absum, "prefill sampled rows")
