"""GPU parity of the general fp32 entry, lmhead_logits_f32: IEEE fp16 operands and the embedding
bias, against the CPU oracle, through the C ABI.

    logits = fl32(alpha * fl32(hidden @ W^T + bias))
("FP32 LM head skip FP32 cast": the fused fp32-accumulate path admits fp16 as well as bf16 hidden
states of the weight's dtype; "[Model] Honor fp32 head_dtype in Inkling muP logits", "Purpose":
the projection with its embedding bias, then the multiply by 1/mup.) Tolerance:
tolerance.assert_fp32_close; exact cases are compared bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import fp32_accumulate_lm_b200 as lm
import synth
from gpu_helpers import check_status
from tolerance import assert_fp32_close

pytestmark = pytest.mark.gpu

TDT = {"bf16": torch.bfloat16, "f16": torch.float16}


def dev(bits, dtype):
    return synth.bits_to_torch(bits, TDT[dtype], "cuda")


def run(h, w, alpha, b=None, dtype="f16"):
    out = lm.logits_f32(dev(h, dtype), dev(w, dtype), alpha,
                        bias=None if b is None else dev(b, dtype))
    check_status()
    return out.cpu().numpy()


def f16_bits(x):
    return np.ascontiguousarray(x, dtype=np.float64).astype(np.float16).view(np.uint16)


def inputs(rows, H, V, seed, dtype):
    return (synth.hidden(rows, H, seed, dtype=TDT[dtype]),
            synth.weight(V, H, 0.02, seed, dtype=TDT[dtype]),
            synth.bias(V, seed, dtype=TDT[dtype]))


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("with_bias", [False, True])
def test_tiny_and_ragged_shapes_match_oracle(dtype, with_bias):
    for rows, H, V, seed in [(4, 256, 1024, 1), (1, 8, 1, 2), (17, 136, 129, 3),
                             (65, 320, 300, 4), (300, 64, 200, 5)]:
        h, w, b = inputs(rows, H, V, seed, dtype)
        b = b if with_bias else None
        for alpha in (1.0 / 8, 0.7):
            ref, absum = oracle.logits_f32(h, w, alpha, bias_bits=b, dtype=dtype)
            got = run(h, w, alpha, b, dtype)
            assert_fp32_close(got, ref, absum, f"{dtype} bias={with_bias} {rows}x{H}x{V}")


def test_f16_integer_valued_sums_are_exact():
    rng = np.random.default_rng(31)
    rows, H, V = 23, 192, 260
    hi = rng.integers(-20, 21, (rows, H))
    wi = rng.integers(-20, 21, (V, H))
    bi = rng.integers(-500, 501, V)
    for b in (None, f16_bits(bi)):
        ref, _ = oracle.logits_f32(f16_bits(hi), f16_bits(wi), 1.0, bias_bits=b, dtype="f16")
        got = run(f16_bits(hi), f16_bits(wi), 1.0, b)
        assert np.array_equal(got, ref)
        assert np.array_equal(got, (hi @ wi.T + (0 if b is None else bi)).astype(np.float32))


def test_f16_extremes_decode_exactly():
    """One-hot rows read single weights: every finite fp16 magnitude class (subnormals, the
    smallest normal, 1, the largest finite 65504) passes through the MMA and epilogue unchanged."""
    vals = np.array([2.0 ** -24, 3 * 2.0 ** -24, 2.0 ** -14, 1.0, -1.5, 1024.0, 65504.0, -65504.0])
    H, V = 64, len(vals)
    w = np.zeros((V, H))
    w[:, 5] = vals
    h = np.zeros((2, H))
    h[0, 5] = 1.0
    h[1, 5] = -1.0
    got = run(f16_bits(h), f16_bits(w), 1.0)
    assert np.array_equal(got[0], vals.astype(np.float32))
    assert np.array_equal(got[1], (-vals).astype(np.float32))


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_bias_alone_and_alpha_fold(dtype):
    """W = 0 gives fl32(alpha * bias) exactly; and with any W, the alpha call equals fl32(alpha *
    (the alpha = 1 call)) bit for bit, since the bias joins the sum before alpha."""
    rows, H, V = 9, 128, 777
    h, w, b = inputs(rows, H, V, 41, dtype)
    zero = np.zeros_like(w)
    bvals = synth.bits_to_torch(b, TDT[dtype]).double().numpy()
    for alpha in (1.0, 0.125, -3.0):
        got = run(h, zero, alpha, b, dtype)
        want = (np.float64(np.float32(alpha)) * bvals).astype(np.float32)
        assert np.array_equal(got, np.broadcast_to(want, (rows, V)))
    one = run(h, w, 1.0, b, dtype)
    for alpha in (0.125, 0.3, -7.0):
        assert np.array_equal(run(h, w, alpha, b, dtype), (np.float32(alpha) * one).astype(np.float32))


def test_general_entry_without_bias_is_the_bf16_entry():
    rows, H, V = 33, 512, 2048
    h, w, _ = inputs(rows, H, V, 51, "bf16")
    a = run(h, w, 0.125, None, "bf16")
    hd, wd = dev(h, "bf16"), dev(w, "bf16")
    b = lm.logits_bf16_f32(hd, wd, 0.125)
    check_status()
    assert np.array_equal(a, b.cpu().numpy())


def test_f16_bias_rows_are_independent_of_the_row_count():
    """Every row of calls with 1, 2, 17, 64, 65 and 200 rows equals the same row of one 300-row
    call, with fp16 operands and a bias."""
    rows, H, V = 300, 1024, 4096
    h, w, b = inputs(rows, H, V, 61, "f16")
    hd, wd, bd = dev(h, "f16"), dev(w, "f16"), dev(b, "f16")
    full = lm.logits_f32(hd, wd, 0.125, bias=bd)
    for r in (1, 2, 17, 64, 65, 200):
        part = lm.logits_f32(hd[:r].contiguous(), wd, 0.125, bias=bd)
        assert torch.equal(part, full[:r]), r
    check_status()


def test_decode_f16_bias_workload_sampled_rows():
    """The decode shape with fp16 operands and bias (rows 1..64, H = 2048, V = 151936,
    alpha = 1/8): rows of the 64-row call against the oracle element by element, and every call's
    rows equal to the same rows of the 64-row call."""
    rows_list, H, V, std, alpha = synth.WORKLOADS["decode_f16_bias"]
    R = max(rows_list)
    h = synth.hidden(R, H, synth.SEED_F16, dtype=torch.float16)
    w = synth.weight(V, H, std, synth.SEED_F16, dtype=torch.float16)
    b = synth.bias(V, synth.SEED_BIAS, dtype=torch.float16)
    hd, wd, bd = dev(h, "f16"), dev(w, "f16"), dev(b, "f16")
    full = lm.logits_f32(hd, wd, alpha, bias=bd)
    check_status()
    sample = [0, 31, 63]
    ref, absum = oracle.logits_f32(h[sample], w, alpha, bias_bits=b, dtype="f16")
    assert_fp32_close(full[sample].cpu().numpy(), ref, absum, "decode f16 + bias")
    for r in rows_list:
        part = lm.logits_f32(hd[:r].contiguous(), wd, alpha, bias=bd)
        assert torch.equal(part, full[:r]), r
    check_status()
