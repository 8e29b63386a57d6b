"""GPU parity of the W4A16 NVFP4 head (entry 2) against the CPU oracle, through the C ABI.

    W[v, k] = e2m1(code) * e4m3(scale[v, k/16]),  logits = bf16(alpha * g * hidden @ W^T)
(lm_head_nvfp4_rows.rs, module doc and lm_head_nvfp4_rows_run: declared W4A16 -- bf16
activations, never cast to E4M3 -- bf16 logits, a row's logits independent of the row count,
64-row calls). Tolerance: tolerance.assert_bf16_close; exact cases are compared bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import fp32_accumulate_lm_b200 as lm
import synth
from oracle_inputs import nvfp4_weights
from gpu_helpers import bf16_bits_of_f32, check_status, dev_bf16, dev_u8, gpu_nvfp4
from tolerance import assert_bf16_close

pytestmark = pytest.mark.gpu


@pytest.fixture(params=[1, 2], ids=["pair_table", "spread"])
def conversion(request):
    """Runs a test under each of the kernel's two code-to-bf16 conversions (the knob lives in the
    test build of the library, which has the same kernels)."""
    with lm.test_hooks():
        lm.set_nvfp4_conversion(request.param)
        try:
            yield request.param
        finally:
            lm.set_nvfp4_conversion(0)


def pack(codes: np.ndarray) -> np.ndarray:
    return (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)


def test_tiny_matches_oracle():
    H, V = 256, 1024
    h = synth.hidden(4, H, synth.SEED_TINY)
    packed, scales, g = nvfp4_weights(V, H, 0.02, synth.SEED_TINY)
    ref, absum = oracle.logits_w4a16_nvfp4(h, packed, scales, g, 0.25)
    got = gpu_nvfp4(h, packed, scales, g, 0.25)
    assert_bf16_close(got, ref, absum, "nvfp4 tiny")


def test_every_code_and_scale_decodes_exactly(conversion):
    """One-hot hidden rows read single weights: with g = 1 and alpha = 1 the logit is the bf16
    of e2m1 * e4m3, exact -- so this checks the dequantiser on all 16 codes (both nibble
    positions, including -0) and all 126 finite non-negative scales, plus negative scales."""
    H = 64
    codes = np.arange(16, dtype=np.uint8)
    scale_codes = np.concatenate([np.arange(0x00, 0x7F), [0x80 | 0x38, 0x80 | 0x01]]).astype(np.uint8)
    V = len(scale_codes) * 16
    c = np.zeros((V, H), np.uint8)
    s = np.zeros((V, H // 16), np.uint8)
    for i, sc in enumerate(scale_codes):
        for j, q in enumerate(codes):
            v = i * 16 + j
            c[v, :] = q                      # every k of row v holds code q
            s[v, :] = sc
    ks = [0, 1, 2, 3, 16, 17, 62, 63]        # low and high nibbles, every scale block
    h = np.zeros((len(ks), H), np.float32)
    for i, k in enumerate(ks):
        h[i, k] = 1.0
    hb = bf16_bits_of_f32(h)
    ref, _ = oracle.logits_w4a16_nvfp4(hb, pack(c), s, 1.0, 1.0)
    got = gpu_nvfp4(hb, pack(c), s, 1.0, 1.0)
    # -0 codes may come out as +0 or -0 logits: compare values, then bits elsewhere
    nz = (ref & 0x7FFF) != 0
    assert np.array_equal(got[nz], ref[nz])
    assert np.all((got[~nz] & 0x7FFF) == 0)


def test_integer_valued_sums_are_exact(conversion):
    rng = np.random.default_rng(12)
    rows, H, V = 23, 192, 260
    codes = rng.integers(0, 16, (V, H)).astype(np.uint8)
    scales = rng.choice(np.array([0x30, 0x38, 0x40], np.uint8), (V, H // 16))  # 0.5, 1, 2
    hi = rng.integers(-3, 4, (rows, H)).astype(np.float32)
    hb = bf16_bits_of_f32(hi)
    ref, _ = oracle.logits_w4a16_nvfp4(hb, pack(codes), scales, 1.0, 1.0)
    got = gpu_nvfp4(hb, pack(codes), scales, 1.0, 1.0)
    assert np.array_equal(got, ref)


def test_ragged_shapes_and_global_scale(conversion):
    for rows, H, V, seed in [(1, 64, 1, 1), (17, 128, 129, 2), (65, 320, 300, 3), (300, 64, 200, 4)]:
        h = synth.hidden(rows, H, seed)
        packed, scales, g = nvfp4_weights(V, H, 0.02, seed)
        for alpha in (1.0 / 8, 0.7):
            ref, absum = oracle.logits_w4a16_nvfp4(h, packed, scales, g, alpha)
            got = gpu_nvfp4(h, packed, scales, g, alpha)
            assert_bf16_close(got, ref, absum, f"nvfp4 {rows}x{H}x{V}")


@pytest.fixture(scope="module")
def nvfp4_inputs():
    rows_list, H, V, std, alpha = synth.WORKLOADS["nvfp4"]
    h = synth.hidden(max(rows_list), H, synth.SEED_NVFP4)
    packed, scales, g = nvfp4_weights(V, H, std, synth.SEED_NVFP4)
    return h, packed, scales, g, dev_u8(packed), dev_u8(scales), rows_list, alpha


def test_nvfp4_workload_matches_oracle_and_is_row_invariant(nvfp4_inputs):
    """rows in {1, 16, 64, 65, 256}, H = 2048, V = 151936, alpha = 1/8: the 65-row call against
    the oracle element by element, 16 sampled rows of the 256-row call too, and every row of
    every call bit-identical to the same row of the 256-row call."""
    h, packed, scales, g, pd, sd, rows_list, alpha = nvfp4_inputs
    full = gpu_nvfp4(h, pd, sd, g, alpha)
    ref, absum = oracle.logits_w4a16_nvfp4(h[:65], packed, scales, g, alpha)
    got65 = gpu_nvfp4(h[:65], pd, sd, g, alpha)
    assert_bf16_close(got65, ref, absum, "nvfp4 R=65")
    sample = np.sort(np.random.default_rng(7).choice(np.arange(65, 256), 16, replace=False))
    ref_s, absum_s = oracle.logits_w4a16_nvfp4(h[sample], packed, scales, g, alpha)
    assert_bf16_close(full[sample], ref_s, absum_s, "nvfp4 R=256 sampled")
    for r in rows_list:
        sub = gpu_nvfp4(h[:r], pd, sd, g, alpha)
        assert np.array_equal(sub, full[:r]), r


def test_64_row_chunked_calls_equal_one_call(nvfp4_inputs):
    """lm_head_nvfp4_rows_run walks rows in calls of at most 64, offsetting hidden by done*h*2
    and logits by done*v*2 bytes; the single call must give the same bits."""
    h, packed, scales, g, pd, sd, rows_list, alpha = nvfp4_inputs
    rows, H = 200, h.shape[1]
    V = packed.shape[0]
    hd = dev_bf16(h[:rows])
    whole = lm.logits_w4a16_nvfp4(hd, pd, sd, g, alpha)
    chunked = torch.empty_like(whole)
    done = 0
    while done < rows:
        m = min(rows - done, 64)
        st = lm.lmhead_logits_w4a16_nvfp4(hd.data_ptr() + done * H * 2, m, H, pd.data_ptr(),
                                          sd.data_ptr(), g, V, alpha,
                                          chunked.data_ptr() + done * V * 2,
                                          torch.cuda.current_stream().cuda_stream)
        assert st == 0
        done += m
    check_status()
    assert torch.equal(whole.view(torch.int16), chunked.view(torch.int16))


def test_pair_table_and_spread_give_identical_bits(nvfp4_inputs):
    """The two conversions are the same arithmetic (the table holds exactly the spread words), so
    every row count the table serves must match the spread path bit for bit."""
    h, packed, scales, g, pd, sd, rows_list, alpha = nvfp4_inputs
    with lm.test_hooks():
        try:
            for r in (1, 8, 9, 16, 17, 33, 64):
                lm.set_nvfp4_conversion(1)
                a = gpu_nvfp4(h[:r], pd, sd, g, alpha)
                lm.set_nvfp4_conversion(2)
                b = gpu_nvfp4(h[:r], pd, sd, g, alpha)
                assert np.array_equal(a, b), r
        finally:
            lm.set_nvfp4_conversion(0)
    # the release library (automatic choice) gives the same bits as well
    for r in (1, 64):
        assert np.array_equal(gpu_nvfp4(h[:r], pd, sd, g, alpha), gpu_nvfp4(h[:r], pd, sd, g, alpha))


@pytest.mark.parametrize("H", [32, 96, 160, 224, 2080])
def test_widths_that_are_odd_multiples_of_32(H, conversion):
    """lm_head_nvfp4_rows_run checks only k = H and lda = H: a width that is a multiple of 32 but
    not of 64 ends in half a K step of 64 (zero codes and zero scales past H, hidden zero-filled
    past H, two MMAs of 16 instead of four). Against the oracle, and every row of the smaller
    calls bit-identical to the same row of the 300-row call (two row tiles)."""
    V = 517
    h = synth.hidden(300, H, 50 + H)
    packed, scales, g = nvfp4_weights(V, H, 0.02, 60 + H)
    full = gpu_nvfp4(h, packed, scales, g, 0.125)
    ref, absum = oracle.logits_w4a16_nvfp4(h[:70], packed, scales, g, 0.125)
    assert_bf16_close(full[:70], ref, absum, f"nvfp4 H={H}")
    for r in (1, 17, 65, 129):
        assert np.array_equal(gpu_nvfp4(h[:r], packed, scales, g, 0.125), full[:r]), (H, r)


def test_odd_width_integer_sums_are_exact():
    """Integer-valued inputs at H = 2080 (32 mod 64): every fp32 order is exact, so the kernel
    must equal the oracle bit for bit -- a dropped or doubled half K step would show."""
    rng = np.random.default_rng(2080)
    rows, H, V = 9, 2080, 300
    codes = rng.integers(0, 16, (V, H)).astype(np.uint8)
    scales = rng.choice(np.array([0x30, 0x38, 0x40], np.uint8), (V, H // 16))
    hi = rng.integers(-2, 3, (rows, H)).astype(np.float32)
    hb = bf16_bits_of_f32(hi)
    ref, _ = oracle.logits_w4a16_nvfp4(hb, pack(codes), scales, 1.0, 1.0)
    got = gpu_nvfp4(hb, pack(codes), scales, 1.0, 1.0)
    assert np.array_equal(got, ref)
    # the last 32 columns alone: hidden zero elsewhere
    hz = np.zeros_like(hi)
    hz[:, H - 32:] = hi[:, H - 32:]
    hb = bf16_bits_of_f32(hz)
    ref, _ = oracle.logits_w4a16_nvfp4(hb, pack(codes), scales, 1.0, 1.0)
    assert np.array_equal(gpu_nvfp4(hb, pack(codes), scales, 1.0, 1.0), ref)
