"""Pins for the CPU oracle: each check ties it to something other than itself -- a library
conversion, a closed form, exact integer arithmetic or a brute-force search -- so that a dropped
term, a wrong sign or index, or a transposed operand in the oracle fails here.

Formats and rules pinned: bf16 and E4M3fn decode (torch's own dtypes), E2M1 decode (the NVFP4
value set +-{0, 0.5, 1, 1.5, 2, 3, 4, 6}), one round-to-nearest-even from double to fp32 (numpy's
cast) and to bf16 (brute-force nearest search), and the head
    logits = RN(alpha * hidden @ W^T)
from "[Model] Honor fp32 head_dtype in Inkling muP logits (target + MTP draft)" ("Purpose";
"muP is folded into the fp32 GEMM") and lm_head_nvfp4_rows.rs (module doc).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from oracle_inputs import nvfp4_weights


def bf16_bits_of_f32(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bits through torch (round-to-nearest-even: a library routine)."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def all_bf16_values() -> np.ndarray:
    codes = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    return torch.from_numpy(codes.view(np.int16)).view(torch.bfloat16).float().double().numpy()


# ---------------------------------------------------------------- element decoders

def test_bf16_decode_all_codes_match_torch_and_ieee_fields():
    lib_vals = all_bf16_values()
    for code in range(65536):
        got = oracle.bf16_value(code)
        want = lib_vals[code]
        if math.isnan(want):
            assert math.isnan(got), hex(code)
            continue
        assert got == want and math.copysign(1, got) == math.copysign(1, want), hex(code)
    # IEEE field reading on a few codes, independent of the bit-shift trick
    for code in [0x0001, 0x007F, 0x0080, 0x3F80, 0x4049, 0xC2F7, 0x7F7F, 0x8001]:
        s, e, m = code >> 15, (code >> 7) & 0xFF, code & 0x7F
        mag = (m / 128.0) * 2.0 ** -126 if e == 0 else (1 + m / 128.0) * 2.0 ** (e - 127)
        assert oracle.bf16_value(code) == (-mag if s else mag)
    assert math.isinf(oracle.bf16_value(0x7F80)) and oracle.bf16_value(0xFF80) < 0


E2M1_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_decode_all_codes_match_value_set():
    for code in range(16):
        want = E2M1_TABLE[code & 7] * (-1.0 if code & 8 else 1.0)
        got = oracle.e2m1_value(code)
        assert got == want, code
        assert math.copysign(1, got) == (-1 if code & 8 else 1), code  # 0x8 is -0


def test_e2m1_decode_matches_torch_float4_where_supported():
    packed = torch.arange(256, dtype=torch.uint8).view(torch.float4_e2m1fn_x2)
    try:
        vals = packed.to(torch.float32)
    except Exception:
        pytest.skip("this torch build cannot convert float4_e2m1fn_x2")
    vals = vals.numpy().reshape(-1)
    if vals.size != 512:
        pytest.skip("float4_e2m1fn_x2 conversion does not unpack to two values per byte")
    for byte in range(256):
        lo, hi = oracle.e2m1_value(byte & 0xF), oracle.e2m1_value(byte >> 4)
        assert {vals[2 * byte], vals[2 * byte + 1]} <= {lo, hi} | {-lo, -hi}


def test_e4m3_decode_all_codes_match_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    lib = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for code in range(256):
        got = oracle.e4m3_value(code)
        if math.isnan(lib[code]):
            assert math.isnan(got), hex(code)
            assert code in (0x7F, 0xFF)
        else:
            assert got == lib[code], hex(code)
    assert oracle.e4m3_value(0x7E) == 448.0
    assert oracle.e4m3_value(0x01) == 2.0 ** -9
    assert oracle.e4m3_value(0x08) == 2.0 ** -6


def test_e2m1_times_e4m3_is_exact_in_bf16():
    """Every E2M1 x E4M3 product (all 8 x 127 non-negative, non-NaN pairs) round-trips through
    bf16 unchanged -- the reason a dequantised NVFP4 weight tile can be held in bf16 exactly."""
    for q in range(8):
        for s in range(0x7F):
            p = oracle.e2m1_value(q) * oracle.e4m3_value(s)
            assert oracle.bf16_value(oracle.round_bf16(p)) == p
            assert bf16_bits_of_f32(np.array([p], np.float32))[0] == oracle.round_bf16(p)


# ---------------------------------------------------------------- rounding

def _bf16_nearest_bruteforce(x: float, finite_sorted: np.ndarray, codes_sorted: np.ndarray) -> int:
    """Nearest finite bf16 by search, ties to the even code, overflow to infinity."""
    maxf = finite_sorted[-1]
    if abs(x) >= maxf + (2.0 ** 128 - maxf) / 2:
        return 0x7F80 | (0x8000 if x < 0 else 0)
    i = int(np.searchsorted(finite_sorted, x))
    cands = [j for j in (i - 1, i) if 0 <= j < len(finite_sorted)]
    best = min(abs(finite_sorted[j] - x) for j in cands)
    ties = [int(codes_sorted[j]) for j in cands if abs(finite_sorted[j] - x) == best]
    if len(ties) == 1:
        return ties[0]
    even = [c for c in ties if c % 2 == 0]
    return even[0]


def test_round_bf16_matches_bruteforce_nearest_even():
    vals = all_bf16_values()
    codes = np.arange(65536)
    finite = np.isfinite(vals) & ~((vals == 0) & (codes >= 0x8000))  # drop NaN/inf and -0
    order = np.argsort(vals[finite], kind="stable")
    fs, cs = vals[finite][order], codes[finite][order]
    rng = np.random.default_rng(7)
    xs = list(rng.standard_normal(2000) * 10.0 ** rng.integers(-45, 39, 2000))
    # exact midpoints between neighbours (ties), subnormal region, overflow boundary
    for c in [0x0001, 0x0002, 0x3F80, 0x3F81, 0x4000, 0x7F7E, 0x007F, 0x0080]:
        a, b = oracle.bf16_value(c), oracle.bf16_value(c + 1)
        xs += [(a + b) / 2, -(a + b) / 2, np.nextafter((a + b) / 2, 0), np.nextafter((a + b) / 2, 1e300)]
    maxf = oracle.bf16_value(0x7F7F)
    xs += [maxf, np.nextafter(maxf + 2.0 ** 119, 0), maxf + 2.0 ** 119, 1e300, -1e300, 1e-300]
    for x in xs:
        x = float(x)
        got = oracle.round_bf16(x)
        want = _bf16_nearest_bruteforce(x, fs, cs)
        if x != 0 and abs(x) < oracle.bf16_value(0x0001) / 2 + 1e-320:  # rounds to a signed zero
            assert got & 0x7FFF == want & 0x7FFF
        else:
            assert got == want, (x, hex(got), hex(want))
    assert oracle.round_bf16(0.0) == 0x0000 and oracle.round_bf16(-0.0) == 0x8000
    assert oracle.round_bf16(float("inf")) == 0x7F80
    assert (oracle.round_bf16(float("nan")) & 0x7FFF) > 0x7F80


def test_round_bf16_matches_torch_on_float32_inputs():
    """Where the double is already a float32, torch's float32 -> bf16 RNE is one rounding."""
    rng = np.random.default_rng(11)
    xs = (rng.standard_normal(5000) * 10.0 ** rng.integers(-30, 30, 5000)).astype(np.float32)
    lib = bf16_bits_of_f32(xs)
    for x, want in zip(xs, lib):
        assert oracle.round_bf16(float(x)) == int(want)


def test_round_f32_matches_numpy_cast():
    rng = np.random.default_rng(3)
    xs = rng.standard_normal(5000) * 10.0 ** rng.integers(-40, 40, 5000)
    with np.errstate(over="ignore"):
        for x in xs:
            assert np.float32(oracle.round_f32(float(x))) == np.float32(x)


# ---------------------------------------------------------------- the fp32 head

def test_hand_computed_dot_products():
    # H = 16, small integers: closed forms written out
    H = 16
    h = np.zeros((2, H), np.float32)
    w = np.zeros((3, H), np.float32)
    h[0] = 1.0                         # row of ones
    h[1] = np.arange(H)                # 0..15
    w[0] = np.arange(H)                # sum k = 120 ; sum k^2 = 1240
    w[1] = -2.0                        # -2 * 16 = -32 ; -2 * 120 = -240
    w[2, 3] = 0.5                      # picks element 3: 0.5 ; 1.5
    out, absum = oracle.logits_bf16_f32(bf16_bits_of_f32(h), bf16_bits_of_f32(w), 1.0)
    assert out.tolist() == [[120.0, -32.0, 0.5], [1240.0, -240.0, 1.5]]
    assert absum.tolist() == [[120.0, 32.0, 0.5], [1240.0, 240.0, 1.5]]
    out, _ = oracle.logits_bf16_f32(bf16_bits_of_f32(h), bf16_bits_of_f32(w), 0.25)
    assert out.tolist() == [[30.0, -8.0, 0.125], [310.0, -60.0, 0.375]]


def test_integer_inputs_equal_exact_integer_matmul():
    """Small-integer operands: every partial sum is an exact integer below 2^24, so the result
    must equal int64 arithmetic bit-for-bit (any sign or index error shows up here)."""
    rng = np.random.default_rng(5)
    rows, H, V = 5, 96, 37
    hi = rng.integers(-8, 9, (rows, H))
    wi = rng.integers(-8, 9, (V, H))
    out, _ = oracle.logits_bf16_f32(bf16_bits_of_f32(hi.astype(np.float32)),
                                    bf16_bits_of_f32(wi.astype(np.float32)), 1.0)
    want = (hi.astype(np.int64) @ wi.astype(np.int64).T).astype(np.float32)
    assert np.array_equal(out, want)
    # non-square shapes with rows != V catch a transposed operand
    out2, _ = oracle.logits_bf16_f32(bf16_bits_of_f32(hi[:2].astype(np.float32)),
                                     bf16_bits_of_f32(wi.astype(np.float32)), 0.5)
    assert np.array_equal(out2, (want[:2] * 0.5).astype(np.float32))


def test_one_hot_rows_pick_columns_of_w():
    H, V = 256, 1024
    w_bits = synth.weight(V, H, 0.02, synth.SEED_TINY)
    wf = synth.bf16_bits_to_f32(w_bits).astype(np.float64)
    ks = [0, 1, 17, 255]
    h = np.zeros((len(ks), H), np.float32)
    for i, k in enumerate(ks):
        h[i, k] = 1.0
    for alpha in (1.0, 0.25, 1.0 / 3.0):
        out, _ = oracle.logits_bf16_f32(bf16_bits_of_f32(h), w_bits, alpha)
        for i, k in enumerate(ks):
            want = (np.float64(np.float32(alpha)) * wf[:, k]).astype(np.float32)
            assert np.array_equal(out[i], want)


def test_zero_and_identity_block_weights():
    rows, H, V = 3, 64, 80
    h_bits = synth.hidden(rows, H, 99)
    hf = synth.bf16_bits_to_f32(h_bits)
    out, _ = oracle.logits_bf16_f32(h_bits, np.zeros((V, H), np.uint16), 0.125)
    assert np.all(out == 0) and not np.any(np.signbit(out))
    eye = np.zeros((V, H), np.float32)
    eye[np.arange(H), np.arange(H)] = 1.0
    out, _ = oracle.logits_bf16_f32(h_bits, bf16_bits_of_f32(eye), 0.125)
    assert np.array_equal(out[:, :H], (hf * np.float32(0.125)).astype(np.float32))
    assert np.all(out[:, H:] == 0)


def test_alpha_fold_against_separate_multiply():
    """RN(alpha*S) vs RN(RN(S)*alpha): equal for power-of-two alpha, within one fp32 ulp else
    (page 1's fold claim, with the double rounding a separate multiply adds)."""
    rows, H, V = 4, 256, 1024
    h = synth.hidden(rows, H, synth.SEED_TINY)
    w = synth.weight(V, H, 0.02, synth.SEED_TINY)
    base, _ = oracle.logits_bf16_f32(h, w, 1.0)
    for alpha in (0.25, 0.125, 1.0 / 16):
        fused, _ = oracle.logits_bf16_f32(h, w, alpha)
        assert np.array_equal(fused, (base * np.float32(alpha)).astype(np.float32))
    for alpha in (1.0 / 3.0, 1.0 / 6.0, 0.7):
        fused, _ = oracle.logits_bf16_f32(h, w, alpha)
        sep = (base * np.float32(alpha)).astype(np.float32)
        ulp = np.spacing(np.abs(fused))
        assert np.all(np.abs(fused.astype(np.float64) - sep) <= ulp)


def test_matches_library_double_matmul():
    """numpy's float64 matmul (BLAS) on the decoded operands: the same real number up to the
    double summation order, so after one fp32 rounding the two agree to within one ulp."""
    for rows, H, V, seed in [(4, 256, 1024, synth.SEED_TINY), (3, 2048, 512, 77)]:
        h = synth.hidden(rows, H, seed)
        w = synth.weight(V, H, 0.02, seed)
        alpha = 0.25
        out, absum = oracle.logits_bf16_f32(h, w, alpha)
        hd = synth.bf16_bits_to_f32(h).astype(np.float64)
        wd = synth.bf16_bits_to_f32(w).astype(np.float64)
        ref = (np.float64(np.float32(alpha)) * (hd @ wd.T)).astype(np.float32)
        diff = np.abs(out.astype(np.float64) - ref)
        assert np.all(diff <= np.spacing(np.abs(ref))), diff.max()
        assert np.mean(out == ref) > 0.99
        assert np.allclose(absum, abs(alpha) * (np.abs(hd) @ np.abs(wd).T), rtol=1e-12)


def test_empty_rows():
    out, absum = oracle.logits_bf16_f32(np.zeros((0, 64), np.uint16), np.zeros((8, 64), np.uint16), 1.0)
    assert out.shape == (0, 8) and absum.shape == (0, 8)


# ---------------------------------------------------------------- the NVFP4 head

def _dequant_with_torch(packed, scales, g):
    """Independent dequantisation through torch's float8_e4m3fn and the NVFP4 value set."""
    V, Hh = packed.shape
    lo, hi = packed & 0xF, packed >> 4
    codes = np.empty((V, 2 * Hh), np.uint8)
    codes[:, 0::2], codes[:, 1::2] = lo, hi
    mags = np.array(E2M1_TABLE)[codes & 7]
    q = np.where(codes & 8, -mags, mags)
    s = torch.from_numpy(scales.copy()).view(torch.float8_e4m3fn).double().numpy()
    return q * np.repeat(s, 16, axis=1) * np.float64(np.float32(g))


def test_nvfp4_weight_decode_matches_torch_dequant():
    V, H = 40, 64
    packed, scales, g = nvfp4_weights(V, H, 0.02, 123)
    ref = _dequant_with_torch(packed, scales, g)
    for v in range(V):
        for k in range(H):
            assert oracle.nvfp4_weight(packed, scales, g, v, k) == ref[v, k]


def test_nvfp4_head_one_hot_and_integer_cases():
    V, H = 48, 64
    packed, scales, g = nvfp4_weights(V, H, 0.02, 321)
    wq = _dequant_with_torch(packed, scales, g)
    ks = [0, 1, 15, 16, 63]
    h = np.zeros((len(ks), H), np.float32)
    for i, k in enumerate(ks):
        h[i, k] = 1.0
    out, _ = oracle.logits_w4a16_nvfp4(bf16_bits_of_f32(h), packed, scales, g, 0.5)
    for i, k in enumerate(ks):
        want = np.array([oracle.round_bf16(0.5 * wq[v, k]) for v in range(V)], np.uint16)
        assert np.array_equal(out[i], want)
        # power-of-two alpha: the bf16 of the exact product, via torch's float32 path (exact here)
        assert np.array_equal(out[i], bf16_bits_of_f32((0.5 * wq[:, k]).astype(np.float32)))
    # integer codes, unit scale (E4M3 0x38 = 1.0), g = 1: exact small sums
    rng = np.random.default_rng(9)
    codes = rng.integers(0, 16, (V, H)).astype(np.uint8)
    pk = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    sc = np.full((V, H // 16), 0x38, np.uint8)
    hi = rng.integers(-4, 5, (3, H)).astype(np.float32)
    out, _ = oracle.logits_w4a16_nvfp4(bf16_bits_of_f32(hi), pk, sc, 1.0, 1.0)
    qv = np.array(E2M1_TABLE)[codes & 7] * np.where(codes & 8, -1.0, 1.0)
    exact = hi.astype(np.float64) @ qv.T  # sums of multiples of 0.5 below 2^8: exact
    assert np.array_equal(out, bf16_bits_of_f32(exact.astype(np.float32)))


def test_nvfp4_head_matches_library_double_matmul():
    rows, H, V = 5, 256, 300
    h = synth.hidden(rows, H, 31)
    packed, scales, g = nvfp4_weights(V, H, 0.02, 32)
    out, _ = oracle.logits_w4a16_nvfp4(h, packed, scales, g, 0.125)
    wq = _dequant_with_torch(packed, scales, g)
    ref = 0.125 * (synth.bf16_bits_to_f32(h).astype(np.float64) @ wq.T)
    got = synth.bf16_bits_to_f32(out).astype(np.float64)
    # one bf16 rounding of the same real number (BLAS sums in another order): within 1 ulp
    assert np.all(np.abs(got - ref) <= np.spacing(np.abs(ref).astype(np.float32)) * 2 ** 16)
    assert np.mean(bf16_bits_of_f32(ref.astype(np.float32)) == out) > 0.98


def test_nvfp4_quantiser_round_trip_bounds():
    """The oracle quantiser (which also makes the NVFP4 test weights): decoded NVFP4 is within one
    E2M1 step (relative to the block scale) of the bf16 weights it came from, and no decoded
    weight exceeds 6 * 448 * g."""
    V, H = 64, 256
    w_bits = synth.weight(V, H, 0.02, 44)
    wf = synth.bf16_bits_to_f32(w_bits).astype(np.float64)
    packed, scales, g = oracle.nvfp4_quantize(w_bits)
    g = float(g)
    wq = _dequant_with_torch(packed, scales, g)
    s = torch.from_numpy(scales.copy()).view(torch.float8_e4m3fn).double().numpy()
    step = np.repeat(s, 16, axis=1) * g  # the value of one E2M1 unit in this block
    # largest gap in the E2M1 grid is 2 (between 4 and 6): error <= 1 unit, and <= 0.25 near 0
    assert np.all(np.abs(wq - wf) <= 1.0 * step + 1e-30)
    assert np.max(np.abs(wq)) <= 6 * 448 * g * (1 + 1e-12)


def f16_bits(x: np.ndarray) -> np.ndarray:
    """float -> IEEE binary16 bits through numpy (round-to-nearest-even: a library routine)."""
    return np.ascontiguousarray(x, dtype=np.float64).astype(np.float16).view(np.uint16)


def test_f16_decode_all_codes_match_numpy():
    codes = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    lib_vals = codes.view(np.float16).astype(np.float64)
    for code in range(65536):
        got = oracle.f16_value(code)
        want = lib_vals[code]
        if math.isnan(want):
            assert math.isnan(got), hex(code)
        else:
            assert got == want and math.copysign(1.0, got) == math.copysign(1.0, want), hex(code)


def test_f16_head_matches_library_double_matmul():
    rng = np.random.default_rng(21)
    rows, H, V = 5, 96, 37
    h = f16_bits(rng.normal(0.0, 1.0, (rows, H)))
    w = f16_bits(rng.normal(0.0, 0.05, (V, H)))
    hd = h.view(np.float16).astype(np.float64)
    wd = w.view(np.float16).astype(np.float64)
    for alpha in (1.0, 0.125, -0.7):
        got, absum = oracle.logits_f32(h, w, alpha, dtype="f16")
        want = (np.float64(np.float32(alpha)) * (hd @ wd.T)).astype(np.float32)
        # products are exact in double; the two double sums differ only in order
        assert np.allclose(got, want, rtol=0, atol=1e-6 * float(absum.max()) + 1e-30)
        assert np.allclose(absum, abs(np.float32(alpha)) * (np.abs(hd) @ np.abs(wd).T))


def test_f16_integer_inputs_equal_exact_integer_matmul():
    rng = np.random.default_rng(22)
    rows, H, V = 7, 64, 19
    hi = rng.integers(-30, 31, (rows, H))
    wi = rng.integers(-30, 31, (V, H))
    got, _ = oracle.logits_f32(f16_bits(hi), f16_bits(wi), 1.0, dtype="f16")
    assert np.array_equal(got, (hi @ wi.T).astype(np.float32))


def test_bias_alone_is_alpha_times_bias():
    """W = 0: logits = RN(alpha * bias[v]) for every row, in both input types."""
    rng = np.random.default_rng(23)
    rows, H, V = 3, 32, 50
    bias = rng.normal(0.0, 2.0, V)
    for dtype, enc in (("bf16", bf16_bits_of_f32), ("f16", f16_bits)):
        bb = enc(bias)
        bvals = (bb.view(np.float16).astype(np.float64) if dtype == "f16"
                 else np.array([oracle.bf16_value(int(x)) for x in bb]))
        h = enc(rng.normal(0.0, 1.0, (rows, H)))
        w = enc(np.zeros((V, H)))
        for alpha in (1.0, 0.25, -3.0):
            got, absum = oracle.logits_f32(h, w, alpha, bias_bits=bb, dtype=dtype)
            want = (np.float64(np.float32(alpha)) * bvals).astype(np.float32)
            assert np.array_equal(got, np.broadcast_to(want, (rows, V))), (dtype, alpha)
            assert np.allclose(absum, abs(np.float32(alpha)) * np.abs(bvals))


def test_bias_is_added_before_alpha():
    """One-hot rows read W[v, k]; the bias joins the sum before the multiply:
    RN(alpha * (W[v, k] + b[v])), which differs from RN(alpha * W[v, k] + b[v]) for alpha != 1."""
    H, V = 16, 8
    w = np.arange(V * H, dtype=np.float64).reshape(V, H) - 40.0
    b = np.linspace(-3.5, 3.5, V)
    wb, bb = bf16_bits_of_f32(w), bf16_bits_of_f32(b)
    ks = [0, 5, 15]
    h = np.zeros((len(ks), H))
    for i, k in enumerate(ks):
        h[i, k] = 1.0
    got, _ = oracle.logits_f32(bf16_bits_of_f32(h), wb, 0.5, bias_bits=bb)
    for i, k in enumerate(ks):
        want = (0.5 * (w[:, k] + b)).astype(np.float32)
        assert np.array_equal(got[i], want)
        assert not np.array_equal(got[i], (0.5 * w[:, k] + b).astype(np.float32))


def test_bf16_entry_without_bias_is_the_plain_head():
    rng = np.random.default_rng(24)
    h = bf16_bits_of_f32(rng.normal(0, 1, (4, 64)))
    w = bf16_bits_of_f32(rng.normal(0, 0.05, (33, 64)))
    a, sa = oracle.logits_f32(h, w, 0.125)
    b, sb = oracle.logits_bf16_f32(h, w, 0.125)
    assert np.array_equal(a, b) and np.array_equal(sa, sb)


# ---------------------------------------------------------------- the NVFP4 quantiser
# lm_head_nvfp4_rows.rs / mtp_head/new_bf16_moe.rs name quantize_to_nvfp4 (absmax, then encode)
# without printing its rules; the oracle's reading takes every decision in IEEE binary32 (see
# lmhead_oracle.c). These pins re-derive each decision independently: exact rationals for the
# nearest-even encoders, torch's float8_e4m3fn conversion, and numpy float32 for the arithmetic.
from fractions import Fraction

E2M1_MAGS = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3),
             Fraction(4), Fraction(6)]


def e4m3_fraction(c: int) -> Fraction:
    e, m = (c >> 3) & 15, c & 7
    return Fraction(m, 8) * Fraction(1, 64) if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)


E4M3_VALS = [e4m3_fraction(c) for c in range(127)]


def brute_nearest_even(x: Fraction, vals) -> int:
    """Index of the nearest value (ties to the even index), saturating at both ends."""
    best = min(range(len(vals)), key=lambda i: (abs(vals[i] - x), i % 2))
    return best


def float32_points(rng, lo, hi, n):
    """Random float32 values in [lo, hi] plus every table midpoint and its float32 neighbours."""
    return np.float32(rng.uniform(lo, hi, n))


def test_rn_e4m3_matches_bruteforce_and_torch():
    rng = np.random.default_rng(71)
    pts = list(float32_points(rng, 0.0, 460.0, 3000)) + list(np.float32(2.0 ** rng.uniform(-12, 9, 3000)))
    for a, b in zip(E4M3_VALS[:-1], E4M3_VALS[1:]):   # midpoints (exact in float32) and neighbours
        mid = np.float32(float((a + b) / 2))
        pts += [mid, np.nextafter(mid, np.float32(0)), np.nextafter(mid, np.float32(1e9))]
    pts += [np.float32(0.0), np.float32(448.0), np.float32(500.0), np.float32(1e30)]
    for t in pts:
        got = oracle.rn_e4m3(float(t))
        want = brute_nearest_even(Fraction(float(t)), E4M3_VALS)
        assert got == want, (float(t), got, want)
        if float(t) <= 448.0:
            via_torch = torch.tensor([float(t)], dtype=torch.float32).to(torch.float8_e4m3fn)
            assert int(via_torch.view(torch.uint8)[0]) == got, float(t)


def test_rn_e2m1_matches_bruteforce():
    rng = np.random.default_rng(72)
    pts = list(np.float32(rng.uniform(-7.0, 7.0, 4000)))
    for a, b in zip(E2M1_MAGS[:-1], E2M1_MAGS[1:]):
        mid = np.float32(float((a + b) / 2))
        for x in (mid, np.nextafter(mid, np.float32(0)), np.nextafter(mid, np.float32(9))):
            pts += [x, -x]
    pts += [np.float32(0.0), np.float32(-0.0), np.float32(6.0), np.float32(-100.0), np.float32(np.inf)]
    for x in pts:
        got = oracle.rn_e2m1(float(x))
        m = brute_nearest_even(Fraction(abs(float(x))) if np.isfinite(x) else Fraction(10 ** 9), E2M1_MAGS)
        want = (m | 8) if (float(x) < 0 and m != 0) else m
        assert got == want, (float(x), got, want)


def numpy_quantize_f32(w_bits: np.ndarray):
    """The reading re-derived with numpy float32 arithmetic and exact nearest-even searches."""
    wf = synth.bf16_bits_to_f32(w_bits)
    V, H = wf.shape
    amax = np.float32(np.max(np.abs(wf)))
    g = np.float32(amax / np.float32(2688.0)) if amax > 0 else np.float32(1.0)
    six_g = np.float32(np.float32(6.0) * g)
    scales = np.zeros((V, H // 16), np.uint8)
    codes = np.zeros((V, H), np.uint8)
    for v in range(V):
        for j in range(H // 16):
            blk = wf[v, 16 * j:16 * j + 16]
            t = np.float32(np.float32(np.max(np.abs(blk))) / six_g)
            s = brute_nearest_even(Fraction(float(t)), E4M3_VALS)
            scales[v, j] = s
            d = np.float32(np.float32(float(E4M3_VALS[s])) * g)
            for i in range(16):
                x = np.float32(blk[i] / d) if d > 0 else np.float32(0.0)
                m = brute_nearest_even(Fraction(abs(float(x))) if np.isfinite(x) else Fraction(10 ** 9),
                                       E2M1_MAGS)
                codes[v, 16 * j + i] = (m | 8) if (x < 0 and m != 0) else m
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return packed, scales, g


def test_quantiser_matches_numpy_float32_rederivation():
    rng = np.random.default_rng(73)
    # a spread of block magnitudes, so scales cover subnormal to large E4M3 codes
    w = rng.normal(0, 1, (6, 64)) * (10.0 ** rng.uniform(-4, 2, (6, 4))).repeat(16, axis=1)
    wb = bf16_bits_of_f32(w)
    p, s, g = oracle.nvfp4_quantize(wb)
    p2, s2, g2 = numpy_quantize_f32(wb)
    assert g == g2
    assert np.array_equal(s, s2)
    assert np.array_equal(p, p2)


def test_quantiser_closed_forms():
    # amax = 2688 gives g = 1; a block whose max is 6 gets scale 1.0 (0x38) and codes that are
    # the E2M1 values themselves
    H = 32
    w = np.zeros((2, H))
    w[0, 0] = 2688.0                                     # block 0 of row 0: t = 448 -> 0x7E
    w[1, :8] = [6.0, 3.0, -1.5, 0.5, -0.0, 2.0, -4.0, 1.0]
    w[1, 16:20] = [-6.0, 0.25, 0.75, 5.0]                # ties: 0.25 -> 0, 0.75 -> 1.0, 5 -> 4
    p, s, g = oracle.nvfp4_quantize(bf16_bits_of_f32(w))
    assert g == np.float32(1.0)
    assert s[0, 0] == 0x7E and s[0, 1] == 0 and s[1, 0] == 0x38 and s[1, 1] == 0x38
    codes = np.stack([p & 0x0F, p >> 4], axis=2).reshape(2, H)
    assert list(codes[1, :8]) == [7, 5, 11, 1, 0, 4, 14, 2]
    assert list(codes[1, 16:20]) == [15, 0, 2, 6]
    assert codes[0, 0] == 7 and not codes[0, 1:].any()


def test_quantiser_block_below_the_smallest_scale_gets_zero_codes():
    """A block whose maximum is far below amax rounds to scale code 0, so its divisor e4m3(0)·g
    is 0; the reading makes every code of that block 0 (not the +-6 that w / 0 would saturate
    to), signs included."""
    H = 32
    w = np.zeros((1, H))
    w[0, 0] = 2688.0                       # g = 1
    w[0, 16:32] = [1e-4, -1e-4, 3e-5, -2e-5] * 4   # t = bmax / 6 < 2^-10: scale code 0
    p, s, g = oracle.nvfp4_quantize(bf16_bits_of_f32(w))
    assert g == np.float32(1.0)
    assert s[0, 1] == 0
    codes = np.stack([p & 0x0F, p >> 4], axis=2).reshape(1, H)
    assert not codes[0, 16:].any()


def test_quantiser_all_zero_weights():
    p, s, g = oracle.nvfp4_quantize(np.zeros((3, 48), np.uint16))
    assert g == np.float32(1.0) and not p.any() and not s.any()


def test_quantiser_round_trip_error_is_within_half_a_code():
    """Dequantising gives each weight back to within half the E2M1 spacing at its magnitude
    (times s * g), except where the scale saturates or underflows."""
    wb = synth.weight(64, 256, 0.02, 74)
    p, s, g = oracle.nvfp4_quantize(wb)
    wf = synth.bf16_bits_to_f32(wb).astype(np.float64)
    for v in range(0, 64, 7):
        for k in range(0, 256, 5):
            deq = oracle.nvfp4_weight(p, s, float(g), v, k)
            unit = oracle.e4m3_value(int(s[v, k // 16])) * float(g)
            x = abs(wf[v, k]) / unit if unit > 0 else 0.0
            step = 0.5 if x < 2 else (1.0 if x < 4 else 2.0)
            assert abs(deq - wf[v, k]) <= 0.5 * step * unit * (1 + 1e-6) + 1e-30, (v, k)


# ---------------------------------------------------------------- log-probabilities of tokens
# The first page's "Purpose": fp32 logits for RL training-inference consistency and for the
# rejection sampling of speculative decoding, which consume the log-softmax. Reading:
#     logprob[r] = z[r, t_r] - log sum_v exp(z[r, v]),  z = the fp32 logits.

def test_logprobs_uniform_logits_give_minus_log_v():
    rows, H, V = 3, 32, 1000
    h = bf16_bits_of_f32(np.random.default_rng(101).normal(0, 1, (rows, H)))
    w = np.zeros((V, H), np.uint16)
    t = np.array([0, 499, 999], np.int32)
    lp, lse = oracle.logprobs_f32(h, w, 0.5, t)
    assert np.allclose(lse, np.float32(math.log(V)), rtol=0, atol=1e-6)
    assert np.allclose(lp, np.float32(-math.log(V)), rtol=0, atol=1e-6)


def test_logprobs_two_level_closed_form():
    """Bias-only logits: one token at a, the other V - 1 at b."""
    rows, H, V, a, b = 2, 16, 64, 3.0, -1.0
    h = bf16_bits_of_f32(np.ones((rows, H)))
    w = np.zeros((V, H), np.uint16)
    bias = np.full(V, b)
    bias[7] = a
    t = np.array([7, 8], np.int32)
    lp, lse = oracle.logprobs_f32(h, w, 1.0, t, bias_bits=bf16_bits_of_f32(bias))
    want_lse = math.log(math.exp(a) + (V - 1) * math.exp(b))
    assert abs(lse[0] - want_lse) < 1e-6 and abs(lse[1] - want_lse) < 1e-6
    assert abs(lp[0] - (a - want_lse)) < 1e-6 and abs(lp[1] - (b - want_lse)) < 1e-6


def test_logprobs_match_scipy_logsumexp_of_the_oracle_logits():
    from scipy.special import logsumexp
    rng = np.random.default_rng(102)
    rows, H, V = 6, 128, 3001
    h = bf16_bits_of_f32(rng.normal(0, 1, (rows, H)))
    w = bf16_bits_of_f32(rng.normal(0, 0.2, (V, H)))
    b = bf16_bits_of_f32(rng.normal(0, 1.0, V))
    t = rng.integers(0, V, rows).astype(np.int32)
    for dtype in ("bf16",):
        z, _ = oracle.logits_f32(h, w, 0.125, bias_bits=b, dtype=dtype)
        lp, lse = oracle.logprobs_f32(h, w, 0.125, t, bias_bits=b, dtype=dtype)
        want_lse = logsumexp(z.astype(np.float64), axis=1)
        assert np.allclose(lse, want_lse, rtol=2e-7, atol=0)
        assert np.allclose(lp, z[np.arange(rows), t] - want_lse, rtol=0, atol=1e-6)


def test_logprobs_out_of_range_target_is_nan():
    h = bf16_bits_of_f32(np.ones((2, 16)))
    w = bf16_bits_of_f32(np.ones((10, 16)))
    lp, _ = oracle.logprobs_f32(h, w, 1.0, np.array([-1, 10], np.int32))
    assert np.isnan(lp).all()


# ---------------------------------------------------------------- vocab-parallel log-probabilities
# "FP32 LM head skip FP32 cast" (key source excerpt, _compute_lm_head) takes the head as a
# VocabParallelEmbedding: W's rows split over GPUs. The log-softmax is still over the whole row;
# a slice contributes (max, sum of exp(z - max), target logit if held).

def _split(V, g):
    base, extra = divmod(V, g)
    starts = [r * base + min(r, extra) for r in range(g)]
    return [(b, base + (1 if r < extra else 0)) for r, b in enumerate(starts)]


def test_shard_merge_matches_scipy_logsumexp_of_the_whole_row():
    from scipy.special import logsumexp
    rng = np.random.default_rng(103)
    rows, H, V = 5, 96, 2003
    h = bf16_bits_of_f32(rng.normal(0, 1, (rows, H)))
    w = bf16_bits_of_f32(rng.normal(0, 0.3, (V, H)))
    t = np.array([0, 667, 668, 2002, 1001], np.int32)
    z, _ = oracle.logits_f32(h, w, 0.25)
    want_lse = logsumexp(z.astype(np.float64), axis=1)
    for g in (1, 2, 3, 7):
        stats = np.stack([oracle.logprob_shard_stats(h, w[b:b + n], b, 0.25, t)
                          for b, n in _split(V, g)])
        lp, lse = oracle.logprob_merge_shards(stats)
        assert np.allclose(lse, want_lse, rtol=2e-7, atol=0), g
        assert np.allclose(lp, z[np.arange(rows), t] - want_lse, rtol=0, atol=1e-6), g


def test_shard_stats_are_max_sum_and_held_target():
    rng = np.random.default_rng(104)
    rows, H, V, b0, n = 4, 64, 300, 100, 120
    h = bf16_bits_of_f32(rng.normal(0, 1, (rows, H)))
    w = bf16_bits_of_f32(rng.normal(0, 0.3, (V, H)))
    t = np.array([99, 100, 219, 220], np.int32)      # just outside, first, last, just outside
    z, _ = oracle.logits_f32(h, w[b0:b0 + n], 2.0)
    st = oracle.logprob_shard_stats(h, w[b0:b0 + n], b0, 2.0, t)
    zmax = z.astype(np.float64).max(axis=1)
    assert np.array_equal(st[:, 0], zmax)
    assert np.allclose(st[:, 1], np.exp(z.astype(np.float64) - zmax[:, None]).sum(axis=1),
                       rtol=1e-15, atol=0)
    assert np.isnan(st[0, 2]) and np.isnan(st[3, 2])
    assert st[1, 2] == z[1, 0] and st[2, 2] == z[2, n - 1]


def test_shard_merge_uniform_logits_and_missing_target():
    """W = 0: every logit is 0, so lse = log V whatever the split; a target no shard holds is
    NaN."""
    rows, H, V = 2, 16, 1000
    h = bf16_bits_of_f32(np.random.default_rng(105).normal(0, 1, (rows, H)))
    w = np.zeros((V, H), np.uint16)
    t = np.array([999, 1000], np.int32)
    stats = np.stack([oracle.logprob_shard_stats(h, w[b:b + n], b, 1.0, t)
                      for b, n in _split(V, 3)])
    lp, lse = oracle.logprob_merge_shards(stats)
    assert np.allclose(lse, np.float32(math.log(V)), rtol=0, atol=1e-6)
    assert abs(lp[0] + math.log(V)) < 1e-6 and np.isnan(lp[1])
