"""GPU parity of the NVFP4 quantiser (lmhead_nvfp4_quantize) against the CPU oracle, bit for bit.

lm_head_nvfp4_rows.rs and mtp_head/new_bf16_moe.rs name a two-kernel quantiser (absmax, then
encode); the rules are this library's reading, every decision one IEEE binary32 operation, so the
codes, scales and g must equal the oracle's exactly. The quantised head then runs through the
NVFP4 entry and is checked against the oracle head.
"""
import numpy as np
import pytest
import torch

import oracle
import fp32_accumulate_lm_b200 as lm
import synth
from gpu_helpers import check_status, dev_bf16, gpu_nvfp4
from tolerance import assert_bf16_close

pytestmark = pytest.mark.gpu


def bf16_bits(x):
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def gpu_quantize(w_bits):
    p, s, g = lm.nvfp4_quantize(dev_bf16(w_bits))
    check_status()
    return p.cpu().numpy(), s.cpu().numpy(), np.float32(g.item())


def assert_same_as_oracle(w_bits, what):
    p, s, g = gpu_quantize(w_bits)
    p0, s0, g0 = oracle.nvfp4_quantize(w_bits)
    assert g == g0, (what, g, g0)
    assert np.array_equal(s, s0), (what, int((s != s0).sum()))
    assert np.array_equal(p, p0), (what, int((p != p0).sum()))
    return p, s, g


@pytest.mark.parametrize("V,H,seed", [(1, 16, 1), (3, 48, 2), (257, 2048, 3), (1024, 4096, 4)])
def test_seeded_weights_match_oracle(V, H, seed):
    assert_same_as_oracle(synth.weight(V, H, 0.02, seed), f"{V}x{H}")


def test_block_magnitudes_across_the_e4m3_range():
    """Blocks scaled from 1e-6 to 1e3 relative to each other: scales from subnormal E4M3 codes
    to saturation, and codes that saturate at 6 where the block scale saturates."""
    rng = np.random.default_rng(81)
    V, H = 64, 512
    w = rng.normal(0, 1, (V, H)) * (10.0 ** rng.uniform(-6, 3, (V, H // 16))).repeat(16, axis=1)
    assert_same_as_oracle(bf16_bits(w), "spread")


def test_ties_signed_zeros_and_exact_values():
    """amax = 2688 makes g = 1; values on E2M1 midpoints exercise ties to the even code, -0 and
    tiny negatives must come out as code 0."""
    H = 64
    w = np.zeros((4, H))
    w[0, 0] = 2688.0
    w[1, :16] = [6, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, -0.25, -0.75, -2.5, -5, -0.0, -1e-3, 3, -6]
    w[2, :16] = [0.5] * 16
    w[3, 16:32] = np.linspace(-6, 6, 16)
    p, s, g = assert_same_as_oracle(bf16_bits(w), "ties")
    assert g == np.float32(1.0)
    codes = np.stack([p & 0x0F, p >> 4], axis=2).reshape(4, H)
    assert list(codes[1, :16]) == [7, 0, 2, 2, 4, 4, 6, 6, 0, 10, 12, 14, 0, 0, 5, 15]


def test_all_zero_and_single_spike():
    z = np.zeros((5, 32), np.uint16)
    p, s, g = assert_same_as_oracle(z, "zero")
    assert g == np.float32(1.0) and not p.any() and not s.any()
    w = np.zeros((3, 64))
    w[2, 63] = -3.0e38                     # near the top of bf16's range
    w[0, 1] = 1e-38                        # below every block scale after g is set by the spike
    assert_same_as_oracle(bf16_bits(w), "spike")


def test_subnormal_weights_divide_every_block():
    """W wholly in bf16's subnormal range: amax < 2^-126 makes g, and every divisor e4m3(s)·g, an
    fp32 subnormal, outside the reciprocal shortcut's range, so every block's codes come from the
    exact quotients, and the block scale's quotient has a subnormal divisor."""
    rng = np.random.default_rng(83)
    w = rng.normal(0, 1, (32, 256)) * 2.0 ** -130
    p, s, g = assert_same_as_oracle(bf16_bits(w), "subnormal")
    assert 0 < g < np.float32(2.0 ** -126)
    assert s.any() and p.any()


def test_rows_scaled_over_120_binades():
    """Rows scaled by 2^-60 .. 2^60: g near 2^50, the small rows' blocks round to scale code 0
    (every code 0), the large rows' span the E4M3 range."""
    rng = np.random.default_rng(84)
    w = rng.normal(0, 1, (96, 256)) * 2.0 ** rng.integers(-60, 61, (96, 1))
    p, s, g = assert_same_as_oracle(bf16_bits(w), "scaled")
    assert (s == 0).any() and (s > 0).any()


def test_quantised_head_runs_through_the_nvfp4_entry():
    """quantise on the GPU, then the W4A16 head on the GPU against the oracle head on the same
    codes."""
    rows, H, V = 17, 1024, 3000
    wb = synth.weight(V, H, 0.02, 85)
    h = synth.hidden(rows, H, 86)
    pd, sd, gd = lm.nvfp4_quantize(dev_bf16(wb))
    g = float(gd.item())
    got = gpu_nvfp4(h, pd, sd, g, 0.125)
    ref, absum = oracle.logits_w4a16_nvfp4(h, pd.cpu().numpy(), sd.cpu().numpy(), g, 0.125)
    assert_bf16_close(got, ref, absum, "quantised head")


def test_workspace_is_reused_and_rejected_when_too_small():
    wb = synth.weight(300, 256, 0.02, 87)
    W = dev_bf16(wb)
    ws = torch.zeros(lm.nvfp4_quantize_workspace_bytes(), dtype=torch.uint8, device="cuda")
    first = lm.nvfp4_quantize(W, workspace=ws)
    second = lm.nvfp4_quantize(W, workspace=ws)
    check_status()
    for a, b in zip(first, second):
        assert torch.equal(a, b)
    tiny = torch.zeros(4, dtype=torch.uint8, device="cuda")
    with pytest.raises(lm.LmheadError):
        lm.nvfp4_quantize(W, workspace=tiny)


def _near_boundary_weights(seed: int, amax: float):
    """Blocks whose elements divide by their block's d = e4m3(s) * g to within a few bf16 steps
    of the E2M1 code boundaries (0.25, 0.75, ..., 5). numpy float32 and torch's E4M3 conversion
    only aim the values; the expected codes are the oracle's."""
    rng = np.random.default_rng(seed)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    V, H = 256, 256
    w = np.zeros((V, H), np.float32)
    w[0, 0] = amax
    g = np.float32(np.float32(bf16_round(amax)) / np.float32(2688.0))
    six_g = np.float32(np.float32(6.0) * g)
    for v in range(V):
        for j in range(H // 16):
            if v == 0 and j == 0:
                continue
            bmax = bf16_round(float(six_g) * 2.0 ** rng.uniform(-6, np.log2(amax / float(six_g))))
            t = np.float32(np.float32(bmax) / six_g)
            s = float(torch.tensor([t]).to(torch.float8_e4m3fn).to(torch.float32)[0])
            d = np.float32(np.float32(s) * g)
            m = rng.choice(mids, 15)
            base = bf16_round_array(m * float(d))
            step = rng.integers(-2, 3, 15)
            vals = bf16_step(base, step) * rng.choice([-1.0, 1.0], 15)
            w[v, 16 * j] = bmax
            w[v, 16 * j + 1:16 * j + 16] = np.clip(vals, -bmax, bmax)
    return w


def bf16_round(x: float) -> float:
    return float(torch.tensor([x], dtype=torch.float32).to(torch.bfloat16).to(torch.float32)[0])


def bf16_round_array(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float32).numpy()


def bf16_step(x: np.ndarray, k: np.ndarray) -> np.ndarray:
    """x (bf16 values, positive) moved by k bf16 steps."""
    bits = (x.astype(np.float32).view(np.uint32) >> 16).astype(np.int64) + k
    return (bits.astype(np.uint32) << 16).view(np.float32)


@pytest.mark.parametrize("seed,amax", [(88, 7.3), (89, 0.0123), (90, 411.0)])
def test_quotients_near_code_boundaries(seed, amax):
    """The encode pass decides most codes from one reciprocal per block and divides exactly only
    near a code boundary; quotients aimed at the boundaries must still give the oracle's codes,
    and enough of them land inside the exact-division band to exercise it."""
    w = _near_boundary_weights(seed, amax)
    bits = bf16_bits(w)
    p, s, g = assert_same_as_oracle(bits, f"near-boundary {amax}")
    # how many quotients fell within 2^-16 of a boundary (numpy float32 = IEEE binary32)
    wf = (bits.astype(np.uint32) << 16).view(np.float32)
    e4m3 = torch.from_numpy(s.view(np.uint8).copy()).view(torch.float8_e4m3fn).to(torch.float32)
    d = (e4m3.numpy() * g).astype(np.float32).repeat(16, axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        x = np.abs(wf / d)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    rel = np.min(np.abs(x[..., None] / mids - 1.0), axis=-1)
    assert int((rel < 2.0 ** -16).sum()) >= 20
