"""The arithmetic argument behind the quantiser's encode pass, checked exhaustively on the host.

The encode pass does not divide each element by its block's d = e4m3(s) * g. It takes
r = fl(1/d), converts the two products w * fl(r (1 - 2^-16)) and w * fl(r (1 + 2^-16)), and keeps
their E2M1 code when the two agree; otherwise it divides. The claim: whenever the two codes
agree, they equal the code of the correctly rounded quotient fl(w / d), which is what the rules
(and the oracle) use. Here every finite bf16 w meets d values across the normal range, in IEEE
binary32 arithmetic (numpy float32: round to nearest, no contraction, subnormals kept), and the
claim must hold for all of them. This tests the method, not the kernel; the kernel's bits are
compared with the oracle's on the GPU.
"""
import numpy as np

MIDPOINTS = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float64)


def e2m1_code(v: np.ndarray) -> np.ndarray:
    """Nearest E2M1 code (ties to the even code, saturating at 6), sign on non-zero magnitudes."""
    m = np.abs(v.astype(np.float64))
    idx = np.searchsorted(MIDPOINTS, m, side="left")        # midpoints strictly below m
    tie = np.isin(m, MIDPOINTS)
    idx = np.where(tie & (idx % 2 == 1), idx + 1, idx)        # a tie goes to the even index
    code = idx.astype(np.uint8)
    return np.where((v < 0) & (code > 0), code | 8, code).astype(np.uint8)


def all_finite_bf16() -> np.ndarray:
    bits = np.arange(65536, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    return f[np.isfinite(f)]


def test_bracketing_products_decide_the_code_of_the_quotient():
    w = all_finite_bf16()
    rng = np.random.default_rng(7)
    e4m3 = np.array([m * 2.0 ** e for e in range(-6, 9) for m in (1, 1.125, 1.25, 1.375, 1.5,
                                                                  1.625, 1.75, 1.875)]
                    + [k * 2.0 ** -9 for k in range(1, 8)], np.float64)
    e4m3 = e4m3[e4m3 <= 448]
    # random global scales, and powers of two (1 = amax 2688), whose quotients land exactly on the
    # E2M1 midpoints: the ties the band exists for
    gs = np.concatenate([
        np.float32(rng.uniform(0.5, 1.0, 12)) * np.float32(2.0) ** rng.integers(-60, 60, 12),
        np.float32(2.0) ** np.arange(-40, 41, 8, dtype=np.float32)])
    band_lo, band_hi = np.float32(1 - 2.0 ** -16), np.float32(1 + 2.0 ** -16)
    fallback = total = 0
    for g in gs.astype(np.float32):
        for s in e4m3.astype(np.float32):
            d = np.float32(s * g)
            if not (2.0 ** -120 <= d <= 2.0 ** 120):
                continue                                     # always divided exactly
            r = np.float32(1) / d
            r_lo, r_hi = np.float32(r * band_lo), np.float32(r * band_hi)
            with np.errstate(over="ignore"):
                q_exact = e2m1_code(w / d)
                q_lo = e2m1_code(w * r_lo)
                q_hi = e2m1_code(w * r_hi)
            agree = q_lo == q_hi
            assert np.array_equal(q_lo[agree], q_exact[agree]), (float(g), float(s))
            fallback += int((~agree).sum())
            total += w.size
    assert total > 10_000_000
    # the exact division is the rare case
    assert fallback < 0.01 * total, fallback / total
