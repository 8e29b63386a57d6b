"""Parity bounds between the CUDA path and the CPU oracle.

fp32 head: the oracle is RN_fp32(alpha * S) with S exact (double); the kernel sums the same
exact bf16 products in an fp32 accumulator, 16 products per tensor-core step, in another order.
Bound (stated with the method's contract):
    |gpu - oracle| <= 1e-4 * |alpha| * sum_k |h_k * w_k| + 1e-7
The fp32 rounding error of a K-term sum is at most ~K * 2^-24 * sum|p| in the worst case and
~sqrt(K) * 2^-24 * sum|p| typically; 1e-4 covers K up to 4096 with a wide margin while still
catching any dropped term, wrong index or wrong scale (those move a logit by O(|h_k w_k|)).

NVFP4 head: the same bound on the dequantised weights (per-tensor scale included), plus one bf16
ulp of the oracle value for the kernel's extra roundings (acc*g, *alpha, then bf16) against the
oracle's single rounding from double.
"""
import numpy as np


def fp32_bound(abs_sum: np.ndarray) -> np.ndarray:
    return 1e-4 * abs_sum + 1e-7


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |x| (2^-133 below the normal range)."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126)
    return np.where(a > 0, 2.0 ** (e - 7), 2.0 ** -133)


def assert_fp32_close(gpu: np.ndarray, ref: np.ndarray, abs_sum: np.ndarray, what: str = ""):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(gpu - ref)
    bound = fp32_bound(abs_sum)
    bad = ~(err <= bound)
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside the bound; first at "
                             f"{tuple(i)}: gpu={gpu[tuple(i)]!r} oracle={ref[tuple(i)]!r} "
                             f"bound={bound[tuple(i)]!r}")


def assert_bf16_close(gpu_bits: np.ndarray, ref_bits: np.ndarray, abs_sum: np.ndarray,
                      what: str = ""):
    def widen(b):
        return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    gpu = widen(gpu_bits)
    ref = widen(ref_bits)
    err = np.abs(gpu - ref)
    bound = fp32_bound(abs_sum) + bf16_ulp(ref)
    bad = ~(err <= bound)
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside the bound; first at "
                             f"{tuple(i)}: gpu={gpu[tuple(i)]!r} oracle={ref[tuple(i)]!r} "
                             f"bound={bound[tuple(i)]!r}")
