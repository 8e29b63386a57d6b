"""NVFP4 test weights made by the oracle's quantiser (test infrastructure, like the oracle).

The NVFP4 head's parity tests need codes and scales that look like a quantised N(0, std) head.
They take them from ``oracle.nvfp4_quantize`` -- the one binary32 reading of the quantiser rules
that the GPU quantiser is also checked against -- applied to a seeded bf16 weight from
``synth``. Nothing here comes from the CUDA path.
"""
import oracle
import synth


def nvfp4_weights(V: int, H: int, std: float, seed: int):
    """(packed [V, H/2] u8, scales [V, H/16] u8, g float) quantised from synth.weight(V, H, std,
    seed)."""
    packed, scales, g = oracle.nvfp4_quantize(synth.weight(V, H, std, seed))
    return packed, scales, float(g)
