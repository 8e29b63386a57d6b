"""Writes oracle_cases.json: small fixed inputs and the CPU oracle's outputs for them.

The pages print no worked numeric example, so no fixture here comes from them. These cases are
chosen so that each output also has a closed form, which tests/test_golden.py checks
independently of the oracle. The file is a regression record of the oracle: a later change that
alters any of these values must say in its commit message which passage, or which reading of
it, justifies the change.

Run from the repository root:  python tests/golden/make_oracle_cases.py
Only oracle/ is called.
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))
import oracle  # noqa: E402


def bf16_bits(values):
    """bf16 bit patterns of values that bf16 holds exactly (checked)."""
    a = np.asarray(values, dtype=np.float32)
    bits = (a.view(np.uint32) >> 16).astype(np.uint16)
    back = (bits.astype(np.uint32) << 16).view(np.float32)
    assert np.array_equal(back, a), "value not exact in bf16"
    return bits


def main():
    cases = []
    # fp32 head: small integers, every sum exact; alpha = 1/4 exact.
    h = [[1, 2, 3, 4], [-1, 0, 5, -2]]
    w = [[1, 0, 0, 0], [0, 1, 1, 0], [2, -1, 3, 1], [0, 0, 0, 0], [-3, 4, -5, 6]]
    logits, _ = oracle.logits_f32(bf16_bits(h), bf16_bits(w), 0.25)
    cases.append({"kind": "logits_f32", "hidden": h, "W": w, "alpha": 0.25, "bias": None,
                  "logits": logits.tolist()})
    # fp32 head with a bias joining the sum before alpha: alpha * (h.w + b).
    b = [0.5, -1.0, 2.0, 0.25, -0.5]
    logits_b, _ = oracle.logits_f32(bf16_bits(h), bf16_bits(w), 0.5, bias_bits=bf16_bits(b))
    cases.append({"kind": "logits_f32", "hidden": h, "W": w, "alpha": 0.5, "bias": b,
                  "logits": logits_b.tolist()})
    # log-probabilities over all-zero logits: lse = log V, logprob = -log V.
    hz = [[1.0, -2.0, 0.5, 3.0]]
    wz = np.zeros((1000, 4)).tolist()
    lp, lse = oracle.logprobs_f32(bf16_bits(hz), bf16_bits(wz), 1.0, np.array([7], np.int32))
    cases.append({"kind": "logprobs_f32", "hidden": hz, "V": 1000, "W": "zeros", "alpha": 1.0,
                  "targets": [7], "logprobs": lp.tolist(), "lse": lse.tolist()})
    # NVFP4 quantiser: amax = 2688 makes g = 1; a block whose max is 6 has scale 1, so its
    # codes are the nearest E2M1 values of the elements themselves, ties to the even code.
    wq = np.zeros((2, 32))
    wq[0, 0] = 2688.0
    wq[1, :16] = [6, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, -0.25, -0.75, -2.5, -5, -0.0, 1, 3, -6]
    packed, scales, g = oracle.nvfp4_quantize(bf16_bits(wq))
    cases.append({"kind": "nvfp4_quantize", "W": wq.tolist(), "packed": packed.tolist(),
                  "scales": scales.tolist(), "g": float(g)})
    with open(os.path.join(HERE, "oracle_cases.json"), "w") as f:
        json.dump({"about": "CPU oracle outputs on fixed inputs; see make_oracle_cases.py",
                   "cases": cases}, f, indent=1)


if __name__ == "__main__":
    main()
