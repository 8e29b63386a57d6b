"""The fixed cases in tests/golden/oracle_cases.json (written by make_oracle_cases.py, which calls
only the oracle): the oracle still reproduces every stored value, and every stored value equals
its closed form, worked out here without the oracle.

The pages print no worked numeric example; the closed forms follow from the definitions they
give ("[Model] Honor fp32 head_dtype in Inkling muP logits (target + MTP draft)", "Purpose":
alpha times the projection, with the embedding bias inside; the log-softmax over the fp32 logits;
the quantiser rules this library reads for the absmax-then-encode pair of
lm_head_nvfp4_rows.rs).
"""
import json
import math
import os
from fractions import Fraction

import numpy as np

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


def load():
    with open(os.path.join(HERE, "golden", "oracle_cases.json")) as f:
        return json.load(f)["cases"]


def bf16_bits(values):
    a = np.asarray(values, dtype=np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


def test_oracle_reproduces_the_stored_cases():
    for c in load():
        if c["kind"] == "logits_f32":
            got, _ = oracle.logits_f32(bf16_bits(c["hidden"]), bf16_bits(c["W"]), c["alpha"],
                                       bias_bits=None if c["bias"] is None else
                                       bf16_bits(c["bias"]))
            assert np.array_equal(got, np.array(c["logits"], np.float32))
        elif c["kind"] == "logprobs_f32":
            w = np.zeros((c["V"], len(c["hidden"][0])), np.uint16)
            lp, lse = oracle.logprobs_f32(bf16_bits(c["hidden"]), w, c["alpha"],
                                          np.array(c["targets"], np.int32))
            assert np.array_equal(lp, np.array(c["logprobs"], np.float32))
            assert np.array_equal(lse, np.array(c["lse"], np.float32))
        else:
            p, s, g = oracle.nvfp4_quantize(bf16_bits(c["W"]))
            assert np.array_equal(p, np.array(c["packed"], np.uint8))
            assert np.array_equal(s, np.array(c["scales"], np.uint8))
            assert float(g) == c["g"]


def test_stored_head_values_are_the_exact_closed_forms():
    """Integer operands: alpha * (sum h w + b) is exact in fp32, so the stored value is it."""
    for c in (x for x in load() if x["kind"] == "logits_f32"):
        a = Fraction(c["alpha"])
        for r, hr in enumerate(c["hidden"]):
            for v, wv in enumerate(c["W"]):
                acc = sum(Fraction(x) * Fraction(y) for x, y in zip(hr, wv))
                if c["bias"] is not None:
                    acc += Fraction(c["bias"][v])
                assert Fraction(c["logits"][r][v]) == a * acc, (r, v)


def test_stored_logprobs_of_uniform_logits_are_minus_log_v():
    (c,) = [x for x in load() if x["kind"] == "logprobs_f32"]
    assert c["lse"][0] == float(np.float32(math.log(c["V"])))
    assert c["logprobs"][0] == float(np.float32(-math.log(c["V"])))


def test_stored_quantiser_codes_follow_the_rules_by_hand():
    """amax = 2688 gives g = 1. Row 0: the block holding 2688 has scale 448 (E4M3 code 0x7E) and
    code 6 (0x7) there; all-zero blocks have scale code 0 and codes 0. Row 1: the block whose
    max is 6 has scale 1 (code 0x38), so each code is the nearest E2M1 value of the element,
    ties to the even code, with no negative zero."""
    (c,) = [x for x in load() if x["kind"] == "nvfp4_quantize"]
    assert c["g"] == 1.0
    assert c["scales"] == [[0x7E, 0x00], [0x38, 0x00]]
    row1 = [0x7, 0x0, 0x2, 0x2, 0x4, 0x4, 0x6, 0x6, 0x0, 0xA, 0xC, 0xE, 0x0, 0x2, 0x5, 0xF]
    want1 = [row1[2 * j] | (row1[2 * j + 1] << 4) for j in range(8)] + [0] * 8
    want0 = [0x7] + [0] * 15
    assert c["packed"] == [want0, want1]
