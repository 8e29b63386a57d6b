"""Full 256-row tiles of the fp32 head run on CTA pairs (cta_group::2 MMAs, 256 vocab rows per
tile, each CTA loading its 128 W rows and half the hidden rows). A pair computes every output
element with the same chain of K = 16 MMA steps as a lone CTA, so the pair tiles must give the
lone-CTA tiles' bits exactly, with and without bias, in fp16, into several vocab-slice buffers,
on ragged shapes, and when V leaves the last pair's odd CTA with some or none of the vocab rows
(V mod 256 in {0, 1..128, 129..255}). The log-prob modes keep lone CTAs. Row-count invariance
(lm_head_nvfp4_rows.rs, module doc) is what this guards: calls below 241 rows use lone CTAs.

The library's test build switches the pair tiles off (lmhead_debug_set_cta_pairs); both sides
of every comparison run through the C ABI on the GPU, and one case per mode is also checked
against the CPU oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import fp32_accumulate_lm_b200 as lm
import synth
from gpu_helpers import check_status, f32_bits
from tolerance import assert_fp32_close

pytestmark = pytest.mark.gpu

TDT = {"bf16": torch.bfloat16, "f16": torch.float16}


def _inputs(rows, H, V, seed, dtype, with_bias):
    h = synth.hidden(rows, H, seed, dtype=TDT[dtype])
    w = synth.weight(V, H, 0.05, seed, dtype=TDT[dtype])
    b = synth.bias(V, seed, dtype=TDT[dtype]) if with_bias else None
    t = np.random.default_rng(seed).integers(0, V, rows).astype(np.int32)
    dev = lambda a: None if a is None else synth.bits_to_torch(a, TDT[dtype], "cuda")
    return (h, w, b, t), (dev(h), dev(w), dev(b), torch.from_numpy(t).cuda())


def _both(fn):
    """fn() with the pair tiles on, then off; each result as numpy arrays."""
    out = []
    with lm.test_hooks():
        try:
            for enabled in (True, False):
                lm.set_cta_pairs(enabled)
                res = fn()
                check_status()
                out.append([r.cpu().numpy() for r in res])
        finally:
            lm.set_cta_pairs(True)
    return out


SHAPES = [
    (256, 64, 256),      # one pair tile, V a multiple of 256
    (257, 136, 300),     # ragged rows (a second row tile of 1), V mod 256 = 44: odd CTA empty
    (300, 200, 1000),    # V mod 256 = 232: odd CTA of the last pair partly filled
    (513, 72, 129),      # one pair v-tile, odd CTA holds one row; H not a multiple of 64
    (600, 320, 2048 + 128),  # V mod 256 = 128: the odd CTA of the last pair empty
    (256, 64, 1),        # one vocab row: the only pair's odd CTA holds nothing
    (241, 136, 128),     # the fewest rows that make a 256-row tile; V = 128: odd CTA empty
]


@pytest.mark.parametrize("rows,H,V", SHAPES)
@pytest.mark.parametrize("dtype,with_bias", [("bf16", False), ("bf16", True), ("f16", False)])
def test_pair_tiles_give_lone_cta_bits(rows, H, V, dtype, with_bias):
    (h, w, b, _), (hd, wd, bd, _) = _inputs(rows, H, V, rows + H + V, dtype, with_bias)
    alpha = 1.0 / 3.0
    on, off = _both(lambda: [lm.logits_f32(hd, wd, alpha, bias=bd)])
    assert np.array_equal(f32_bits(on[0]), f32_bits(off[0]))
    if (rows, H, V) == SHAPES[2]:
        ref, absum = oracle.logits_f32(h, w, alpha, bias_bits=b, dtype=dtype)
        assert_fp32_close(on[0], ref, absum, f"pair tiles {dtype} bias={with_bias}")


@pytest.mark.parametrize("rows,H,V", SHAPES)
def test_pair_tiles_vocab_slice_copies_and_logprob_modes(rows, H, V):
    """The vocab-slice entry's copies (two buffers, the slice at column 3 of rows of V + 10
    floats) are the pair tiles' bits with or without pairs; the log-prob modes, which keep lone
    CTAs, are unchanged by the switch."""
    (h, w, b, t), (hd, wd, bd, td) = _inputs(rows, H, V, 7 * rows + V, "bf16", True)
    alpha = 0.125

    def calls():
        bufs = [torch.full((rows, V + 10), float("nan"), device="cuda") for _ in range(2)]
        lm.logits_vocab_slice_f32(hd, wd, 3, bufs, alpha, bias_slice=bd)
        lp, lse = lm.logprobs_f32(hd, wd, td, alpha, bias=bd)
        stats = lm.logprobs_shard_stats_f32(hd, wd, 1000, td + 1000, alpha, bias_shard=bd)
        return bufs + [lp, lse, stats]

    on, off = _both(calls)
    for a, b_ in zip(on, off):
        assert np.array_equal(f32_bits(a), f32_bits(b_))
    whole = lm.logits_f32(hd, wd, alpha, bias=bd).cpu().numpy()
    for buf in on[:2]:
        assert np.array_equal(f32_bits(buf[:, 3:3 + V]), f32_bits(whole))
        assert np.isnan(buf[:, :3]).all() and np.isnan(buf[:, 3 + V:]).all()
    assert np.all(np.isfinite(on[2])) and np.all(on[2] <= 1e-6)
