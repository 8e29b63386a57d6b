"""The fp32 head's persistent units take the tiles after their first by cluster launch control
(one unit launched per tile; a running unit cancels the launch of the next pending one and
computes its tile instead), so tiles are taken in launch order by whichever units are free. The
schedule decides only who computes a tile and when: every output element is the same chain of
K = 16 MMA steps either way, so the dynamic schedule must give the static schedule's bits in
every mode, for single CTAs and CTA pairs, on ragged shapes and with more tiles than SMs. Row-count
invariance (lm_head_nvfp4_rows.rs, module doc) depends on that.

The library's test build switches to the static schedule (lmhead_debug_set_dynamic_tiles);
both sides run through the C ABI on the GPU, and one case per mode is checked against the CPU
oracle.
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


def _both(fn):
    """fn() with dynamic tiles, then with the static schedule; each result as numpy arrays."""
    out = []
    with lm.test_hooks():
        try:
            for enabled in (True, False):
                lm.set_dynamic_tiles(enabled)
                res = fn()
                check_status()
                out.append([r.cpu().numpy() for r in res])
        finally:
            lm.set_dynamic_tiles(True)
    return out


SHAPES = [
    (1, 256, 30000),       # one row tile, 235 v-tiles: more tiles than SMs
    (64, 512, 151936),     # the decode width, 1187 v-tiles
    (200, 320, 5000),      # single CTAs, 208-row tiles
    (300, 320, 2048 + 128),  # CTA pairs, ragged rows, the last pair's odd CTA empty
    (1000, 136, 40000),    # CTA pairs, 4 row tiles x 157 v-tiles, H not a multiple of 64
]


@pytest.mark.parametrize("rows,H,V", SHAPES)
def test_dynamic_tiles_give_static_bits(rows, H, V):
    seed = rows + H
    h = synth.hidden(rows, H, seed)
    w = synth.weight(V, H, 0.03, seed)
    b = synth.bias(V, seed)
    hd, wd = synth.bits_to_torch_bf16(h, "cuda"), synth.bits_to_torch_bf16(w, "cuda")
    bd = synth.bits_to_torch_bf16(b, "cuda")
    t = torch.from_numpy(np.random.default_rng(seed).integers(0, V, rows).astype(np.int32)).cuda()
    alpha = 0.125

    def calls():
        z = lm.logits_f32(hd, wd, alpha, bias=bd)
        lp, lse = lm.logprobs_f32(hd, wd, t, alpha, bias=bd)
        bufs = [torch.full((rows, V + 4), float("nan"), device="cuda") for _ in range(2)]
        lm.logits_vocab_slice_f32(hd, wd, 2, bufs, alpha, bias_slice=bd)
        return [z, lp, lse] + bufs

    dyn, sta = _both(calls)
    for a, b_ in zip(dyn, sta):
        assert np.array_equal(f32_bits(a), f32_bits(b_))
    assert np.array_equal(f32_bits(dyn[3][:, 2:2 + V]), f32_bits(dyn[0]))
    sample = np.unique(np.array([0, rows // 2, rows - 1]))
    ref, absum = oracle.logits_f32(h[sample], w, alpha, bias_bits=b)
    assert_fp32_close(dyn[0][sample], ref, absum, f"dynamic tiles {rows}x{H}x{V}")
