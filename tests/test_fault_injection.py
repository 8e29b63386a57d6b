"""Failure detection without a GPU fault: with loads starved on the host side, the kernels'
consumers wait on barriers that never complete; each bounded wait must give up after its limit,
record LMHEAD_ERR_TIMEOUT in the device status word and return, leaving the context usable."""
import time

import numpy as np
import pytest
import torch

import fp32_accumulate_lm_b200 as lm
import synth
from gpu_helpers import dev_bf16, dev_u8, gpu_bf16_f32
from oracle_inputs import nvfp4_weights

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("entry,rows,V", [
    ("bf16", 8, 512),
    # many more tiles than SMs: units that gave up leave launches pending, which then start,
    # take no tile answers of their own and give up as well
    ("bf16", 8, 151936),
    # CTA pairs (256-row tiles) with their dynamic tiles: both CTAs of a pair give up
    ("bf16", 300, 2048),
    ("nvfp4", 8, 512),
])
def test_starved_loads_time_out_cleanly(entry, rows, V):
    H = 128
    h = dev_bf16(synth.hidden(rows, H, 1))
    w = dev_bf16(synth.weight(V, H, 0.02, 1))
    packed, scales, g = nvfp4_weights(V, H, 0.02, 1)
    pd, sd = dev_u8(packed), dev_u8(scales)
    torch.cuda.synchronize()
    with lm.test_hooks():           # the knob exists only in the test build (same kernels)
        lm.device_status(clear=True)
        lm.set_fault_injection(True, wait_limit_ns=20_000_000)  # 20 ms per wait
        try:
            t0 = time.time()
            if entry == "bf16":
                lm.logits_bf16_f32(h, w, 1.0)
            else:
                lm.logits_w4a16_nvfp4(h, pd, sd, g, 1.0)
            torch.cuda.synchronize()
            elapsed = time.time() - t0
        finally:
            lm.set_fault_injection(False, 0)
        st = lm.device_status(clear=True)
        assert st & 0xFF == lm.LMHEAD_ERR_TIMEOUT, hex(st)
        assert (st >> 8) & 0xFF in (1, 2, 3, 4, 5)
        assert elapsed < 10.0
        assert lm.device_status() == 0
        # the context is still usable and the next call is correct
        out = gpu_bf16_f32(synth.hidden(2, 64, 2), np.zeros((16, 64), np.uint16), 1.0)
        assert np.all(out == 0)


def test_check_raises_on_a_timed_out_call():
    """A call whose kernel gave up returned LMHEAD_OK before it ran; the wrappers' check=True
    (lmhead_stream_status underneath) must turn the recorded timeout into an exception, and the
    next checked call must pass."""
    h = dev_bf16(synth.hidden(4, 128, 3))
    w = dev_bf16(synth.weight(300, 128, 0.02, 3))
    torch.cuda.synchronize()
    with lm.test_hooks():
        lm.device_status(clear=True)
        lm.set_fault_injection(True, wait_limit_ns=20_000_000)
        try:
            with pytest.raises(lm.LmheadError) as e:
                lm.logits_bf16_f32(h, w, 1.0, check=True)
            assert e.value.status == lm.LMHEAD_ERR_TIMEOUT
        finally:
            lm.set_fault_injection(False, 0)
        out = lm.logits_bf16_f32(h, w, 1.0, check=True)
        assert lm.stream_status() == 0
    assert torch.isfinite(out).all()
