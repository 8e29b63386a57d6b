"""The quantiser entry point that allocates nothing (lmhead_nvfp4_quantize_noalloc).

It serves callers that get their device buffers from another component and may not call
cudaMalloc themselves, so they cannot pass the quantiser a workspace; the library's own 4 KB
per-GPU scratch takes its place. Its results must be the workspace entry's, bit for bit, on two
calls in a row (the second call finds the first one's leftovers in the shared scratch).

This file sorts last so that a run stopping at its first failure has run every other test.
"""
import pytest
import torch

import fp32_accumulate_lm_b200 as lm
from fp32_accumulate_lm_b200 import synth

pytestmark = pytest.mark.gpu


def outputs(V, H):
    return (torch.empty((V, H // 2), dtype=torch.uint8, device="cuda"),
            torch.empty((V, H // 16), dtype=torch.uint8, device="cuda"),
            torch.empty((1,), dtype=torch.float32, device="cuda"))


def quantize_with_workspace(W):
    V, H = W.shape
    p, s, g = outputs(V, H)
    ws = torch.empty(lm.nvfp4_quantize_workspace_bytes(), dtype=torch.uint8, device="cuda")
    st = lm.lmhead_nvfp4_quantize(W.data_ptr(), V, H, p.data_ptr(), s.data_ptr(), g.data_ptr(),
                                  ws.data_ptr(), ws.numel(), torch.cuda.current_stream().cuda_stream)
    assert st == 0
    return p, s, g


def quantize_without_allocation(W):
    V, H = W.shape
    p, s, g = outputs(V, H)
    st = lm.lmhead_nvfp4_quantize_noalloc(W.data_ptr(), V, H, p.data_ptr(), s.data_ptr(),
                                          g.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == 0
    return p, s, g


def test_matches_the_workspace_entry_on_two_calls_in_a_row():
    shapes = [(151936 // 8, 2048, 91), (513, 4096, 92)]
    for V, H, seed in shapes:      # two calls, different shapes and amax, sharing the scratch
        W = synth.weight(V, H, 0.02 * (1 + seed % 3), seed, device="cuda")
        got = quantize_without_allocation(W)
        want = quantize_with_workspace(W)
        torch.cuda.synchronize()
        assert lm.device_status(clear=True) == 0
        for a, b in zip(got, want):
            assert torch.equal(a, b), (V, H)


def test_rejects_bad_arguments_before_touching_the_device():
    A = 0x10000
    f = lm.lmhead_nvfp4_quantize_noalloc
    assert f(A, 0, 64, A * 2, A * 3, A * 4, 0) == 2
    assert f(A, 4, 40, A * 2, A * 3, A * 4, 0) == 3
    assert f(0, 4, 64, A * 2, A * 3, A * 4, 0) == 1
