"""The quantiser entry point that allocates nothing (lmhead_nvfp4_quantize_noalloc).

It serves callers that get their device buffers from another component and may not call
cudaMalloc themselves, so they cannot pass the quantiser a workspace; the library's own 4 KB
per-GPU scratch takes its place. Its results must be the workspace entry's, bit for bit, on
calls in a row that share the scratch, a later call writing fewer words than an earlier one.

This file sorts last so that a run stopping at its first failure has run every other test.
"""
import pytest
import torch

import fp32_accumulate_lm_b200 as lm
import synth

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


def absmax_grid(V, H):
    """CTAs of the quantiser's absmax pass, each writing one word of the scratch: a few per SM,
    no more than the work needs, at most the 1024 words the scratch holds."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    return min(6 * sms, -(-(V * H // 8) // 256), 1024)


def test_matches_the_workspace_entry_on_two_calls_in_a_row():
    """Consecutive calls share the scratch. The first writes many partial maxima of a large
    amax; the later ones write fewer words of smaller amaxes. If a later call read any word it
    did not write itself, its global scale (and then its codes) would come from the first
    call's amax and differ from the workspace entry's."""
    calls = [(151936 // 8, 2048, 0.2, 91), (16, 64, 0.01, 92), (300, 2048, 0.005, 93)]
    grids = [absmax_grid(V, H) for V, H, _, _ in calls]
    assert grids[0] > grids[1] and grids[0] > grids[2]
    for V, H, std, seed in calls:
        W = synth.weight(V, H, std, seed, device="cuda")
        got = quantize_without_allocation(W)
        torch.cuda.synchronize()
        want = quantize_with_workspace(W)
        torch.cuda.synchronize()
        assert lm.device_status(clear=True) == 0
        for a, b in zip(got, want):
            assert torch.equal(a, b), (V, H)
    # and again in the order small, large: each call's result depends on its own inputs only
    for V, H, std, seed in reversed(calls):
        W = synth.weight(V, H, std, seed, device="cuda")
        got = quantize_without_allocation(W)
        want = quantize_with_workspace(W)
        torch.cuda.synchronize()
        for a, b in zip(got, want):
            assert torch.equal(a, b), (V, H)


def test_rejects_bad_arguments_before_touching_the_device():
    A = 0x10000
    f = lm.lmhead_nvfp4_quantize_noalloc
    assert f(A, 0, 64, A * 2, A * 3, A * 4, 0) == 2
    assert f(A, 4, 40, A * 2, A * 3, A * 4, 0) == 3
    assert f(0, 4, 64, A * 2, A * 3, A * 4, 0) == 1
    assert f(A + 8, 4, 64, A * 2, A * 3, A * 4, 0) == 3           # misaligned W
    assert f(A, 4, 64, A * 2, A * 2 + 64, A * 4, 0) == 7          # scales over the codes
    assert f(A, 2 ** 31, 64, A * 2, A * 3, A * 4, 0) == 2         # V past int32
