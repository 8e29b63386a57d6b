"""The binding's argument checks run before any call into the library: a tensor on another GPU than
the hidden rows (weights, bias, targets) is refused with ValueError, so the kernels never get a
pointer into another device's memory by mistake. The output buffers of the vocab-slice entry
are the exception by design (they may be peers' buffers mapped for peer access).

CPU only: stand-in CUDA tensors carry the attributes the checks read, and fail the test if the
wrapper ever asks for a data pointer (that is, gets as far as the library call)."""
import pytest
import torch

import fp32_accumulate_lm_b200 as lm


class ReachedTheLibrary(AssertionError):
    pass


class FakeCuda:
    def __init__(self, shape, dtype, dev=0):
        self.shape = torch.Size(shape)
        self.dtype = dtype
        self.device = torch.device("cuda", dev)
        self.is_cuda = True

    def dim(self):
        return len(self.shape)

    def is_contiguous(self):
        return True

    def numel(self):
        n = 1
        for d in self.shape:
            n *= d
        return n

    def element_size(self):
        return torch.empty((), dtype=self.dtype).element_size()

    def data_ptr(self):
        raise ReachedTheLibrary("the wrapper got as far as the library call")


BF16, F32, I32, U8 = torch.bfloat16, torch.float32, torch.int32, torch.uint8
R, H, V = 4, 64, 256


def inputs(w_dev=0, bias_dev=0, t_dev=0):
    return (FakeCuda((R, H), BF16), FakeCuda((V, H), BF16, w_dev), FakeCuda((V,), BF16, bias_dev),
            FakeCuda((R,), I32, t_dev))


def test_logits_refuse_weights_or_bias_on_another_gpu():
    h, w, b, _ = inputs(w_dev=1)
    with pytest.raises(ValueError, match="one device"):
        lm.logits_bf16_f32(h, w, out=FakeCuda((R, V), F32))
    with pytest.raises(ValueError, match="one device"):
        lm.logits_f32(h, w, bias=b, out=FakeCuda((R, V), F32))
    h, w, b, _ = inputs(bias_dev=1)
    with pytest.raises(ValueError, match="bias"):
        lm.logits_f32(h, w, bias=b, out=FakeCuda((R, V), F32))


def test_logprobs_refuse_inputs_on_another_gpu():
    out = (FakeCuda((R,), F32), FakeCuda((R,), F32))
    ws = FakeCuda((1 << 20,), U8)
    for kw, match in (({"w_dev": 1}, "one device"), ({"t_dev": 1}, "targets"),
                      ({"bias_dev": 1}, "bias")):
        h, w, b, t = inputs(**kw)
        with pytest.raises(ValueError, match=match):
            lm.logprobs_f32(h, w, t, bias=b, workspace=ws, out=out)
        with pytest.raises(ValueError, match=match):
            lm.logprobs_shard_stats_f32(h, w, 0, t, bias_shard=b, workspace=ws,
                                        out=FakeCuda((R, 3), F32))


def test_vocab_slice_refuses_weights_on_another_gpu_but_takes_peer_outputs():
    outs = [FakeCuda((R, 2 * V), F32, 0), FakeCuda((R, 2 * V), F32, 1)]
    h, w, b, _ = inputs(w_dev=1)
    with pytest.raises(ValueError, match="one device"):
        lm.logits_vocab_slice_f32(h, w, 0, outs)
    h, w, b, _ = inputs(bias_dev=1)
    with pytest.raises(ValueError, match="bias_slice"):
        lm.logits_vocab_slice_f32(h, w, 0, outs, bias_slice=b)
    # every check passes: the buffers on GPU 1 stand for a peer's, and the call goes ahead
    h, w, b, _ = inputs()
    with pytest.raises(ReachedTheLibrary):
        lm.logits_vocab_slice_f32(h, w, V, outs, bias_slice=b)
