"""Seeded synthetic inputs for the LM head (hidden rows, bf16 and fp16 weights, biases, random
NVFP4 codes for timing).

This module makes data only; it holds none of the head's arithmetic (no products, sums, alpha,
output rounding or quantisation). Tests, the smoke run and the benchmark draw every input from
here, so both sides of a parity check see the same bits. It is not part of the library.

Recipe (the pages name no dataset; shapes and value distributions follow the workloads):
  * hidden[rows, H]  ~ N(0, 1) drawn in fp32 from a seeded ``torch.Generator``, rounded to bf16
    (round-to-nearest-even, ``Tensor.to(torch.bfloat16)``).
  * W[V, H]          ~ N(0, std) the same way (std 0.02, or 0.015 for the 4096-wide head).
  * NVFP4 test weights come from quantising such a bf16 W with the oracle's quantiser (the
    tests do that, not this module); timing runs use uniformly random codes and scales instead.

Arrays are returned as numpy (bf16 as uint16 bit patterns) unless a torch device is given.
"""
from __future__ import annotations

import numpy as np
import torch

# Seeds per workload: 1000 + index of the workload in the sweep (tiny, decode, spec-verify,
# prefill, NVFP4); sampled prefill rows use their own seed.
SEED_TINY = 1000
SEED_DECODE = 1001
SEED_SPEC = 1002
SEED_PREFILL = 1003
SEED_NVFP4 = 1004
SEED_PREFILL_SAMPLE = 2003
SEED_F16 = 1005
SEED_BIAS = 1006
BIAS_STD = 0.5  # embedding bias ~ N(0, 0.5), a few logit units like a trained head's bias

WORKLOADS = {
    # name: (rows list, H, V, weight std, alpha)
    "tiny": ([4, 1, 2, 3], 256, 1024, 0.02, 1.0 / 4),
    "decode": ([1, 2, 4, 8, 16, 32, 64], 2048, 151936, 0.02, 1.0 / 8),
    "spec_verify": ([128, 97, 32], 4096, 128256, 0.015, 1.0 / 16),
    "prefill": ([8192], 4096, 151936, 0.02, 1.0 / 8),
    "nvfp4": ([1, 16, 64, 65, 256], 2048, 151936, 0.02, 1.0 / 8),
    # the prefill shape computing log-probabilities of one target token per row (no logits out)
    "prefill_logprobs": ([8192], 4096, 151936, 0.02, 1.0 / 8),
    # the prefill log-probabilities with W's rows split over the GPUs (each holds one slice)
    "vocab_parallel_logprobs": ([8192], 4096, 151936, 0.02, 1.0 / 8),
    # the NVFP4 quantiser on the NVFP4 head's weight shape (rows = the V rows quantised per call)
    "nvfp4_quantize": ([151936], 2048, 151936, 0.02, 1.0),
    # the decode shape with fp16 operands and an fp16 embedding bias
    "decode_f16_bias": ([1, 2, 4, 8, 16, 32, 64], 2048, 151936, 0.02, 1.0 / 8),
    # profiling case: the prefill kernel and tile shape on 2048 rows (a few GB on the device)
    "prefill_2048": ([2048], 4096, 151936, 0.02, 1.0 / 8),
    # profiling case with two row-tile groups (16 + 2 tiles of 256 rows), as at 8192 rows
    "prefill_4608": ([4608], 4096, 151936, 0.02, 1.0 / 8),
    # profiling case of the log-prob mode: 2048 rows, one row-tile group
    "prefill_logprobs_2048": ([2048], 4096, 151936, 0.02, 1.0 / 8),
}


def _normal(shape, std: float, seed: int, device=None, dtype=torch.bfloat16) -> torch.Tensor:
    dev = torch.device(device) if device is not None else torch.device("cpu")
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    x = torch.randn(*shape, generator=gen, device=dev, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def _normal_bf16(shape, std: float, seed: int, device=None) -> torch.Tensor:
    return _normal(shape, std, seed, device, torch.bfloat16)


def _as_bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def hidden(rows: int, H: int, seed: int, device=None, dtype=torch.bfloat16):
    """hidden[rows, H] ~ N(0,1) in bf16 (or ``dtype``, e.g. torch.float16). numpy uint16 bits,
    or a tensor on ``device``."""
    t = _normal((rows, H), 1.0, seed, device, dtype)
    return t if device is not None else _as_bits(t)


def weight(V: int, H: int, std: float, seed: int, device=None, dtype=torch.bfloat16):
    """W[V, H] ~ N(0, std) in bf16 (or ``dtype``). numpy uint16 bits, or a tensor on ``device``."""
    t = _normal((V, H), std, seed + 500_000, device, dtype)
    return t if device is not None else _as_bits(t)


def bias(V: int, seed: int, device=None, dtype=torch.bfloat16, std: float = BIAS_STD):
    """Embedding bias[V] ~ N(0, std) in ``dtype``. numpy uint16 bits, or a tensor on ``device``."""
    t = _normal((V,), std, seed + 900_000, device, dtype)
    return t if device is not None else _as_bits(t)


def bits_to_torch(bits: np.ndarray, dtype, device="cpu") -> torch.Tensor:
    """uint16 bit patterns -> bf16 or fp16 tensor (a reinterpretation, no rounding)."""
    a = np.ascontiguousarray(bits, dtype=np.uint16)
    return torch.from_numpy(a.view(np.int16)).view(dtype).to(device)


def bits_to_torch_bf16(bits: np.ndarray, device="cpu") -> torch.Tensor:
    """uint16 bit patterns -> bf16 tensor (a reinterpretation, no rounding)."""
    a = np.ascontiguousarray(bits, dtype=np.uint16)
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def random_nvfp4_codes(V: int, H: int, seed: int, device=None):
    """Uniformly random E2M1 codes and finite non-negative E4M3 scales in [2^-4, 2^4]
    (for timing runs, where the value distribution does not matter)."""
    dev = torch.device(device) if device is not None else torch.device("cpu")
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    packed = torch.randint(0, 256, (V, H // 2), generator=gen, device=dev, dtype=torch.int32)
    sc = torch.randint(0x18, 0x58, (V, H // 16), generator=gen, device=dev, dtype=torch.int32)
    packed = packed.to(torch.uint8)
    sc = sc.to(torch.uint8)
    if device is None:
        return packed.numpy(), sc.numpy()
    return packed, sc
