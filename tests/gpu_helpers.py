"""Helpers for the GPU parity tests: move seeded numpy inputs to the device, call the library
through its C ABI, and bring the results back as numpy bit patterns."""
import numpy as np
import torch

import fp32_accumulate_lm_b200 as lm
import synth


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return synth.bits_to_torch_bf16(bits, "cuda")


def dev_u8(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).to("cuda")


def check_status():
    torch.cuda.synchronize()
    st = lm.device_status(clear=True)
    assert st == 0, f"device status word {st:#x}"


def gpu_bf16_f32(h, w, alpha: float) -> np.ndarray:
    """h, w: numpy bf16 bits or bf16 CUDA tensors. Returns fp32 logits as numpy."""
    hd = h if isinstance(h, torch.Tensor) else dev_bf16(h)
    wd = w if isinstance(w, torch.Tensor) else dev_bf16(w)
    out = lm.logits_bf16_f32(hd, wd, alpha)
    check_status()
    return out.cpu().numpy()


def gpu_nvfp4(h, packed, scales, g: float, alpha: float) -> np.ndarray:
    """Returns bf16 logits as numpy uint16 bits."""
    hd = h if isinstance(h, torch.Tensor) else dev_bf16(h)
    pd = packed if isinstance(packed, torch.Tensor) else dev_u8(packed)
    sd = scales if isinstance(scales, torch.Tensor) else dev_u8(scales)
    out = lm.logits_w4a16_nvfp4(hd, pd, sd, g, alpha)
    check_status()
    return out.view(torch.int16).cpu().numpy().view(np.uint16)


def f32_bits(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


def bf16_bits_of_f32(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)
