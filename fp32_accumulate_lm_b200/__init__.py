"""B200 (sm_100a) LM-head logits projection: Python binding of the C ABI in include/lmhead.h.

    logits[rows, V] = alpha * (hidden[rows, H] @ W[V, H]^T)

``logits_bf16_f32`` takes bf16 operands and returns fp32 logits (fp32 accumulation, alpha folded
into the epilogue -- "[Model] Honor fp32 head_dtype in Inkling muP logits (target + MTP draft)",
"muP is folded into the fp32 GEMM"); ``logits_w4a16_nvfp4`` is the W4A16 NVFP4 head with bf16
logits (lm_head_nvfp4_rows.rs, lm_head_nvfp4_rows_run).

This module only marshals arguments: every step of the computation runs in the CUDA library
``liblmhead.so`` built in-tree by ``fp32_accumulate_lm_b200._build``. If that library is
missing or fails to load, every call raises; there is no other code path.

Calls are asynchronous. A kernel that gives up on one of its bounded waits records a timeout in
a per-device status word instead of faulting; pass ``check=True`` to a wrapper (or call
``check(stream)``) to synchronise and raise ``LmheadError`` if that happened.

``test_hooks()`` routes every call to ``liblmhead_test.so`` (the same kernels plus two
host-side test knobs, see ``set_fault_injection`` and ``set_nvfp4_conversion``); only the tests
use it.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import threading

__all__ = [
    "LmheadError", "load_library", "library_path", "logits_bf16_f32", "logits_f32", "logprobs_f32",
    "lmhead_logprobs_f32", "logprobs_workspace_bytes", "lmhead_logprobs_shard_stats_f32",
    "lmhead_logprobs_merge_shards", "logprobs_shard_stats_f32", "logprobs_merge_shards",
    "vocab_shard", "gather_shard_stats", "logprobs_vocab_parallel",
    "logits_w4a16_nvfp4", "lmhead_logits_bf16_f32", "lmhead_logits_f32",
    "lmhead_logits_w4a16_nvfp4", "lmhead_nvfp4_quantize", "lmhead_nvfp4_quantize_noalloc",
    "nvfp4_quantize",
    "nvfp4_quantize_workspace_bytes", "status_string", "device_status", "DTYPE_BF16", "DTYPE_F16",
    "version", "set_fault_injection", "set_nvfp4_conversion", "STATUS", "lmhead_stream_status",
    "stream_status", "check", "test_hooks", "load_test_library",
]

STATUS = {
    0: "LMHEAD_OK", 1: "LMHEAD_ERR_NULL", 2: "LMHEAD_ERR_SHAPE", 3: "LMHEAD_ERR_ALIGN",
    4: "LMHEAD_ERR_ARCH", 5: "LMHEAD_ERR_LAUNCH", 6: "LMHEAD_ERR_TIMEOUT", 7: "LMHEAD_ERR_ALIAS",
}
LMHEAD_OK = 0
LMHEAD_ERR_TIMEOUT = 6
DTYPE_BF16 = 0  # lmhead_dtype
DTYPE_F16 = 1

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liblmhead.so")
_TEST_LIB_PATH = os.path.join(_HERE, "liblmhead_test.so")
_lock = threading.Lock()
_lib = None
_test_lib = None
_use_test = False


class LmheadError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)} ({status_string(status)})")


def library_path() -> str:
    return _LIB_PATH


def _bind(lib, test: bool):
    vp, i64, f32, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_int
    lib.lmhead_logits_bf16_f32.argtypes = [vp, i64, i64, vp, i64, f32, vp, vp]
    lib.lmhead_logits_bf16_f32.restype = i32
    lib.lmhead_logits_f32.argtypes = [vp, i32, i64, i64, vp, i64, f32, vp, vp, vp]
    lib.lmhead_logits_f32.restype = i32
    lib.lmhead_logprobs_workspace_bytes.argtypes = [i64, i64]
    lib.lmhead_logprobs_workspace_bytes.restype = ctypes.c_size_t
    lib.lmhead_logprobs_f32.argtypes = [vp, i32, i64, i64, vp, i64, f32, vp, vp, vp, vp, vp,
                                        ctypes.c_size_t, vp]
    lib.lmhead_logprobs_f32.restype = i32
    lib.lmhead_logprobs_shard_stats_f32.argtypes = [vp, i32, i64, i64, vp, i64, i64, f32, vp,
                                                    vp, vp, vp, ctypes.c_size_t, vp]
    lib.lmhead_logprobs_shard_stats_f32.restype = i32
    lib.lmhead_logprobs_merge_shards.argtypes = [vp, i64, i64, vp, vp, vp]
    lib.lmhead_logprobs_merge_shards.restype = i32
    lib.lmhead_logits_vocab_slice_f32.argtypes = [vp, i32, i64, i64, vp, i64, i64, f32, vp,
                                                  ctypes.POINTER(vp), i32, i64, vp]
    lib.lmhead_logits_vocab_slice_f32.restype = i32
    lib.lmhead_logits_w4a16_nvfp4.argtypes = [vp, i64, i64, vp, vp, f32, i64, f32, vp, vp]
    lib.lmhead_logits_w4a16_nvfp4.restype = i32
    lib.lmhead_nvfp4_quantize_workspace_bytes.argtypes = []
    lib.lmhead_nvfp4_quantize_workspace_bytes.restype = ctypes.c_size_t
    lib.lmhead_nvfp4_quantize.argtypes = [vp, i64, i64, vp, vp, vp, vp, ctypes.c_size_t, vp]
    lib.lmhead_nvfp4_quantize.restype = i32
    lib.lmhead_nvfp4_quantize_noalloc.argtypes = [vp, i64, i64, vp, vp, vp, vp]
    lib.lmhead_nvfp4_quantize_noalloc.restype = i32
    lib.lmhead_status_string.argtypes = [i32]
    lib.lmhead_status_string.restype = ctypes.c_char_p
    lib.lmhead_device_status.argtypes = [i32]
    lib.lmhead_device_status.restype = i32
    lib.lmhead_stream_status.argtypes = [vp]
    lib.lmhead_stream_status.restype = i32
    lib.lmhead_version.argtypes = []
    lib.lmhead_version.restype = i32
    if test:
        lib.lmhead_debug_set_fault_injection.argtypes = [i32, ctypes.c_uint64]
        lib.lmhead_debug_set_fault_injection.restype = None
        lib.lmhead_debug_set_nvfp4_conversion.argtypes = [i32]
        lib.lmhead_debug_set_nvfp4_conversion.restype = None
        lib.lmhead_debug_set_cta_pairs.argtypes = [i32]
        lib.lmhead_debug_set_cta_pairs.restype = None
        lib.lmhead_debug_set_dynamic_tiles.argtypes = [i32]
        lib.lmhead_debug_set_dynamic_tiles.restype = None
    return lib


def load_library():
    """Load liblmhead.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                               "`python -m fp32_accumulate_lm_b200._build`")
        _lib = _bind(ctypes.CDLL(_LIB_PATH), test=False)
        return _lib


def load_test_library():
    """Load liblmhead_test.so, the test build (raises if it has not been built)."""
    global _test_lib
    with _lock:
        if _test_lib is not None:
            return _test_lib
        if not os.path.exists(_TEST_LIB_PATH):
            raise RuntimeError(f"{_TEST_LIB_PATH} is missing: build it with "
                               "`python -m fp32_accumulate_lm_b200._build`")
        _test_lib = _bind(ctypes.CDLL(_TEST_LIB_PATH), test=True)
        return _test_lib


def _active():
    return load_test_library() if _use_test else load_library()


@contextlib.contextmanager
def test_hooks():
    """Route every call of this module to the test build for the duration (tests only). The test
    build has its own per-device status word; read it inside the block."""
    global _use_test
    load_test_library()
    prev = _use_test
    _use_test = True
    try:
        yield load_test_library()
    finally:
        _use_test = prev


# ---------------------------------------------------------------- raw C-ABI (integers in, status out)

def lmhead_logits_bf16_f32(hidden_ptr: int, rows: int, H: int, w_ptr: int, V: int, alpha: float,
                           logits_ptr: int, stream: int = 0) -> int:
    return _active().lmhead_logits_bf16_f32(hidden_ptr, rows, H, w_ptr, V, alpha,
                                                  logits_ptr, stream)


def lmhead_logits_f32(hidden_ptr: int, dtype: int, rows: int, H: int, w_ptr: int, V: int,
                      alpha: float, bias_ptr: int, logits_ptr: int, stream: int = 0) -> int:
    return _active().lmhead_logits_f32(hidden_ptr, dtype, rows, H, w_ptr, V, alpha,
                                             bias_ptr or None, logits_ptr, stream)


def logprobs_workspace_bytes(rows: int, V: int) -> int:
    return int(_active().lmhead_logprobs_workspace_bytes(rows, V))


def lmhead_logprobs_f32(hidden_ptr: int, dtype: int, rows: int, H: int, w_ptr: int, V: int,
                        alpha: float, bias_ptr: int, targets_ptr: int, logprobs_ptr: int,
                        lse_ptr: int, workspace_ptr: int, workspace_bytes: int,
                        stream: int = 0) -> int:
    return _active().lmhead_logprobs_f32(hidden_ptr, dtype, rows, H, w_ptr, V, alpha,
                                               bias_ptr or None, targets_ptr, logprobs_ptr,
                                               lse_ptr or None, workspace_ptr, workspace_bytes,
                                               stream)


def lmhead_logprobs_shard_stats_f32(hidden_ptr: int, dtype: int, rows: int, H: int,
                                    w_shard_ptr: int, V_shard: int, v_begin: int, alpha: float,
                                    bias_shard_ptr: int, targets_ptr: int, stats_ptr: int,
                                    workspace_ptr: int, workspace_bytes: int,
                                    stream: int = 0) -> int:
    return _active().lmhead_logprobs_shard_stats_f32(
        hidden_ptr, dtype, rows, H, w_shard_ptr, V_shard, v_begin, alpha, bias_shard_ptr or None,
        targets_ptr, stats_ptr, workspace_ptr, workspace_bytes, stream)


def lmhead_logprobs_merge_shards(stats_ptr: int, shards: int, rows: int, logprobs_ptr: int,
                                 lse_ptr: int, stream: int = 0) -> int:
    return _active().lmhead_logprobs_merge_shards(stats_ptr, shards, rows, logprobs_ptr,
                                                       lse_ptr or None, stream)


def lmhead_logits_vocab_slice_f32(hidden_ptr: int, dtype: int, rows: int, H: int,
                                  w_slice_ptr: int, V_slice: int, v_begin: int, alpha: float,
                                  bias_slice_ptr: int, logits_ptrs, ld_logits: int,
                                  stream: int = 0) -> int:
    """logits_ptrs: a sequence of device addresses (ints); passed as a host array."""
    n = len(logits_ptrs)
    arr = (ctypes.c_void_p * max(n, 1))(*[p or None for p in logits_ptrs])
    return _active().lmhead_logits_vocab_slice_f32(
        hidden_ptr, dtype, rows, H, w_slice_ptr, V_slice, v_begin, alpha, bias_slice_ptr or None,
        arr if n else None, n, ld_logits, stream)


def lmhead_logits_w4a16_nvfp4(hidden_ptr: int, rows: int, H: int, packed_ptr: int,
                              scales_ptr: int, w_global_scale: float, V: int, alpha: float,
                              logits_ptr: int, stream: int = 0) -> int:
    return _active().lmhead_logits_w4a16_nvfp4(hidden_ptr, rows, H, packed_ptr, scales_ptr,
                                                     w_global_scale, V, alpha, logits_ptr, stream)


def nvfp4_quantize_workspace_bytes() -> int:
    return int(_active().lmhead_nvfp4_quantize_workspace_bytes())


def lmhead_nvfp4_quantize(w_ptr: int, V: int, H: int, packed_ptr: int, scales_ptr: int,
                          g_ptr: int, workspace_ptr: int, workspace_bytes: int,
                          stream: int = 0) -> int:
    return _active().lmhead_nvfp4_quantize(w_ptr, V, H, packed_ptr, scales_ptr, g_ptr,
                                                workspace_ptr, workspace_bytes, stream)


def lmhead_nvfp4_quantize_noalloc(w_ptr: int, V: int, H: int, packed_ptr: int, scales_ptr: int,
                                  g_ptr: int, stream: int = 0) -> int:
    """The quantiser for callers that cannot allocate device memory: the library's own 4 KB
    per-GPU scratch replaces the workspace (see include/lmhead.h)."""
    return _active().lmhead_nvfp4_quantize_noalloc(w_ptr, V, H, packed_ptr, scales_ptr,
                                                        g_ptr, stream)


def nvfp4_quantize(W, workspace=None, out=None, stream=None, check: bool = False):
    """Quantise a bf16 CUDA tensor W [V, H] (H % 16 == 0) for the NVFP4 head. Returns (packed uint8
    [V, H/2], scales uint8 [V, H/16], g: fp32 CUDA tensor of one element), all on W's device;
    runs asynchronously on ``stream``. ``workspace`` (a CUDA tensor of at least
    nvfp4_quantize_workspace_bytes() bytes) is allocated here when not given, and so are the
    outputs unless ``out`` = (packed, scales, g) supplies them."""
    import torch
    _check(W.dtype == torch.bfloat16 and W.dim() == 2 and W.is_cuda and W.is_contiguous(),
           "a contiguous bf16 CUDA matrix is required")
    V, H = W.shape
    if out is None:
        packed = torch.empty((V, H // 2), dtype=torch.uint8, device=W.device)
        scales = torch.empty((V, H // 16), dtype=torch.uint8, device=W.device)
        g = torch.empty((1,), dtype=torch.float32, device=W.device)
    else:
        packed, scales, g = out
        _check_out(packed, torch.uint8, (V, H // 2), W.device, "out[0] (packed codes)")
        _check_out(scales, torch.uint8, (V, H // 16), W.device, "out[1] (block scales)")
        _check_out(g, torch.float32, (1,), W.device, "out[2] (global scale)")
    need = nvfp4_quantize_workspace_bytes()
    if workspace is None:
        workspace = torch.empty((need,), dtype=torch.uint8, device=W.device)
    _check(workspace.is_cuda and workspace.is_contiguous() and workspace.device == W.device,
           "workspace must be a contiguous CUDA tensor on W's device")
    nbytes = workspace.numel() * workspace.element_size()
    st = lmhead_nvfp4_quantize(W.data_ptr(), V, H, packed.data_ptr(), scales.data_ptr(),
                               g.data_ptr(), workspace.data_ptr(), nbytes, _stream_handle(stream))
    _finish(st, "lmhead_nvfp4_quantize", check, stream)
    return packed, scales, g


def status_string(status: int) -> str:
    try:
        return _active().lmhead_status_string(int(status)).decode()
    except RuntimeError:
        return STATUS.get(status, "unknown status")


def device_status(clear: bool = False) -> int:
    """Status word of the current device (0, or LMHEAD_ERR_TIMEOUT | role << 8). Does not
    synchronise: read it after the work of interest has finished."""
    return _active().lmhead_device_status(1 if clear else 0)


def lmhead_stream_status(stream: int = 0) -> int:
    return _active().lmhead_stream_status(stream)


def stream_status(stream=None) -> int:
    """Synchronise ``stream`` (default: torch's current stream), then return and clear the
    device's status word (0 when no kernel wait ran out)."""
    return lmhead_stream_status(_stream_handle(stream))


def check(stream=None) -> None:
    """Synchronise ``stream`` and raise LmheadError if a kernel of this device gave up on one of
    its waits since the last check (its outputs are undefined) or the stream reported an error."""
    st = stream_status(stream)
    if st != LMHEAD_OK:
        raise LmheadError(st & 0xFF, f"kernel status word {st:#x} (role {(st >> 8) & 0xFF})")


def version() -> int:
    return _active().lmhead_version()


def set_nvfp4_conversion(path: int) -> None:
    """Test build only (inside ``test_hooks()``): 1 pair table, 2 integer spreading, 0 automatic
    (the same bits either way)."""
    _require_test_build("set_nvfp4_conversion")
    _active().lmhead_debug_set_nvfp4_conversion(int(path))


def set_cta_pairs(enabled: bool) -> None:
    """Test build only (inside ``test_hooks()``): whether the fp32 head may run full 256-row
    tiles on CTA pairs (the default) or keeps every tile on one CTA (the same bits either way)."""
    _require_test_build("set_cta_pairs")
    _active().lmhead_debug_set_cta_pairs(1 if enabled else 0)


def set_dynamic_tiles(enabled: bool) -> None:
    """Test build only (inside ``test_hooks()``): whether the fp32 head's units take their later
    tiles by cluster launch control (the default) or follow the static schedule (the same bits
    either way)."""
    _require_test_build("set_dynamic_tiles")
    _active().lmhead_debug_set_dynamic_tiles(1 if enabled else 0)


def set_fault_injection(starve_loads: bool, wait_limit_ns: int = 0) -> None:
    """Test build only (inside ``test_hooks()``): make launches issue no loads, so their waits
    time out after wait_limit_ns."""
    _require_test_build("set_fault_injection")
    _active().lmhead_debug_set_fault_injection(1 if starve_loads else 0, int(wait_limit_ns))


def _require_test_build(what: str):
    if not _use_test:
        raise RuntimeError(f"{what} exists only in the test build: call it inside "
                           "fp32_accumulate_lm_b200.test_hooks()")


# ---------------------------------------------------------------- torch-tensor convenience wrappers

def _stream_handle(stream) -> int:
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(cond: bool, msg: str):
    if not cond:
        raise ValueError(msg)


def _check_out(t, dtype, shape, device, what: str):
    """A caller-supplied output must be a contiguous CUDA tensor of this dtype and shape on the
    inputs' device: the kernels write exactly that many elements and check nothing."""
    _check(t is not None and t.dtype == dtype and t.is_cuda and t.is_contiguous()
           and tuple(t.shape) == tuple(shape) and t.device == device,
           f"{what} must be a contiguous {dtype} CUDA tensor of shape {tuple(shape)} on {device}")


def _finish(st: int, what: str, check_after: bool, stream):
    if st != LMHEAD_OK:
        raise LmheadError(st, what)
    if check_after:
        check(stream)


def logits_bf16_f32(hidden, W, alpha: float = 1.0, out=None, stream=None, check: bool = False):
    """fp32 logits[rows, V] = alpha * hidden @ W^T for bf16 CUDA tensors hidden [rows, H] and
    W [V, H]. Runs asynchronously on ``stream`` (default: torch's current stream); with
    ``check`` it synchronises and raises if a kernel wait timed out."""
    import torch
    _check(hidden.dtype == torch.bfloat16 and W.dtype == torch.bfloat16, "bf16 operands required")
    _check(hidden.dim() == 2 and W.dim() == 2 and hidden.shape[1] == W.shape[1], "shape mismatch")
    _check(hidden.is_cuda and W.is_cuda, "CUDA tensors required")
    _check(hidden.is_contiguous() and W.is_contiguous(), "contiguous tensors required")
    rows, H = hidden.shape
    V = W.shape[0]
    if out is None:
        out = torch.empty((rows, V), dtype=torch.float32, device=hidden.device)
    _check_out(out, torch.float32, (rows, V), hidden.device, "out")
    _check(W.device == hidden.device, "hidden and W must be on one device")
    st = lmhead_logits_bf16_f32(hidden.data_ptr(), rows, H, W.data_ptr(), V, float(alpha),
                                out.data_ptr(), _stream_handle(stream))
    _finish(st, "lmhead_logits_bf16_f32", check, stream)
    return out


def logits_f32(hidden, W, alpha: float = 1.0, bias=None, out=None, stream=None,
               check: bool = False):
    """fp32 logits[rows, V] = alpha * (hidden @ W^T + bias) for bf16 or fp16 CUDA tensors hidden
    [rows, H], W [V, H] and optional bias [V], all of one dtype. Runs asynchronously on
    ``stream`` (default: torch's current stream)."""
    import torch
    dt = {torch.bfloat16: DTYPE_BF16, torch.float16: DTYPE_F16}.get(hidden.dtype)
    _check(dt is not None and W.dtype == hidden.dtype, "bf16 or fp16 operands of one dtype required")
    _check(hidden.dim() == 2 and W.dim() == 2 and hidden.shape[1] == W.shape[1], "shape mismatch")
    _check(hidden.is_cuda and W.is_cuda, "CUDA tensors required")
    _check(hidden.is_contiguous() and W.is_contiguous(), "contiguous tensors required")
    rows, H = hidden.shape
    V = W.shape[0]
    _check(W.device == hidden.device, "hidden and W must be on one device")
    if bias is not None:
        _check(bias.dtype == hidden.dtype and bias.is_cuda and bias.is_contiguous()
               and tuple(bias.shape) == (V,), "bias must be a contiguous [V] tensor of the dtype")
        _check(bias.device == hidden.device, "bias must be on the inputs' device")
    if out is None:
        out = torch.empty((rows, V), dtype=torch.float32, device=hidden.device)
    _check_out(out, torch.float32, (rows, V), hidden.device, "out")
    st = lmhead_logits_f32(hidden.data_ptr(), dt, rows, H, W.data_ptr(), V, float(alpha),
                           0 if bias is None else bias.data_ptr(), out.data_ptr(),
                           _stream_handle(stream))
    _finish(st, "lmhead_logits_f32", check, stream)
    return out


def logprobs_f32(hidden, W, targets, alpha: float = 1.0, bias=None, workspace=None, out=None,
                 stream=None, check: bool = False):
    """(logprobs [rows], lse [rows]) fp32: the log-softmax of the fp32 logits alpha * (hidden @
    W^T + bias) at each row's target token (int32 CUDA tensor [rows]), without writing logits.
    The workspace (logprobs_workspace_bytes(rows, V) bytes) and outputs are allocated here unless
    given (``out`` = (logprobs, lse))."""
    import torch
    dt = {torch.bfloat16: DTYPE_BF16, torch.float16: DTYPE_F16}.get(hidden.dtype)
    _check(dt is not None and W.dtype == hidden.dtype, "bf16 or fp16 operands of one dtype required")
    _check(hidden.dim() == 2 and W.dim() == 2 and hidden.shape[1] == W.shape[1], "shape mismatch")
    _check(hidden.is_cuda and W.is_cuda and hidden.is_contiguous() and W.is_contiguous(),
           "contiguous CUDA tensors required")
    rows, H = hidden.shape
    V = W.shape[0]
    _check(W.device == hidden.device, "hidden and W must be on one device")
    _check(targets.dtype == torch.int32 and targets.is_cuda and targets.is_contiguous()
           and tuple(targets.shape) == (rows,), "targets must be a contiguous int32 [rows] tensor")
    _check(targets.device == hidden.device, "targets must be on the inputs' device")
    if bias is not None:
        _check(bias.dtype == hidden.dtype and bias.is_cuda and bias.is_contiguous()
               and tuple(bias.shape) == (V,), "bias must be a contiguous [V] tensor of the dtype")
        _check(bias.device == hidden.device, "bias must be on the inputs' device")
    if out is None:
        lp = torch.empty((rows,), dtype=torch.float32, device=hidden.device)
        lse = torch.empty((rows,), dtype=torch.float32, device=hidden.device)
    else:
        lp, lse = out
        _check_out(lp, torch.float32, (rows,), hidden.device, "out[0] (logprobs)")
        if lse is not None:
            _check_out(lse, torch.float32, (rows,), hidden.device, "out[1] (lse)")
    need = logprobs_workspace_bytes(rows, V)
    if workspace is None:
        workspace = torch.empty((max(need, 8),), dtype=torch.uint8, device=hidden.device)
    _check(workspace.is_cuda and workspace.is_contiguous() and workspace.device == hidden.device,
           "workspace must be a contiguous CUDA tensor on the inputs' device")
    st = lmhead_logprobs_f32(hidden.data_ptr(), dt, rows, H, W.data_ptr(), V, float(alpha),
                             0 if bias is None else bias.data_ptr(), targets.data_ptr(),
                             lp.data_ptr(), 0 if lse is None else lse.data_ptr(),
                             workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                             _stream_handle(stream))
    _finish(st, "lmhead_logprobs_f32", check, stream)
    return lp, lse


def vocab_shard(V: int, world: int, rank: int):
    """(v_begin, V_shard): the contiguous slice of W's V rows that GPU ``rank`` of ``world`` holds
    for the vocab-parallel head. The first V % world ranks hold one row more; V >= world."""
    _check(world >= 1 and 0 <= rank < world and V >= world, "need V >= world > rank >= 0")
    base, extra = divmod(V, world)
    return rank * base + min(rank, extra), base + (1 if rank < extra else 0)


def logprobs_shard_stats_f32(hidden, W_shard, v_begin: int, targets, alpha: float = 1.0,
                             bias_shard=None, workspace=None, out=None, stream=None,
                             check: bool = False):
    """fp32 [rows, 3] per-row (max, sum of exp(z - max), target logit or NaN) over the logits of
    this GPU's vocab slice W_shard = W[v_begin : v_begin + V_shard] (targets are global ids)."""
    import torch
    dt = {torch.bfloat16: DTYPE_BF16, torch.float16: DTYPE_F16}.get(hidden.dtype)
    _check(dt is not None and W_shard.dtype == hidden.dtype,
           "bf16 or fp16 operands of one dtype required")
    _check(hidden.dim() == 2 and W_shard.dim() == 2 and hidden.shape[1] == W_shard.shape[1],
           "shape mismatch")
    _check(hidden.is_cuda and W_shard.is_cuda and hidden.is_contiguous()
           and W_shard.is_contiguous(), "contiguous CUDA tensors required")
    rows, H = hidden.shape
    V_shard = W_shard.shape[0]
    _check(W_shard.device == hidden.device, "hidden and W_shard must be on one device")
    _check(targets.dtype == torch.int32 and targets.is_cuda and targets.is_contiguous()
           and tuple(targets.shape) == (rows,), "targets must be a contiguous int32 [rows] tensor")
    _check(targets.device == hidden.device, "targets must be on the inputs' device")
    if bias_shard is not None:
        _check(bias_shard.dtype == hidden.dtype and bias_shard.is_cuda
               and bias_shard.is_contiguous() and tuple(bias_shard.shape) == (V_shard,),
               "bias_shard must be a contiguous [V_shard] tensor of the dtype")
        _check(bias_shard.device == hidden.device, "bias_shard must be on the inputs' device")
    if out is None:
        out = torch.empty((rows, 3), dtype=torch.float32, device=hidden.device)
    _check_out(out, torch.float32, (rows, 3), hidden.device, "out (stats)")
    need = logprobs_workspace_bytes(rows, V_shard)
    if workspace is None:
        workspace = torch.empty((max(need, 8),), dtype=torch.uint8, device=hidden.device)
    _check(workspace.is_cuda and workspace.is_contiguous() and workspace.device == hidden.device,
           "workspace must be a contiguous CUDA tensor on the inputs' device")
    st = lmhead_logprobs_shard_stats_f32(
        hidden.data_ptr(), dt, rows, H, W_shard.data_ptr(), V_shard, int(v_begin), float(alpha),
        0 if bias_shard is None else bias_shard.data_ptr(), targets.data_ptr(), out.data_ptr(),
        workspace.data_ptr(), workspace.numel() * workspace.element_size(),
        _stream_handle(stream))
    _finish(st, "lmhead_logprobs_shard_stats_f32", check, stream)
    return out


def logprobs_merge_shards(stats, out=None, stream=None, check: bool = False):
    """(logprobs [rows], lse [rows]) fp32 from the gathered shard stats, fp32 [g, rows, 3] in
    shard order."""
    import torch
    _check(stats.dtype == torch.float32 and stats.is_cuda and stats.is_contiguous()
           and stats.dim() == 3 and stats.shape[2] == 3, "stats must be a contiguous fp32 "
           "[g, rows, 3] CUDA tensor")
    g, rows = stats.shape[0], stats.shape[1]
    if out is None:
        lp = torch.empty((rows,), dtype=torch.float32, device=stats.device)
        lse = torch.empty((rows,), dtype=torch.float32, device=stats.device)
    else:
        lp, lse = out
        _check_out(lp, torch.float32, (rows,), stats.device, "out[0] (logprobs)")
        if lse is not None:
            _check_out(lse, torch.float32, (rows,), stats.device, "out[1] (lse)")
    st = lmhead_logprobs_merge_shards(stats.data_ptr(), g, rows, lp.data_ptr(),
                                      0 if lse is None else lse.data_ptr(),
                                      _stream_handle(stream))
    _finish(st, "lmhead_logprobs_merge_shards", check, stream)
    return lp, lse


def gather_shard_stats(stats, group=None):
    """The exchange of the vocab-parallel log-probs: every rank's [rows, 3] stats gathered into
    [world, rows, 3] in rank order (one all-gather of rows * 12 bytes per rank; NCCL for CUDA
    tensors). Rank r must hold the r-th vocab slice."""
    import torch
    import torch.distributed as dist
    if not dist.is_initialized() or dist.get_world_size(group) == 1:
        return stats.view(1, *stats.shape)   # a single process holds the whole vocabulary
    world = dist.get_world_size(group)
    flat = stats.reshape(-1)
    out = torch.empty((world * flat.numel(),), dtype=stats.dtype, device=stats.device)
    dist.all_gather_into_tensor(out, flat, group=group)
    return out.view(world, *stats.shape)


def logprobs_vocab_parallel(hidden, W_shard, v_begin: int, targets, alpha: float = 1.0,
                            bias_shard=None, group=None, workspace=None, stats=None, out=None,
                            stream=None, check: bool = False):
    """(logprobs [rows], lse [rows]) of the whole vocabulary on every rank of ``group``, each
    rank holding its slice W_shard = W[v_begin : v_begin + V_shard] (vocab_shard gives the
    split) and the same hidden rows and targets: shard stats, one all-gather, merge. Without a
    process group the caller is the only rank. ``workspace``, ``stats`` ([rows, 3]) and ``out``
    are allocated here unless given."""
    import torch
    _check(stream is None or isinstance(stream, torch.cuda.Stream),
           "stream must be a torch.cuda.Stream (the all-gather is ordered on it)")
    stats = logprobs_shard_stats_f32(hidden, W_shard, v_begin, targets, alpha, bias_shard,
                                     workspace=workspace, out=stats, stream=stream)
    with torch.cuda.stream(stream if stream is not None else torch.cuda.current_stream()):
        gathered = gather_shard_stats(stats, group)
    return logprobs_merge_shards(gathered, out=out, stream=stream, check=check)


def logits_vocab_slice_f32(hidden, W_slice, v_begin: int, outs, alpha: float = 1.0,
                           bias_slice=None, stream=None, check: bool = False):
    """Write this GPU's slice of the fp32 logits, alpha * (hidden @ W_slice^T + bias_slice), into
    columns [v_begin, v_begin + V_slice) of every fp32 [>= rows, ld] tensor in ``outs`` (at most
    8; this GPU's own buffer and peers' buffers mapped for peer access alike). Nothing else of
    them is written. Returns ``outs``."""
    import torch
    dt = {torch.bfloat16: DTYPE_BF16, torch.float16: DTYPE_F16}.get(hidden.dtype)
    _check(dt is not None and W_slice.dtype == hidden.dtype,
           "bf16 or fp16 operands of one dtype required")
    _check(hidden.dim() == 2 and W_slice.dim() == 2 and hidden.shape[1] == W_slice.shape[1],
           "shape mismatch")
    _check(hidden.is_cuda and W_slice.is_cuda and hidden.is_contiguous()
           and W_slice.is_contiguous(), "contiguous CUDA tensors required")
    rows, H = hidden.shape
    V_slice = W_slice.shape[0]
    _check(W_slice.device == hidden.device, "hidden and W_slice must be on one device")
    if bias_slice is not None:
        _check(bias_slice.dtype == hidden.dtype and bias_slice.is_cuda
               and bias_slice.is_contiguous() and tuple(bias_slice.shape) == (V_slice,),
               "bias_slice must be a contiguous [V_slice] tensor of the dtype")
        _check(bias_slice.device == hidden.device, "bias_slice must be on the inputs' device")
    outs = list(outs)
    _check(1 <= len(outs) <= 8, "between 1 and 8 output buffers")
    ld = outs[0].shape[1] if outs[0].dim() == 2 else -1
    for o in outs:
        _check(o.dtype == torch.float32 and o.is_cuda and o.is_contiguous() and o.dim() == 2
               and o.shape[1] == ld and o.shape[0] >= rows,
               "outs must be contiguous fp32 CUDA tensors [>= rows, ld] of one width")
    _check(v_begin >= 0 and v_begin + V_slice <= ld, "the slice's columns must fit the buffers")
    st = lmhead_logits_vocab_slice_f32(
        hidden.data_ptr(), dt, rows, H, W_slice.data_ptr(), V_slice, int(v_begin), float(alpha),
        0 if bias_slice is None else bias_slice.data_ptr(), [o.data_ptr() for o in outs], ld,
        _stream_handle(stream))
    _finish(st, "lmhead_logits_vocab_slice_f32", check, stream)
    return outs


class VocabParallelLogits:
    """fp32 logits [rows, V] of a vocab-parallel head on every rank of ``group``: rank r holds
    W[v_begin, v_begin + V_shard) with (v_begin, V_shard) = vocab_shard(V, world, r), and the
    same hidden rows. Each rank's head kernel stores its slice into every rank's logits buffer
    (symmetric memory, peer stores over NVLink), between two barriers across the ranks; there is
    no separate gather pass. The buffers hold ``max_rows`` rows; a call returns a view of this
    rank's buffer, valid until the next call. Without a process group (or with one rank) the
    call is lmhead_logits_f32 into a local buffer, unless ``symmetric=True`` asks for the
    symmetric-memory buffer and barriers anyway (a process group is needed then)."""

    def __init__(self, max_rows: int, V: int, group=None, device=None, symmetric=None):
        import torch
        import torch.distributed as dist
        grouped = dist.is_initialized()
        multi = grouped and dist.get_world_size(group) > 1
        self.world = dist.get_world_size(group) if grouped else 1
        self.rank = dist.get_rank(group) if grouped else 0
        self.V, self.max_rows = int(V), int(max_rows)
        self.v_begin, self.V_shard = vocab_shard(self.V, self.world, self.rank)
        device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
        self._handle = None
        use_symm = multi if symmetric is None else bool(symmetric)
        _check(not use_symm or grouped, "symmetric memory needs an initialised process group")
        if use_symm:
            import torch.distributed._symmetric_memory as symm_mem
            self.buffer = symm_mem.empty((self.max_rows, self.V), dtype=torch.float32,
                                         device=device)
            self._handle = symm_mem.rendezvous(self.buffer, group or dist.group.WORLD)
            self._peers = [self._handle.get_buffer(r, (self.max_rows, self.V), torch.float32)
                           for r in range(self.world)]
        else:
            self.buffer = torch.empty((self.max_rows, self.V), dtype=torch.float32,
                                      device=device)
            self._peers = [self.buffer]

    def __call__(self, hidden, W_shard, alpha: float = 1.0, bias_shard=None, stream=None,
                 check: bool = False):
        import torch
        rows = hidden.shape[0]
        _check(rows <= self.max_rows, f"at most {self.max_rows} rows")
        _check(W_shard.dim() == 2 and W_shard.shape[0] == self.V_shard,
               f"rank {self.rank} holds {self.V_shard} vocab rows")
        s = stream if stream is not None else torch.cuda.current_stream()
        with torch.cuda.stream(s):
            if self._handle is not None:
                self._handle.barrier(channel=0)   # every rank is done reading the last logits
            logits_vocab_slice_f32(hidden, W_shard, self.v_begin, self._peers, alpha,
                                   bias_slice=bias_shard, stream=s, check=check)
            if self._handle is not None:
                self._handle.barrier(channel=0)   # every slice has landed in every buffer
        return self.buffer[:rows]


def logits_w4a16_nvfp4(hidden, w_packed, w_scales, w_global_scale: float, alpha: float = 1.0,
                       out=None, stream=None, check: bool = False):
    """bf16 logits[rows, V] for the NVFP4 head: w_packed uint8 [V, H/2], w_scales uint8
    (E4M3) [V, H/16], bf16 hidden [rows, H]."""
    import torch
    _check(hidden.dtype == torch.bfloat16, "bf16 hidden required")
    _check(w_packed.dtype == torch.uint8 and w_scales.dtype == torch.uint8, "uint8 codes/scales")
    rows, H = hidden.shape
    V = w_packed.shape[0]
    _check(tuple(w_packed.shape) == (V, H // 2) and tuple(w_scales.shape) == (V, H // 16),
           "w_packed must be [V, H/2] and w_scales [V, H/16]")
    _check(all(t.is_cuda and t.is_contiguous() for t in (hidden, w_packed, w_scales)),
           "contiguous CUDA tensors required")
    if out is None:
        out = torch.empty((rows, V), dtype=torch.bfloat16, device=hidden.device)
    _check_out(out, torch.bfloat16, (rows, V), hidden.device, "out")
    _check(w_packed.device == hidden.device and w_scales.device == hidden.device,
           "hidden, codes and scales must be on one device")
    st = lmhead_logits_w4a16_nvfp4(hidden.data_ptr(), rows, H, w_packed.data_ptr(),
                                   w_scales.data_ptr(), float(w_global_scale), V, float(alpha),
                                   out.data_ptr(), _stream_handle(stream))
    _finish(st, "lmhead_logits_w4a16_nvfp4", check, stream)
    return out
