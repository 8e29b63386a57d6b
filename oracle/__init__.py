"""CPU oracle for the LM-head logits projection -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this package. The CUDA library never imports, links or calls it, and shares no code with it.

The arithmetic lives in ``lmhead_oracle.c`` (plain C, double precision, one rounding at the end);
this module only compiles it with gcc and marshals numpy arrays through ctypes. It computes

    fp32 head:  logits[r, v] = RN_fp32(alpha * (sum_k hidden[r, k] * W[v, k] + bias[v]))
                (bf16 or fp16 inputs; bias optional)
    NVFP4 head: logits[r, v] = RN_bf16(alpha * sum_k hidden[r, k] * e2m1(q[v, k]) * e4m3(s[v, k/16]) * g)
    log-probs:  logprob[r] = z[r, t_r] - log sum_v exp z[r, v] over the fp32 logits z, whole or
                from per-slice (max, sum, target logit) stats merged in double
    quantiser:  the NVFP4 codes, block scales and global scale of a bf16 W

following "[Model] Honor fp32 head_dtype in Inkling muP logits (target + MTP draft)" ("Purpose";
"muP is folded into the fp32 GEMM"), "FP32 LM head skip FP32 cast" (implementation breakdown) and
lm_head_nvfp4_rows.rs (module doc; lm_head_nvfp4_rows_run).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lmhead_oracle.c")
_HDR = os.path.join(_HERE, "lmhead_oracle.h")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile lmhead_oracle.c into oracle/liboracle.so (gcc, OpenMP, no fast-math, no FMA)."""
    newest_src = max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= newest_src:
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           "-fno-fast-math", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True, cwd=_HERE)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        u16p = ctypes.POINTER(ctypes.c_uint16)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        f32p = ctypes.POINTER(ctypes.c_float)
        f64p = ctypes.POINTER(ctypes.c_double)
        i64 = ctypes.c_int64
        lib.oracle_bf16_value.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_value.restype = ctypes.c_double
        lib.oracle_f16_value.argtypes = [ctypes.c_uint16]
        lib.oracle_f16_value.restype = ctypes.c_double
        lib.oracle_e2m1_value.argtypes = [ctypes.c_uint8]
        lib.oracle_e2m1_value.restype = ctypes.c_double
        lib.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_value.restype = ctypes.c_double
        lib.oracle_round_f32.argtypes = [ctypes.c_double]
        lib.oracle_round_f32.restype = ctypes.c_float
        lib.oracle_round_bf16.argtypes = [ctypes.c_double]
        lib.oracle_round_bf16.restype = ctypes.c_uint16
        lib.oracle_nvfp4_weight.argtypes = [u8p, u8p, ctypes.c_float, i64, i64, i64]
        lib.oracle_nvfp4_weight.restype = ctypes.c_double
        lib.oracle_logits_bf16_f32.argtypes = [u16p, i64, i64, u16p, i64, ctypes.c_float, f32p,
                                               f64p, ctypes.c_int]
        lib.oracle_logits_bf16_f32.restype = ctypes.c_int
        lib.oracle_logits_f32.argtypes = [u16p, ctypes.c_int, i64, i64, u16p, i64, ctypes.c_float,
                                          ctypes.c_void_p, f32p, f64p, ctypes.c_int]
        lib.oracle_logits_f32.restype = ctypes.c_int
        lib.oracle_logits_w4a16_nvfp4.argtypes = [u16p, i64, i64, u8p, u8p, ctypes.c_float, i64,
                                                  ctypes.c_float, u16p, f64p, ctypes.c_int]
        lib.oracle_logits_w4a16_nvfp4.restype = ctypes.c_int
        lib.oracle_logprobs_f32.argtypes = [u16p, ctypes.c_int, i64, i64, u16p, i64,
                                            ctypes.c_float, ctypes.c_void_p,
                                            ctypes.POINTER(ctypes.c_int32), f32p, f32p,
                                            ctypes.c_int]
        lib.oracle_logprobs_f32.restype = ctypes.c_int
        lib.oracle_logprob_shard_stats.argtypes = [u16p, ctypes.c_int, i64, i64, u16p, i64, i64,
                                                   ctypes.c_float, ctypes.c_void_p,
                                                   ctypes.POINTER(ctypes.c_int32), f64p,
                                                   ctypes.c_int]
        lib.oracle_logprob_shard_stats.restype = ctypes.c_int
        lib.oracle_logprob_merge_shards.argtypes = [f64p, i64, i64, f32p, f32p]
        lib.oracle_logprob_merge_shards.restype = ctypes.c_int
        lib.oracle_nvfp4_quantize.argtypes = [u16p, i64, i64, u8p, u8p, f32p]
        lib.oracle_nvfp4_quantize.restype = ctypes.c_int
        lib.oracle_rn_e4m3.argtypes = [ctypes.c_float]
        lib.oracle_rn_e4m3.restype = ctypes.c_uint8
        lib.oracle_rn_e2m1.argtypes = [ctypes.c_float]
        lib.oracle_rn_e2m1.restype = ctypes.c_uint8
        _lib = lib
        return lib


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


# ---------------------------------------------------------------- scalar decoders / rounding

def bf16_value(bits: int) -> float:
    return _load().oracle_bf16_value(int(bits) & 0xFFFF)


def f16_value(bits: int) -> float:
    return _load().oracle_f16_value(int(bits) & 0xFFFF)


def e2m1_value(code: int) -> float:
    return _load().oracle_e2m1_value(int(code) & 0x0F)


def e4m3_value(code: int) -> float:
    return _load().oracle_e4m3_value(int(code) & 0xFF)


def round_f32(x: float) -> float:
    return _load().oracle_round_f32(float(x))


def round_bf16(x: float) -> int:
    return int(_load().oracle_round_bf16(float(x)))


def nvfp4_weight(packed: np.ndarray, scales: np.ndarray, g: float, v: int, k: int) -> float:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    H = packed.shape[1] * 2
    return _load().oracle_nvfp4_weight(_ptr(packed, ctypes.c_uint8), _ptr(scales, ctypes.c_uint8),
                                       float(g), H, int(v), int(k))


# ---------------------------------------------------------------- the two heads

def logits_bf16_f32(hidden_bits: np.ndarray, w_bits: np.ndarray, alpha: float,
                    threads: int | None = None):
    """fp32 logits and |alpha|*sum|h*w| for bf16 hidden [rows, H] and W [V, H] (uint16 bits)."""
    h = np.ascontiguousarray(hidden_bits, dtype=np.uint16)
    w = np.ascontiguousarray(w_bits, dtype=np.uint16)
    if h.ndim != 2 or w.ndim != 2 or h.shape[1] != w.shape[1]:
        raise ValueError(f"shape mismatch: hidden {h.shape}, W {w.shape}")
    rows, H = h.shape
    V = w.shape[0]
    out = np.zeros((rows, V), dtype=np.float32)
    absum = np.zeros((rows, V), dtype=np.float64)
    if rows == 0:
        return out, absum
    rc = _load().oracle_logits_bf16_f32(_ptr(h, ctypes.c_uint16), rows, H,
                                        _ptr(w, ctypes.c_uint16), V, ctypes.c_float(alpha),
                                        _ptr(out, ctypes.c_float), _ptr(absum, ctypes.c_double),
                                        threads or default_threads())
    if rc != 0:
        raise RuntimeError(f"oracle_logits_bf16_f32 failed with {rc}")
    return out, absum


def logits_w4a16_nvfp4(hidden_bits: np.ndarray, packed: np.ndarray, scales: np.ndarray,
                       g: float, alpha: float, threads: int | None = None):
    """bf16 logits (uint16 bits) and |alpha|*sum|h*w| for the NVFP4 head."""
    h = np.ascontiguousarray(hidden_bits, dtype=np.uint16)
    p = np.ascontiguousarray(packed, dtype=np.uint8)
    s = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, H = h.shape
    V = p.shape[0]
    if p.shape != (V, H // 2) or s.shape != (V, H // 16) or H % 16:
        raise ValueError(f"shape mismatch: hidden {h.shape}, packed {p.shape}, scales {s.shape}")
    out = np.zeros((rows, V), dtype=np.uint16)
    absum = np.zeros((rows, V), dtype=np.float64)
    if rows == 0:
        return out, absum
    rc = _load().oracle_logits_w4a16_nvfp4(_ptr(h, ctypes.c_uint16), rows, H,
                                           _ptr(p, ctypes.c_uint8), _ptr(s, ctypes.c_uint8),
                                           ctypes.c_float(g), V, ctypes.c_float(alpha),
                                           _ptr(out, ctypes.c_uint16),
                                           _ptr(absum, ctypes.c_double),
                                           threads or default_threads())
    if rc != 0:
        raise RuntimeError(f"oracle_logits_w4a16_nvfp4 failed with {rc}")
    return out, absum


def logits_f32(hidden_bits: np.ndarray, w_bits: np.ndarray, alpha: float, bias_bits=None,
               dtype: str = "bf16", threads: int | None = None):
    """fp32 logits and the error-bound scale for bf16 or fp16 ("f16") hidden [rows, H], W [V, H]
    and optional bias [V], all given as uint16 bit patterns."""
    if dtype not in ("bf16", "f16"):
        raise ValueError(f"dtype {dtype!r}")
    h = np.ascontiguousarray(hidden_bits, dtype=np.uint16)
    w = np.ascontiguousarray(w_bits, dtype=np.uint16)
    if h.ndim != 2 or w.ndim != 2 or h.shape[1] != w.shape[1]:
        raise ValueError(f"shape mismatch: hidden {h.shape}, W {w.shape}")
    rows, H = h.shape
    V = w.shape[0]
    b = None
    if bias_bits is not None:
        b = np.ascontiguousarray(bias_bits, dtype=np.uint16)
        if b.shape != (V,):
            raise ValueError(f"bias shape {b.shape}, expected ({V},)")
    out = np.zeros((rows, V), dtype=np.float32)
    absum = np.zeros((rows, V), dtype=np.float64)
    if rows == 0:
        return out, absum
    rc = _load().oracle_logits_f32(_ptr(h, ctypes.c_uint16), 1 if dtype == "f16" else 0, rows, H,
                                   _ptr(w, ctypes.c_uint16), V, ctypes.c_float(alpha),
                                   None if b is None else b.ctypes.data,
                                   _ptr(out, ctypes.c_float), _ptr(absum, ctypes.c_double),
                                   threads or default_threads())
    if rc != 0:
        raise RuntimeError(f"oracle_logits_f32 failed with {rc}")
    return out, absum


# ---------------------------------------------------------------- the NVFP4 quantiser

def rn_e4m3(t: float) -> int:
    return int(_load().oracle_rn_e4m3(ctypes.c_float(t)))


def rn_e2m1(x: float) -> int:
    return int(_load().oracle_rn_e2m1(ctypes.c_float(x)))


def nvfp4_quantize(w_bits: np.ndarray):
    """(packed [V, H/2] u8, scales [V, H/16] u8, g float32) for bf16 W [V, H] given as uint16 bits
    (H % 16 == 0), by the binary32 reading in lmhead_oracle.c."""
    w = np.ascontiguousarray(w_bits, dtype=np.uint16)
    V, H = w.shape
    packed = np.zeros((V, H // 2), dtype=np.uint8)
    scales = np.zeros((V, H // 16), dtype=np.uint8)
    g = np.zeros(1, dtype=np.float32)
    rc = _load().oracle_nvfp4_quantize(_ptr(w, ctypes.c_uint16), V, H, _ptr(packed, ctypes.c_uint8),
                                       _ptr(scales, ctypes.c_uint8), _ptr(g, ctypes.c_float))
    if rc != 0:
        raise RuntimeError(f"oracle_nvfp4_quantize failed with {rc}")
    return packed, scales, np.float32(g[0])


# ---------------------------------------------------------------- log-probabilities

def logprobs_f32(hidden_bits: np.ndarray, w_bits: np.ndarray, alpha: float, targets: np.ndarray,
                 bias_bits=None, dtype: str = "bf16", threads: int | None = None):
    """(logprobs [rows], lse [rows]) as float32: the log-softmax of the fp32 logits of
    logits_f32 at each row's target token (NaN for a target outside [0, V))."""
    h = np.ascontiguousarray(hidden_bits, dtype=np.uint16)
    w = np.ascontiguousarray(w_bits, dtype=np.uint16)
    t = np.ascontiguousarray(targets, dtype=np.int32)
    rows, H = h.shape
    V = w.shape[0]
    if w.shape[1] != H or t.shape != (rows,):
        raise ValueError("shape mismatch")
    b = None if bias_bits is None else np.ascontiguousarray(bias_bits, dtype=np.uint16)
    lp = np.zeros(rows, dtype=np.float32)
    lse = np.zeros(rows, dtype=np.float32)
    if rows == 0:
        return lp, lse
    rc = _load().oracle_logprobs_f32(_ptr(h, ctypes.c_uint16), 1 if dtype == "f16" else 0, rows, H,
                                     _ptr(w, ctypes.c_uint16), V, ctypes.c_float(alpha),
                                     None if b is None else b.ctypes.data,
                                     _ptr(t, ctypes.c_int32), _ptr(lp, ctypes.c_float),
                                     _ptr(lse, ctypes.c_float), threads or default_threads())
    if rc != 0:
        raise RuntimeError(f"oracle_logprobs_f32 failed with {rc}")
    return lp, lse


def logprob_shard_stats(hidden_bits: np.ndarray, w_shard_bits: np.ndarray, v_begin: int,
                        alpha: float, targets: np.ndarray, bias_bits=None, dtype: str = "bf16",
                        threads: int | None = None) -> np.ndarray:
    """float64 [rows, 3]: (max, sum of exp(z - max), target logit or NaN) over the fp32 logits of
    the vocab slice W[v_begin : v_begin + V_shard] (targets are global ids)."""
    h = np.ascontiguousarray(hidden_bits, dtype=np.uint16)
    w = np.ascontiguousarray(w_shard_bits, dtype=np.uint16)
    t = np.ascontiguousarray(targets, dtype=np.int32)
    rows, H = h.shape
    if w.shape[1] != H or t.shape != (rows,):
        raise ValueError("shape mismatch")
    b = None if bias_bits is None else np.ascontiguousarray(bias_bits, dtype=np.uint16)
    stats = np.zeros((rows, 3), dtype=np.float64)
    if rows == 0:
        return stats
    rc = _load().oracle_logprob_shard_stats(
        _ptr(h, ctypes.c_uint16), 1 if dtype == "f16" else 0, rows, H, _ptr(w, ctypes.c_uint16),
        w.shape[0], int(v_begin), ctypes.c_float(alpha), None if b is None else b.ctypes.data,
        _ptr(t, ctypes.c_int32), _ptr(stats, ctypes.c_double), threads or default_threads())
    if rc != 0:
        raise RuntimeError(f"oracle_logprob_shard_stats failed with {rc}")
    return stats


def logprob_merge_shards(stats: np.ndarray):
    """(logprobs [rows], lse [rows]) float32 from float64 shard stats [shards, rows, 3]."""
    st = np.ascontiguousarray(stats, dtype=np.float64)
    if st.ndim != 3 or st.shape[2] != 3:
        raise ValueError(f"stats shape {st.shape}")
    rows = st.shape[1]
    lp = np.zeros(rows, dtype=np.float32)
    lse = np.zeros(rows, dtype=np.float32)
    if rows == 0:
        return lp, lse
    rc = _load().oracle_logprob_merge_shards(_ptr(st, ctypes.c_double), st.shape[0], rows,
                                             _ptr(lp, ctypes.c_float), _ptr(lse, ctypes.c_float))
    if rc != 0:
        raise RuntimeError(f"oracle_logprob_merge_shards failed with {rc}")
    return lp, lse
