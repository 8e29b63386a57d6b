"""Host-side checks of the C ABI (no GPU needed): the library builds and loads, exports every
function include/lmhead.h declares, and rejects bad arguments synchronously -- launching
nothing, as lm_head_nvfp4_rows.rs's lm_head_nvfp4_rows_run does when its head cannot run."""
import ctypes
import os
import re
import subprocess

import pytest

import fp32_accumulate_lm_b200 as lm
from fp32_accumulate_lm_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lmhead.h")


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return lm.load_library()


def _functions(text: str):
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lmhead_[a-z0-9_]+)\s*\(", text)))


def _test_block(text: str) -> str:
    m = re.search(r"#if defined\(LMHEAD_TEST_HOOKS\) && LMHEAD_TEST_HOOKS(.*?)#endif", text, re.S)
    return m.group(1) if m else ""


def declared_functions():
    """Functions of the release library: everything outside the test-build block."""
    text = open(HEADER).read()
    test_only = set(_functions(_test_block(text)))
    return [f for f in _functions(text) if f not in test_only]


def hook_functions():
    return _functions(_test_block(open(HEADER).read()))


def exported(path: str):
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True,
                         check=True).stdout
    return {line.split()[-1] for line in out.splitlines() if line.strip()}


def test_header_declares_the_two_entry_points():
    names = declared_functions()
    assert "lmhead_logits_bf16_f32" in names and "lmhead_logits_w4a16_nvfp4" in names


def test_library_exports_every_declared_symbol(lib):
    syms = exported(lm.library_path())
    for name in declared_functions():
        assert name in syms, name
        assert getattr(lib, name) is not None
    # nothing from the statically linked CUDA runtime leaks out
    assert not any(s.startswith("cuda") for s in syms)


def test_test_knobs_exist_only_in_the_test_build(lib):
    """The fault-injection and conversion knobs are declared for LMHEAD_TEST_HOOKS builds only:
    the release library does not export them, the test build exports them and everything else."""
    knobs = hook_functions()
    assert set(knobs) == {"lmhead_debug_set_fault_injection", "lmhead_debug_set_nvfp4_conversion",
                          "lmhead_debug_set_cta_pairs", "lmhead_debug_set_dynamic_tiles"}
    release, test = exported(lm.library_path()), exported(_build.TEST_LIB)
    assert not set(knobs) & release
    assert set(knobs) | set(declared_functions()) <= test
    assert not any(s.startswith("cuda") for s in test)
    with pytest.raises(RuntimeError):
        lm.set_fault_injection(True, 1)       # outside test_hooks(): refused, nothing changes
    with lm.test_hooks() as tlib:
        assert tlib is lm.load_test_library()
        lm.set_nvfp4_conversion(0)           # reachable inside


def test_header_compiles_as_c():
    src = f'#include "{HEADER}"\nint main(void) {{ return lmhead_version() < 0; }}\n'
    for defs in ([], ["-DLMHEAD_TEST_HOOKS=1"]):
        res = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-fsyntax-only", *defs,
                              "-x", "c", "-"], input=src, capture_output=True, text=True)
        assert res.returncode == 0, res.stderr


def test_status_strings_and_version(lib):
    for code in range(8):
        assert lm.status_string(code) and lm.status_string(code) != "unknown status"
    assert lm.status_string(99) == "unknown status"
    assert lm.version() >= 100


# Pointer values below are never dereferenced: every case fails validation first.
A16 = 0x10000  # 16-byte aligned fake device addresses
B16 = 0x20000000
C16 = 0x40000000


@pytest.mark.parametrize("rows,H,V,want", [
    (-1, 64, 128, 2), (4, 0, 128, 2), (4, 64, 0, 2), (4, -8, 128, 2),
    (4, 60, 128, 3),            # H % 8 != 0: 16-byte row pitch impossible
    (2 ** 31, 64, 128, 2),      # beyond the int32 tile coordinates
])
def test_bf16_shape_errors(lib, rows, H, V, want):
    assert lm.lmhead_logits_bf16_f32(A16, rows, H, B16, V, 1.0, C16, 0) == want


def test_bf16_null_align_alias(lib):
    assert lm.lmhead_logits_bf16_f32(0, 4, 64, B16, 128, 1.0, C16, 0) == 1
    assert lm.lmhead_logits_bf16_f32(A16, 4, 64, 0, 128, 1.0, C16, 0) == 1
    assert lm.lmhead_logits_bf16_f32(A16, 4, 64, B16, 128, 1.0, 0, 0) == 1
    assert lm.lmhead_logits_bf16_f32(A16 + 8, 4, 64, B16, 128, 1.0, C16, 0) == 3
    assert lm.lmhead_logits_bf16_f32(A16, 4, 64, B16 + 2, 128, 1.0, C16, 0) == 3
    assert lm.lmhead_logits_bf16_f32(A16, 4, 64, B16, 128, 1.0, C16 + 2, 0) == 3
    # logits overlapping W or hidden
    assert lm.lmhead_logits_bf16_f32(A16, 4, 64, B16, 128, 1.0, B16 + 64, 0) == 7
    assert lm.lmhead_logits_bf16_f32(A16, 4, 64, B16, 128, 1.0, A16 - 16, 0) == 7


def test_general_entry_argument_errors(lib):
    """lmhead_logits_f32: operand type, bias alignment and bias/logits overlap are checked on the
    host before anything is launched; without a bias it takes the bf16 entry's checks."""
    f = lm.lmhead_logits_f32
    for dt in (lm.DTYPE_BF16, lm.DTYPE_F16):
        assert f(A16, dt, -1, 64, B16, 128, 1.0, 0, C16, 0) == 2
        assert f(A16, dt, 4, 60, B16, 128, 1.0, 0, C16, 0) == 3
        assert f(0, dt, 4, 64, B16, 128, 1.0, 0, C16, 0) == 1
        assert f(A16, dt, 4, 64, B16, 128, 1.0, 0x7000001, C16, 0) == 3     # odd bias address
        assert f(A16, dt, 4, 64, B16, 128, 1.0, C16 + 64, C16, 0) == 7      # bias inside logits
        assert f(A16, dt, 4, 64, B16, 128, 1.0, 0, B16 + 64, 0) == 7
    for bad in (2, -1, 7):
        assert f(A16, bad, 4, 64, B16, 128, 1.0, 0, C16, 0) == 2
    assert f(0, lm.DTYPE_F16, 0, 64, 0, 128, 1.0, 0, 0, 0) == 0             # rows == 0: no-op


def test_quantiser_argument_errors(lib):
    f = lm.lmhead_nvfp4_quantize
    WS = 0x50000000
    need = lm.nvfp4_quantize_workspace_bytes()
    assert need >= 4 and need % 4 == 0
    assert f(A16, 0, 64, B16, C16, 0x60000000, WS, need, 0) == 2
    assert f(A16, 4, 40, B16, C16, 0x60000000, WS, need, 0) == 3        # H % 16 != 0
    assert f(0, 4, 64, B16, C16, 0x60000000, WS, need, 0) == 1
    assert f(A16, 4, 64, B16, C16, 0x60000000, 0, need, 0) == 1         # no workspace
    assert f(A16 + 8, 4, 64, B16, C16, 0x60000000, WS, need, 0) == 3
    assert f(A16, 4, 64, B16 + 4, C16, 0x60000000, WS, need, 0) == 3    # packed not 8-aligned
    assert f(A16, 4, 64, B16, C16, 0x60000002, WS, need, 0) == 3
    assert f(A16, 4, 64, A16 + 16, C16, 0x60000000, WS, need, 0) == 7   # packed over W
    assert f(A16, 4, 64, B16, C16, B16 + 8, WS, need, 0) == 7           # g inside packed


def test_noalloc_quantiser_checks_everything_before_the_device(lib):
    """lmhead_nvfp4_quantize_noalloc rejects every invalid call before it looks up its scratch
    or touches any device state, so these codes come back the same on a host without a GPU."""
    f = lm.lmhead_nvfp4_quantize_noalloc
    G = 0x60000000
    assert f(A16, 0, 64, B16, C16, G, 0) == 2                  # V = 0
    assert f(A16, 4, 40, B16, C16, G, 0) == 3                  # H % 16 != 0
    assert f(A16, 2 ** 31, 64, B16, C16, G, 0) == 2            # V past int32
    assert f(A16, 4, 2 ** 31 + 16, B16, C16, G, 0) == 2        # H past int32
    assert f(0, 4, 64, B16, C16, G, 0) == 1
    assert f(A16, 4, 64, B16, C16, 0, 0) == 1
    assert f(A16 + 8, 4, 64, B16, C16, G, 0) == 3              # W not 16-byte aligned
    assert f(A16, 4, 64, B16 + 4, C16, G, 0) == 3              # codes not 8-byte aligned
    assert f(A16, 4, 64, B16, C16, G + 2, 0) == 3              # g not 4-byte aligned
    assert f(A16, 4, 64, B16, B16 + 64, G, 0) == 7             # scales over the codes
    assert f(A16, 4, 64, A16 + 128, C16, G, 0) == 7            # codes over W
    assert f(A16, 4, 64, B16, C16, C16 + 8, 0) == 7            # g inside the scales


def test_stream_status_without_a_device(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert lm.lmhead_stream_status(0) == 5                     # the synchronisation fails


def test_logprobs_argument_errors(lib):
    f = lm.lmhead_logprobs_f32
    T, LP, LSE, WS = 0x60000000, 0x61000000, 0x62000000, 0x63000000
    need = lm.logprobs_workspace_bytes(4, 300)
    assert need == 4 * 4 * 3 * 8                       # rows x 4 chunks per 128 vocab x 8 bytes
    assert f(A16, 0, 4, 64, B16, 300, 1.0, 0, T, LP, LSE, WS, need, 0) != 2   # valid shape passes
    assert f(A16, 5, 4, 64, B16, 300, 1.0, 0, T, LP, LSE, WS, need, 0) == 2   # bad dtype
    assert f(A16, 0, 4, 64, B16, 300, 1.0, 0, 0, LP, LSE, WS, need, 0) == 1   # no targets
    assert f(A16, 0, 4, 64, B16, 300, 1.0, 0, T, 0, LSE, WS, need, 0) == 1    # no logprobs
    assert f(A16, 0, 4, 64, B16, 300, 1.0, 0, T, LP, LSE, 0, need, 0) == 1    # no workspace
    assert f(A16, 0, 4, 64, B16, 300, 1.0, 0, T, LP, LSE, WS, need - 8, 0) == 2  # too small
    assert f(A16, 0, 4, 64, B16, 300, 1.0, 0, T + 2, LP, LSE, WS, need, 0) == 3
    assert f(A16, 0, 4, 64, B16, 300, 1.0, 0, T, LP, LSE, WS + 4, need, 0) == 3
    assert f(A16, 0, 4, 64, B16, 300, 1.0, 0, T, LP, LP + 8, WS, need, 0) == 7  # lse over logprobs
    assert f(A16, 0, 4, 64, B16, 300, 1.0, 0, T, B16 + 16, LSE, WS, need, 0) == 7  # over W
    assert f(A16, 0, 0, 64, B16, 300, 1.0, 0, 0, 0, 0, 0, 0, 0) == 0            # rows == 0


def test_rows_zero_launches_nothing(lib):
    # rows == 0 is a no-op even with NULL pointers (no CUDA call is made)
    assert lm.lmhead_logits_bf16_f32(0, 0, 64, 0, 128, 1.0, 0, 0) == 0
    assert lm.lmhead_logits_w4a16_nvfp4(0, 0, 64, 0, 0, 1.0, 128, 1.0, 0, 0) == 0


def test_nvfp4_argument_errors(lib):
    f = lm.lmhead_logits_w4a16_nvfp4
    assert f(A16, 4, 64, B16, C16, 1.0, 128, 1.0, 0x7000000, 0) != 2  # valid shape gets past
    assert f(A16, -1, 64, B16, C16, 1.0, 128, 1.0, 0x7000000, 0) == 2
    assert f(A16, 4, 80, B16, C16, 1.0, 128, 1.0, 0x7000000, 0) == 3   # H % 32 != 0
    assert f(A16, 4, 96, B16, C16, 1.0, 128, 1.0, 0x7000000, 0) not in (1, 2, 3, 7)  # 32 mod 64
    assert f(A16, 4, 64, B16, C16, 1.0, 0, 1.0, 0x7000000, 0) == 2
    assert f(0, 4, 64, B16, C16, 1.0, 128, 1.0, 0x7000000, 0) == 1
    assert f(A16, 4, 64, 0, C16, 1.0, 128, 1.0, 0x7000000, 0) == 1
    assert f(A16, 4, 64, B16, 0, 1.0, 128, 1.0, 0x7000000, 0) == 1
    assert f(A16, 4, 64, B16 + 4, C16, 1.0, 128, 1.0, 0x7000000, 0) == 3
    assert f(A16, 4, 64, B16, C16 + 2, 1.0, 128, 1.0, 0x7000000, 0) == 3
    assert f(A16, 4, 64, B16, C16, 1.0, 128, 1.0, 0x7000001, 0) == 3
    assert f(A16, 4, 64, B16, C16, 1.0, 128, 1.0, B16 + 16, 0) == 7   # logits over the codes
    assert f(A16, 4, 64, B16, C16, 1.0, 128, 1.0, C16, 0) == 7        # logits over the scales


def test_no_cpu_fallback_without_a_device(lib):
    """On a host without a usable GPU a valid call must fail loudly, never compute on the CPU."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    st = lm.lmhead_logits_bf16_f32(A16, 4, 64, B16, 128, 1.0, C16, 0)
    assert st in (4, 5)


def test_torch_wrapper_rejects_wrong_dtypes():
    import torch
    h = torch.zeros(2, 64, dtype=torch.float32)
    w = torch.zeros(8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        lm.logits_bf16_f32(h, w, 1.0)


def test_vocab_shard_argument_errors(lib):
    """lmhead_logprobs_shard_stats_f32 / lmhead_logprobs_merge_shards: the shard must lie inside
    the int32 token-id range, and outputs may not overlap inputs, the workspace or each other."""
    f = lm.lmhead_logprobs_shard_stats_f32
    T, ST, WS = 0x60000000, 0x61000000, 0x63000000
    need = lm.logprobs_workspace_bytes(4, 300)
    args = lambda **kw: dict(dict(h=A16, dt=0, rows=4, H=64, w=B16, V=300, v0=1000, alpha=1.0,
                                  bias=0, t=T, st=ST, ws=WS, nb=need), **kw)
    call = lambda a: f(a["h"], a["dt"], a["rows"], a["H"], a["w"], a["V"], a["v0"], a["alpha"],
                       a["bias"], a["t"], a["st"], a["ws"], a["nb"], 0)
    assert call(args()) not in (1, 2, 3, 7)                  # valid: reaches the device check
    assert call(args(v0=-1)) == 2
    assert call(args(v0=2 ** 31 - 300)) not in (1, 2, 3, 7)  # last id 2^31 - 1: still valid
    assert call(args(v0=2 ** 31 - 299)) == 2                 # one past the int32 ids
    assert call(args(dt=3)) == 2
    assert call(args(t=0)) == 1 and call(args(st=0)) == 1 and call(args(ws=0)) == 1
    assert call(args(nb=need - 8)) == 2
    assert call(args(t=T + 2)) == 3 and call(args(st=ST + 2)) == 3 and call(args(ws=WS + 4)) == 3
    assert call(args(st=B16 + 64)) == 7                      # stats over the weight slice
    assert call(args(st=T)) == 7                             # stats over the targets
    assert call(args(st=WS + 8)) == 7                        # stats inside the workspace
    assert call(args(ws=A16)) == 7                           # workspace over hidden
    assert call(args(rows=0, h=0, w=0, t=0, st=0, ws=0)) == 0
    m = lm.lmhead_logprobs_merge_shards
    LP, LSE = 0x64000000, 0x65000000
    assert m(ST, 0, 4, LP, LSE, 0) == 2                      # no shards
    assert m(ST, 2, -1, LP, LSE, 0) == 2
    assert m(0, 2, 4, LP, LSE, 0) == 1 and m(ST, 2, 4, 0, LSE, 0) == 1
    assert m(ST + 2, 2, 4, LP, LSE, 0) == 3 and m(ST, 2, 4, LP + 1, LSE, 0) == 3
    assert m(ST, 2, 4, ST + 88, LSE, 0) == 7                 # logprobs inside the 96-byte stats
    assert m(ST, 2, 4, LP, LP + 4, 0) == 7                   # lse over logprobs
    assert m(ST, 2, 4, LP, 0, 0) not in (1, 2, 3, 7)         # lse is optional
    assert m(0, 3, 0, 0, 0, 0) == 0                          # rows == 0


def test_vocab_shard_split():
    """vocab_shard: contiguous, disjoint, covering slices whose sizes differ by at most one."""
    for V in (8, 1000, 128256, 151936):
        for world in range(1, 9):
            parts = [lm.vocab_shard(V, world, r) for r in range(world)]
            assert parts[0][0] == 0
            for (b0, n0), (b1, _) in zip(parts, parts[1:]):
                assert b0 + n0 == b1
            assert parts[-1][0] + parts[-1][1] == V
            sizes = [n for _, n in parts]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    with pytest.raises(ValueError):
        lm.vocab_shard(3, 4, 0)
    with pytest.raises(ValueError):
        lm.vocab_shard(100, 2, 2)


def test_vocab_parallel_wrappers_reject_bad_tensors():
    import torch
    h = torch.zeros(2, 64, dtype=torch.bfloat16)
    w = torch.zeros(8, 64, dtype=torch.bfloat16)
    t = torch.zeros(2, dtype=torch.int32)
    with pytest.raises(ValueError):                      # host tensors
        lm.logprobs_shard_stats_f32(h, w, 0, t)
    with pytest.raises(ValueError):                      # mixed operand dtypes
        lm.logprobs_shard_stats_f32(h, w.half(), 0, t)
    with pytest.raises(ValueError):                      # stats must be [g, rows, 3] fp32
        lm.logprobs_merge_shards(torch.zeros(2, 4, dtype=torch.float32))
    with pytest.raises(ValueError):
        lm.logprobs_merge_shards(torch.zeros(2, 4, 3, dtype=torch.float64))


def test_vocab_slice_logits_argument_errors(lib):
    """lmhead_logits_vocab_slice_f32: 1..8 buffers, the slice's columns inside the row stride,
    every buffer aligned and apart from the inputs and from each other; all checked before any
    CUDA call."""
    f = lm.lmhead_logits_vocab_slice_f32
    O1, O2 = 0x70000000, 0x78000000
    args = lambda **kw: dict(dict(h=A16, dt=0, rows=4, H=64, w=B16, V=300, v0=100, alpha=1.0,
                                  bias=0, outs=[O1, O2], ld=1000), **kw)
    call = lambda a: f(a["h"], a["dt"], a["rows"], a["H"], a["w"], a["V"], a["v0"], a["alpha"],
                       a["bias"], a["outs"], a["ld"], 0)
    assert call(args()) not in (1, 2, 3, 7)                  # valid: reaches the device check
    assert call(args(outs=[O1])) not in (1, 2, 3, 7)
    assert call(args(v0=700)) not in (1, 2, 3, 7)            # last column ld - 1
    assert call(args(v0=701)) == 2                           # one column past ld
    assert call(args(v0=-1)) == 2
    assert call(args(ld=0)) == 2
    assert call(args(outs=[])) == 2                          # no buffer
    assert call(args(outs=[O1 + 0x100000 * i for i in range(9)])) == 2   # more than 8
    assert call(args(dt=2)) == 2
    assert call(args(rows=2 ** 40, ld=2 ** 30)) == 2         # rows * ld * 4 bytes overflows
    assert call(args(outs=[O1, 0])) == 1
    assert call(args(outs=[O1, O2 + 2])) == 3
    assert call(args(outs=[O1, O1 + 4 * 1000])) == 7         # second buffer inside the first
    assert call(args(outs=[B16 - 64, O2])) == 7              # a buffer over W
    assert call(args(rows=0, h=0, w=0, outs=[0])) == 0       # rows == 0 launches nothing


def test_vocab_parallel_logits_wrappers_reject_bad_tensors():
    import torch
    h = torch.zeros(2, 64, dtype=torch.bfloat16)
    w = torch.zeros(8, 64, dtype=torch.bfloat16)
    o = torch.zeros(2, 16, dtype=torch.float32)
    with pytest.raises(ValueError):                      # host tensors
        lm.logits_vocab_slice_f32(h, w, 0, [o])
    with pytest.raises(ValueError):                      # no buffer
        lm.logits_vocab_slice_f32(h, w, 0, [])
