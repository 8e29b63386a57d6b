"""Build the CUDA library in-tree, for sm_100a only:

    fp32_accumulate_lm_b200/liblmhead.so        the release library
    fp32_accumulate_lm_b200/liblmhead_test.so   the same kernels plus two host-side test knobs
                                                (LMHEAD_TEST_HOOKS=1), loaded only by the tests

    python -m fp32_accumulate_lm_b200._build [--force] [--verbose]

nvcc compiles csrc/lmhead.cu with the static CUDA runtime; the runtime's symbols are kept local
to the library (--exclude-libs, -Bsymbolic) so that the CUDA runtime loaded by another library
in the same process (PyTorch's, for instance) cannot interpose on them. No fast-math flags:
the epilogue's alpha multiply must stay an IEEE multiply without flush-to-zero.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "liblmhead.so")
TEST_LIB = os.path.join(PKG, "liblmhead_test.so")
ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  glob.glob(os.path.join(INCLUDE, "*.h")))


def _compile(out: str, defines: list[str], force: bool, verbose: bool) -> str:
    newest = max(os.path.getmtime(s) for s in sources() + [os.path.abspath(__file__)])
    if not force and os.path.exists(out) and os.path.getmtime(out) >= newest:
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = [nvcc_path(), *ARCH_FLAGS, "-O3", "-lineinfo", "-std=c++17", "-shared",
           "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
           "-Xlinker", "--exclude-libs,ALL", "-Xlinker", "-Bsymbolic",
           "-I", INCLUDE, "-I", CSRC, "-cudart", "static", *defines,
           "-o", tmp, os.path.join(CSRC, "lmhead.cu")]
    if verbose:
        cmd.insert(-3, "-Xptxas")
        cmd.insert(-3, "-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError(f"nvcc failed ({res.returncode}): {' '.join(cmd)}")
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(tmp, out)
    return out


def build(force: bool = False, verbose: bool = False, test_hooks: bool = True) -> str:
    """Build the release library (and, unless test_hooks is False, the test build); return the
    release library's path."""
    _compile(LIB, [], force, verbose)
    if test_hooks:
        _compile(TEST_LIB, ["-DLMHEAD_TEST_HOOKS=1"], force, False)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
