"""Build libkda.so in-tree with nvcc for sm_100a.

    python -m gated_delta_rule_110_b200.build [--force] [--verbose-ptxas]

The library is a single translation unit (csrc/kda_api.cu includes the kernel
headers), compiled for ``-gencode arch=compute_100a,code=sm_100a`` only.  A
second copy, libkda_testhooks.so, is built with -DKDA_TEST_HOOKS for the
failure-detection test.
"""
from __future__ import annotations

import os
import subprocess
import sys
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
CSRC = PKG / "csrc"
INCLUDE = ROOT / "include"
LIB = PKG / "libkda.so"

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def sources():
    return sorted(CSRC.glob("*.cu")) + sorted(CSRC.glob("*.cuh")) + [INCLUDE / "kda.h"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (Path(cand).exists() or cand == "nvcc"):
            return cand
    return "nvcc"


# Test-only build: short bounded waits and a host-armed missing signal, for
# the failure-detection test (tests/test_gpu_timeout.py).  Never loaded by the
# package itself.
TEST_LIB = PKG / "libkda_testhooks.so"


def up_to_date_lib(lib: Path) -> bool:
    if not lib.exists():
        return False
    t = lib.stat().st_mtime
    return all(p.stat().st_mtime <= t for p in sources())


def _compile(out: Path, extra, verbose_ptxas: bool):
    tmp = out.with_suffix(f".so.tmp{os.getpid()}")
    cmd = [nvcc(), *NVCC_FLAGS, *extra, f"-I{INCLUDE}", f"-I{CSRC}", str(CSRC / "kda_api.cu"), "-o", str(tmp)]
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    os.replace(tmp, out)


def build(force: bool = False, verbose_ptxas: bool = False, test_hooks: bool = True) -> Path:
    if force or not up_to_date_lib(LIB):
        _compile(LIB, [], verbose_ptxas)
    if test_hooks and (force or not up_to_date_lib(TEST_LIB)):
        _compile(TEST_LIB, ["-DKDA_TEST_HOOKS"], False)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose_ptxas="--verbose-ptxas" in sys.argv)
    print(LIB)
