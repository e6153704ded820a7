"""In-tree build of the CUDA library (nvcc, sm_100a).

``build_library()`` compiles ``csrc/kda_api.cu`` (which includes every kernel)
into ``libkda_b200.so`` next to this file.  The build is skipped when the
library is newer than every source file.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB_PATH = os.path.join(HERE, "libkda_b200.so")
ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH_FLAGS + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-shared"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libkda_b200.so")


def _sources():
    return (glob.glob(os.path.join(HERE, "csrc", "*.cu")) + glob.glob(os.path.join(HERE, "csrc", "*.cuh"))
            + [os.path.join(ROOT, "include", "kda.h")])


def _stale(target, sources):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def compile_so(src: str, out: str, deps, extra=(), force=False) -> str:
    if force or _stale(out, list(deps) + [src]):
        tmp = out + f".tmp{os.getpid()}"
        cmd = [nvcc()] + NVCC_FLAGS + list(extra) + ["-o", tmp, src]
        subprocess.check_call(cmd)
        os.replace(tmp, out)
    return out


def build_library(force: bool = False) -> str:
    return compile_so(os.path.join(HERE, "csrc", "kda_api.cu"), LIB_PATH, _sources(), force=force)


def build_probe(force: bool = False) -> str:
    """Test-only tcgen05 probe library (tests/csrc)."""
    src = os.path.join(ROOT, "tests", "csrc", "tc_probe.cu")
    out = os.path.join(ROOT, "tests", "csrc", "libtc_probe.so")
    return compile_so(src, out, _sources(), force=force)


if __name__ == "__main__":
    print(build_library(force=True))
    print(build_probe(force=True))
