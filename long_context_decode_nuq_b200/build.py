"""Build libkvq.so (and the input generator's libkvqsynth.so) in-tree with nvcc for sm_100a.

Usage: python -m long_context_decode_nuq_b200.build [--force]
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libkvq.so")
SYNTH_SRC = os.path.join(ROOT, "synth", "gen.cu")
SYNTH_LIB = os.path.join(ROOT, "synth", "libkvqsynth.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def _stale(target: str, sources) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def _compile(target: str, sources, extra=(), force=False) -> None:
    if not force and not _stale(target, sources):
        return
    tmp = target + ".tmp"
    cu = [s for s in sources if s.endswith(".cu")]
    cmd = [_nvcc(), *NVCC_FLAGS, *extra, "-o", tmp, *cu]
    subprocess.run(cmd, check=True)
    os.replace(tmp, target)


def build(force: bool = False) -> str:
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + [os.path.join(ROOT, "include", "kvq.h")])
    _compile(LIB, srcs, force=force)
    _compile(SYNTH_LIB, [SYNTH_SRC], force=force)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
