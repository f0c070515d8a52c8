"""Builds librtlayer.so in-tree with nvcc for sm_100a (B200).

Usage: python -m blocked_attention_b200.build [--force] [--verbose] [--bounds-check]

--bounds-check builds the debug library librtlayer_check.so instead (device
bounds checks on the kernels' computed indexes, recorded in the error word).
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
LIB = os.path.join(PKG, "librtlayer.so")
# debug build: device-side bounds checks on the kernels' computed indexes
# (-DRT_BOUNDS_CHECK), recorded in the error word instead of trapping
LIB_CHECK = os.path.join(PKG, "librtlayer_check.so")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    p = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(p):
        raise RuntimeError("nvcc not found")
    return p


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(INCLUDE, "*.h")))


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(s) <= t for s in _sources())


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None,
          bounds_check: bool = False) -> str:
    lib = LIB_CHECK if bounds_check else LIB
    if not force and up_to_date(lib):
        return lib
    # a per-process temporary, atomically renamed: concurrent builders (one
    # process per GPU) never write the same file, and readers see either the
    # old or the new library, whole
    tmp = f"{lib}.tmp{os.getpid()}"
    cmd = [nvcc_path(), *ARCH_FLAGS, "-O3", "-lineinfo", "-std=c++17", "--shared",
           "-Xcompiler", "-fPIC", "-I", INCLUDE, "-o", tmp,
           *(["-DRT_BOUNDS_CHECK"] if bounds_check else []),
           *sorted(glob.glob(os.path.join(CSRC, "*.cu")))]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    if extra:
        cmd[1:1] = extra
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        if os.path.exists(tmp):
            os.remove(tmp)
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    os.replace(tmp, lib)
    if verbose:
        sys.stdout.write(r.stdout + r.stderr)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv,
                bounds_check="--bounds-check" in sys.argv))
