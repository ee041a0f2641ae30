"""Build libmmaemu.so (and its bounds-checking twin) in-tree with nvcc for sm_100a.

libmmaemu.so        -- the library.
libmmaemu_check.so  -- the same sources with MMAEMU_BOUNDS_CHECK: every
                       kernel index is checked against its buffer and a
                       violation is recorded in the device status word
                       instead of being made (selected with MMAEMU_LIB=check).
libmmaemu_peaks.so  -- issue-rate probes of the instruction classes the
                       kernels use (bench.py --pipe-rates), for their rooflines.
"""

from __future__ import annotations

import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = os.path.join(PKG, "csrc", "mmaemu.cu")
SOURCES = [SRC, os.path.join(PKG, "csrc", "probe.cpp")]
DEPS = SOURCES + [os.path.join(PKG, "csrc", "mmaemu_core.cuh"), os.path.join(PKG, "csrc", "host_slabs.h"),
                  os.path.join(ROOT, "include", "mmaemu.h"),
                  os.path.join(ROOT, "include", "mmaemu_probe.h"), os.path.abspath(__file__)]
LIB = os.path.join(PKG, "libmmaemu.so")
LIB_CHECK = os.path.join(PKG, "libmmaemu_check.so")
LIB_PEAKS = os.path.join(PKG, "libmmaemu_peaks.so")
PEAKS_SRC = os.path.join(PKG, "csrc", "peaks.cu")

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
              "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2"]
VARIANTS = {LIB: [], LIB_CHECK: ["-DMMAEMU_BOUNDS_CHECK"]}


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def needs_build(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(d) > t for d in DEPS)


def _build_one(lib: str, extra: list[str], verbose: bool) -> str:
    tmp = lib + f".{os.getpid()}.tmp"
    srcs = [PEAKS_SRC] if lib == LIB_PEAKS else SOURCES
    cmd = [nvcc(), *NVCC_FLAGS, *extra, "-I", os.path.join(ROOT, "include"), *srcs, "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


def build_library(force: bool = False, verbose: bool = False, checking: bool = True) -> str:
    todo = [(lib, extra) for lib, extra in VARIANTS.items()
            if (checking or lib == LIB) and (force or needs_build(lib))]
    if force or not os.path.exists(LIB_PEAKS) or os.path.getmtime(LIB_PEAKS) < os.path.getmtime(PEAKS_SRC):
        todo.append((LIB_PEAKS, []))
    with ThreadPoolExecutor(max_workers=len(todo) or 1) as ex:
        for f in [ex.submit(_build_one, lib, extra, verbose) for lib, extra in todo]:
            f.result()
    return LIB


if __name__ == "__main__":
    print(build_library(force=True, verbose=True))
