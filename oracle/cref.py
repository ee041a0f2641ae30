"""Build and call the plain C oracle (``mmaemu_ref.c``).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  The C oracle restates
the same per-element rules as ``mma_model.py`` and exists because the
full-size workloads (hundreds of millions of emulated MACs) are far beyond a
pure-Python loop.  Inputs and outputs are numpy arrays of raw bit patterns:
uint16 for fp16/bf16, uint8 for e4m3, uint32 for fp32.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mmaemu_ref.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB = os.path.join(_BUILD, "liborc.so")

MODEL = {"ampere": 0, "hopper": 1, "b200": 2}
FMT = {"fp16": 0, "bf16": 1, "e4m3": 2}
IN_DTYPE = {"fp16": np.uint16, "bf16": np.uint16, "e4m3": np.uint8}

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into oracle/_build/liborc.so (gcc, -O2)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.run(["gcc", "-O2", "-std=c99", "-Wall", "-Wextra", "-shared", "-fPIC",
                        "-pthread", _SRC, "-o", tmp], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            vp, sz, u32, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_uint32, ctypes.c_int
            L.orc_supported.argtypes = [i32, i32]
            L.orc_mma_element.argtypes = [i32, i32, vp, vp, u32]
            L.orc_mma_element.restype = u32
            L.orc_tiles.argtypes = [i32, i32, vp, vp, vp, vp, sz, i32]
            L.orc_gemm_element.argtypes = [i32, i32, i32, i32, i32, vp, vp, vp, i32, i32]
            L.orc_gemm_element.restype = u32
            L.orc_gemm_region.argtypes = [i32, i32, i32, i32, i32, vp, vp, vp, vp, i32, i32, i32, i32, i32]
            L.orc_xorsum.argtypes = [vp, sz]
            L.orc_xorsum.restype = u32
            L.orc_tile_fingerprints.argtypes = [vp, i32, i32, vp]
            _lib = L
        return _lib


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def _check_in(fmt: str, x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x)
    assert x.dtype == IN_DTYPE[fmt], (x.dtype, fmt)
    return x


def mma_element(model: str, fmt: str, a16, b16, c_bits: int) -> int:
    a = _check_in(fmt, np.asarray(a16, dtype=IN_DTYPE[fmt]))
    b = _check_in(fmt, np.asarray(b16, dtype=IN_DTYPE[fmt]))
    assert a.size == 16 and b.size == 16
    return int(lib().orc_mma_element(MODEL[model], FMT[fmt], _ptr(a), _ptr(b), int(c_bits)))


def tiles(model: str, fmt: str, A: np.ndarray, B: np.ndarray, C: np.ndarray | None,
          nthreads: int | None = None) -> np.ndarray:
    """A, B: [ntiles,16,16] raw patterns; C: [ntiles,16,16] uint32 or None."""
    A, B = _check_in(fmt, A), _check_in(fmt, B)
    nt = A.shape[0]
    assert A.shape == (nt, 16, 16) and B.shape == (nt, 16, 16)
    if C is not None:
        C = np.ascontiguousarray(C, dtype=np.uint32)
        assert C.shape == (nt, 16, 16)
    D = np.empty((nt, 16, 16), dtype=np.uint32)
    rc = lib().orc_tiles(MODEL[model], FMT[fmt], _ptr(A), _ptr(B), _ptr(C), _ptr(D), nt,
                         nthreads or default_threads())
    if rc != 0:
        raise ValueError(f"unsupported pair {model}/{fmt}")
    return D


def gemm(model: str, fmt: str, A: np.ndarray, B: np.ndarray, C: np.ndarray | None,
         rows: tuple[int, int] | None = None, cols: tuple[int, int] | None = None,
         nthreads: int | None = None) -> np.ndarray:
    """Full (or a rectangular region of the) K-chained GEMM; returns D [M,N]
    uint32 with only the requested region filled (the rest is zero)."""
    A, B = _check_in(fmt, A), _check_in(fmt, B)
    M, K = A.shape
    K2, N = B.shape
    assert K == K2
    if C is not None:
        C = np.ascontiguousarray(C, dtype=np.uint32)
        assert C.shape == (M, N)
    D = np.zeros((M, N), dtype=np.uint32)
    r0, r1 = rows or (0, M)
    c0, c1 = cols or (0, N)
    rc = lib().orc_gemm_region(MODEL[model], FMT[fmt], M, N, K, _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                               r0, r1, c0, c1, nthreads or default_threads())
    if rc != 0:
        raise ValueError("unsupported pair or shape")
    return D


def gemm_element(model: str, fmt: str, A: np.ndarray, B: np.ndarray, C: np.ndarray | None,
                 m: int, n: int) -> int:
    A, B = _check_in(fmt, A), _check_in(fmt, B)
    M, K = A.shape
    N = B.shape[1]
    if C is not None:
        C = np.ascontiguousarray(C, dtype=np.uint32)
    return int(lib().orc_gemm_element(MODEL[model], FMT[fmt], M, N, K, _ptr(A), _ptr(B), _ptr(C), m, n))


def xorsum(words: np.ndarray) -> int:
    w = np.ascontiguousarray(words).view(np.uint32).ravel()
    return int(lib().orc_xorsum(_ptr(w), w.size))


def tile_fingerprints(D: np.ndarray) -> np.ndarray:
    D = np.ascontiguousarray(D, dtype=np.uint32)
    M, N = D.shape
    fp = np.empty((M // 16) * (N // 16), dtype=np.uint32)
    lib().orc_tile_fingerprints(_ptr(D), M, N, _ptr(fp))
    return fp
