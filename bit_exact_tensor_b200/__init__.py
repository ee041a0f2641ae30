"""Python binding for libmmaemu (bit-exact Tensor Core MMA emulation on B200).

Argument marshalling only: every arithmetic step runs in the CUDA kernels of
``libmmaemu.so`` behind the C ABI of ``include/mmaemu.h``.  PyTorch supplies
device memory and streams.  There is no CPU fallback: if the library has not
been built, or the device is not an sm_100 GPU, the calls raise.

Tensors: A and B hold fp16 / bf16 / e4m3 data (the matching torch dtype, or
raw uint16/int16/uint8 bit patterns), C and D fp32 (or raw int32 views).
"""

from __future__ import annotations

import ctypes
import os
import threading

__all__ = ["MODELS", "FORMATS", "MmaEmuError", "lib", "tiles", "gemm", "xorsum", "xorsum_noalloc", "gemm_host",
           "set_stream"]

MODELS = {"ampere": 0, "hopper": 1}
FORMATS = {"fp16": 0, "bf16": 1, "e4m3": 2}

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmmaemu.so")
_lock = threading.Lock()
_lib = None


class MmaEmuError(RuntimeError):
    def __init__(self, code: int, where: str):
        msg = lib().mmaemu_strerror(code).decode()
        super().__init__(f"{where}: {msg} (code {code})")
        self.code = code


def lib() -> ctypes.CDLL:
    """Load libmmaemu.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it first (python -c "
                                   "'import __graft_entry__ as g; g.build()')")
            L = ctypes.CDLL(LIB_PATH)
            vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
            L.mmaemu_set_stream.argtypes = [vp]
            L.mmaemu_set_stream.restype = i32
            L.mmaemu_tiles.argtypes = [i32, i32, vp, vp, vp, vp, sz]
            L.mmaemu_tiles.restype = i32
            L.mmaemu_gemm.argtypes = [i32, i32, i32, i32, i32, vp, vp, vp, vp, vp]
            L.mmaemu_gemm.restype = i32
            L.mmaemu_xorsum.argtypes = [vp, sz, ctypes.POINTER(ctypes.c_uint32)]
            L.mmaemu_xorsum.restype = i32
            L.mmaemu_strerror.argtypes = [i32]
            L.mmaemu_strerror.restype = ctypes.c_char_p
            _lib = L
        return _lib


def _torch():
    import torch

    return torch


def _check(rc: int, where: str):
    if rc != 0:
        raise MmaEmuError(rc, where)


def set_stream(stream=None):
    """Make later calls from this thread enqueue on ``stream`` (a
    torch.cuda.Stream or raw handle; None: torch's current stream)."""
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    _check(lib().mmaemu_set_stream(ctypes.c_void_p(handle)), "mmaemu_set_stream")


_IN_DTYPES = None


def _in_dtypes():
    global _IN_DTYPES
    if _IN_DTYPES is None:
        torch = _torch()
        _IN_DTYPES = {"fp16": (torch.float16, torch.int16, torch.uint16),
                      "bf16": (torch.bfloat16, torch.int16, torch.uint16),
                      "e4m3": (torch.float8_e4m3fn, torch.uint8, torch.int8)}
    return _IN_DTYPES


def _check_operand(t, fmt: str, name: str):
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype not in _in_dtypes()[fmt]:
        raise TypeError(f"{name} has dtype {t.dtype}, expected one of {_in_dtypes()[fmt]} for {fmt}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _check_f32(t, name: str):
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype not in (torch.float32, torch.int32, torch.uint32):
        raise TypeError(f"{name} must be fp32 (or an int32 view)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _model_fmt(model: str, fmt: str):
    if model not in MODELS or fmt not in FORMATS:
        raise ValueError(f"unknown model/format {model}/{fmt}")
    return MODELS[model], FORMATS[fmt]


def tiles(model: str, fmt: str, A, B, C=None, out=None):
    """D[t] = C[t] + A[t] B[t] for 16x16x16 tiles; A, B: [ntiles,16,16]."""
    torch = _torch()
    mi, fi = _model_fmt(model, fmt)
    _check_operand(A, fmt, "A")
    _check_operand(B, fmt, "B")
    nt = A.shape[0] if A.dim() == 3 else A.numel() // 256
    if A.numel() != nt * 256 or B.numel() != nt * 256:
        raise ValueError("A and B must hold ntiles*256 elements")
    if C is not None:
        _check_f32(C, "C")
        if C.numel() != nt * 256:
            raise ValueError("C must hold ntiles*256 elements")
    if out is None:
        out = torch.empty((nt, 16, 16), dtype=torch.float32, device=A.device)
    else:
        _check_f32(out, "out")
    set_stream()
    _check(lib().mmaemu_tiles(mi, fi, A.data_ptr(), B.data_ptr(), C.data_ptr() if C is not None else None,
                              out.data_ptr(), nt), "mmaemu_tiles")
    return out


def gemm(model: str, fmt: str, A, B, C=None, out=None, fingerprint: bool = True, fp_out=None):
    """D = C + A B with K walked in ascending 16-wide chunks; returns (D, fp)
    where fp holds the per-16x16-tile xorsum (None if fingerprint=False)."""
    torch = _torch()
    mi, fi = _model_fmt(model, fmt)
    _check_operand(A, fmt, "A")
    _check_operand(B, fmt, "B")
    if A.dim() != 2 or B.dim() != 2 or A.shape[1] != B.shape[0]:
        raise ValueError("A must be [M,K] and B [K,N]")
    M, K = A.shape
    N = B.shape[1]
    if C is not None:
        _check_f32(C, "C")
        if tuple(C.shape) != (M, N):
            raise ValueError("C must be [M,N]")
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32, device=A.device)
    else:
        _check_f32(out, "out")
    fp = None
    if fingerprint:
        fp = fp_out if fp_out is not None else torch.empty(((M // 16) * (N // 16),), dtype=torch.int32,
                                                           device=A.device)
    set_stream()
    _check(lib().mmaemu_gemm(mi, fi, M, N, K, A.data_ptr(), B.data_ptr(),
                             C.data_ptr() if C is not None else None, out.data_ptr(),
                             fp.data_ptr() if fp is not None else None), "mmaemu_gemm")
    return out, fp


def xorsum(t) -> int:
    """XOR of the 32-bit words of a CUDA tensor (synchronous)."""
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda or not t.is_contiguous():
        raise TypeError("xorsum needs a contiguous CUDA tensor")
    nbytes = t.numel() * t.element_size()
    if nbytes % 4:
        raise ValueError("tensor size must be a whole number of 32-bit words")
    res = ctypes.c_uint32(0)
    set_stream()
    _check(lib().mmaemu_xorsum(t.data_ptr(), nbytes // 4, ctypes.byref(res)), "mmaemu_xorsum")
    return int(res.value)


def gemm_host(model: str, fmt: str, A_host, B_host, C_host=None, fingerprint: bool = True, device="cuda"):
    """End-to-end call from host memory: copies A, B (and C) to the device,
    runs the emulated GEMM and copies D (and fingerprints) back.  Host
    tensors should be pinned for full-speed copies.  Returns CPU tensors."""
    torch = _torch()
    A = A_host.to(device, non_blocking=True)
    B = B_host.to(device, non_blocking=True)
    C = C_host.to(device, non_blocking=True) if C_host is not None else None
    D, fp = gemm(model, fmt, A, B, C, fingerprint=fingerprint)
    D_host = torch.empty(D.shape, dtype=D.dtype, pin_memory=True)
    D_host.copy_(D, non_blocking=True)
    fp_host = None
    if fp is not None:
        fp_host = torch.empty(fp.shape, dtype=fp.dtype, pin_memory=True)
        fp_host.copy_(fp, non_blocking=True)
    torch.cuda.current_stream().synchronize()
    return D_host, fp_host


def xorsum_noalloc(t) -> int:
    """Same value as :func:`xorsum`, computed without allocating any device
    memory: the library keeps a fixed scratch array for it.  Meant for code
    that cannot allocate when it needs the fingerprint (for instance a check
    that runs after the device ran out of memory, or a process whose device
    memory is fully reserved by another allocator).  At most 2^27 words;
    concurrent calls on different streams must not overlap (they share the
    scratch).  Synchronous."""
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda or not t.is_contiguous():
        raise TypeError("xorsum_noalloc needs a contiguous CUDA tensor")
    nbytes = t.numel() * t.element_size()
    if nbytes % 4:
        raise ValueError("tensor size must be a whole number of 32-bit words")
    if nbytes // 4 > NOALLOC_MAX_WORDS:
        raise ValueError(f"xorsum_noalloc handles at most {NOALLOC_MAX_WORDS} words (its fixed scratch "
                         f"limit); got {nbytes // 4}")
    fn = lib().mmaemu_xorsum_noalloc
    fn.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.POINTER(ctypes.c_uint32)]
    fn.restype = ctypes.c_int
    res = ctypes.c_uint32(0)
    set_stream()
    _check(fn(t.data_ptr(), nbytes // 4, ctypes.byref(res)), "mmaemu_xorsum_noalloc")
    return int(res.value)


NOALLOC_MAX_WORDS = 1 << 27  # MMAEMU_XORSUM_NOALLOC_MAX_WORDS
