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

__all__ = ["MODELS", "FORMATS", "MmaEmuError", "lib", "tiles", "gemm", "gemm_verify", "gemm_batched", "xorsum",
           "xorsum_noalloc", "gemm_host", "tiles_host", "set_stream", "trim_workspace", "set_workspace_cache", "workspace_reserved",
           "device_status", "selftest_wait_timeout", "bounds_checking", "NO_MISMATCH"]

MODELS = {"ampere": 0, "hopper": 1, "b200": 2, "lovelace": 0}
FORMATS = {"fp16": 0, "bf16": 1, "e4m3": 2}

_HERE = os.path.dirname(os.path.abspath(__file__))
# MMAEMU_LIB=check selects the bounds-checking build (libmmaemu_check.so):
# every kernel index is checked against its buffer and a violation is
# recorded in the device status word (see device_status) instead of being
# made.  It is slower and meant for tests.  MMAEMU_LIB=<path to a .so>
# loads another build of the same sources (for instance one compiled with
# other tuning constants).
_SEL = os.environ.get("MMAEMU_LIB", "")
LIB_PATH = (os.path.join(_HERE, "libmmaemu_check.so") if _SEL == "check"
            else _SEL if _SEL.endswith(".so") else os.path.join(_HERE, "libmmaemu.so"))
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
            L.mmaemu_gemm_verify.argtypes = [i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp]
            L.mmaemu_gemm_verify.restype = i32
            i64 = ctypes.c_longlong
            L.mmaemu_gemm_strided_batched.argtypes = [i32, i32, i32, i32, i32, i32, i32, i32, vp, i64, i64, vp, i64,
                                                      i64, vp, i64, i64, vp, i64, i64, vp, i64]
            L.mmaemu_gemm_strided_batched.restype = i32
            L.mmaemu_xorsum.argtypes = [vp, sz, ctypes.POINTER(ctypes.c_uint32)]
            L.mmaemu_xorsum.restype = i32
            L.mmaemu_strerror.argtypes = [i32]
            L.mmaemu_strerror.restype = ctypes.c_char_p
            L.mmaemu_set_workspace_cache.argtypes = [i32]
            L.mmaemu_set_workspace_cache.restype = i32
            L.mmaemu_workspace_reserved.argtypes = [ctypes.POINTER(sz)]
            L.mmaemu_workspace_reserved.restype = i32
            L.mmaemu_trim_workspace.argtypes = []
            L.mmaemu_trim_workspace.restype = i32
            L.mmaemu_device_status.argtypes = [i32, ctypes.POINTER(ctypes.c_uint32)]
            L.mmaemu_device_status.restype = i32
            L.mmaemu_selftest_wait_timeout.argtypes = [ctypes.c_uint, ctypes.POINTER(i32)]
            L.mmaemu_selftest_wait_timeout.restype = i32
            L.mmaemu_bounds_checking.argtypes = []
            L.mmaemu_bounds_checking.restype = i32
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


def _device_of(*tensors):
    """The one CUDA device all given tensors live on (None entries are
    skipped); raises before any launch if they differ.  Calls run with that
    device current and on its current stream, so a tensor on another GPU
    than the current one is never handed to a kernel on the wrong device."""
    devs = {t.device for t in tensors if t is not None}
    if len(devs) != 1:
        raise ValueError(f"operands must all be on one CUDA device, got {sorted(str(d) for d in devs)}")
    (dev,) = devs
    if dev.type != "cuda":
        raise TypeError("operands must be CUDA tensors")
    return dev


class _on_device:
    """Context: make ``dev`` current and select its current stream."""

    def __init__(self, dev):
        self.dev = dev

    def __enter__(self):
        torch = _torch()
        self.ctx = torch.cuda.device(self.dev)
        self.ctx.__enter__()
        set_stream(torch.cuda.current_stream(self.dev))
        return self

    def __exit__(self, *exc):
        return self.ctx.__exit__(*exc)


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
    with _on_device(_device_of(A, B, C, out)):
        _check(lib().mmaemu_tiles(mi, fi, A.data_ptr(), B.data_ptr(), C.data_ptr() if C is not None else None,
                                  out.data_ptr(), nt), "mmaemu_tiles")
    return out


def _gemm_shapes(A, B, C, fmt):
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
    return M, N, K


def gemm(model: str, fmt: str, A, B, C=None, out=None, fingerprint: bool = True, fp_out=None,
         store_d: bool = True):
    """D = C + A B with K walked in ascending 16-wide chunks; returns (D, fp)
    where fp holds the per-16x16-tile xorsum (None if fingerprint=False).
    store_d=False is the fingerprint-only mode: D is not written (None)."""
    torch = _torch()
    mi, fi = _model_fmt(model, fmt)
    M, N, K = _gemm_shapes(A, B, C, fmt)
    if not store_d:
        if not fingerprint:
            raise ValueError("store_d=False needs fingerprint=True")
        out = None
    elif out is None:
        out = torch.empty((M, N), dtype=torch.float32, device=A.device)
    else:
        _check_f32(out, "out")
    fp = None
    if fingerprint:
        fp = fp_out if fp_out is not None else torch.empty(((M // 16) * (N // 16),), dtype=torch.int32,
                                                           device=A.device)
    if fp is not None and (not fp.is_cuda or fp.numel() != (M // 16) * (N // 16) or fp.element_size() != 4
                           or not fp.is_contiguous()):
        raise ValueError("fp_out must be a contiguous CUDA tensor of (M/16)*(N/16) 32-bit words")
    with _on_device(_device_of(A, B, C, out, fp)):
        _check(lib().mmaemu_gemm(mi, fi, M, N, K, A.data_ptr(), B.data_ptr(),
                                 C.data_ptr() if C is not None else None, out.data_ptr() if out is not None else None,
                                 fp.data_ptr() if fp is not None else None), "mmaemu_gemm")
    return out, fp


NO_MISMATCH = -1  # mismatch index word when nothing differs (2^64 - 1 read as int64)


def gemm_verify(model: str, fmt: str, A, B, C, D_claimed, fingerprint: bool = False, mismatch_out=None):
    """Recompute D = C + A B and compare it bit for bit with D_claimed
    without storing it.  Returns (mismatch, fp): mismatch is an int64 CUDA
    tensor [count, first] (first = smallest row-major index of a differing
    element, NO_MISMATCH if none), filled asynchronously; fp the fingerprints
    of the recomputed D (None if fingerprint=False)."""
    torch = _torch()
    mi, fi = _model_fmt(model, fmt)
    M, N, K = _gemm_shapes(A, B, C, fmt)
    _check_f32(D_claimed, "D_claimed")
    if tuple(D_claimed.shape) != (M, N):
        raise ValueError("D_claimed must be [M,N]")
    mism = mismatch_out if mismatch_out is not None else torch.empty((2,), dtype=torch.int64, device=A.device)
    if mism.dtype != torch.int64 or mism.numel() != 2 or not mism.is_cuda:
        raise TypeError("mismatch_out must be a CUDA int64 tensor of 2 elements")
    fp = torch.empty(((M // 16) * (N // 16),), dtype=torch.int32, device=A.device) if fingerprint else None
    with _on_device(_device_of(A, B, C, D_claimed, fp, mism)):
        _check(lib().mmaemu_gemm_verify(mi, fi, M, N, K, A.data_ptr(), B.data_ptr(),
                                        C.data_ptr() if C is not None else None, D_claimed.data_ptr(),
                                        fp.data_ptr() if fp is not None else None, mism.data_ptr()),
               "mmaemu_gemm_verify")
    return mism, fp


def _operand_layout(t, name: str):
    """(trans, ld, batch stride) of a [batch, rows, cols] (or [rows, cols])
    view whose rows or columns are contiguous."""
    rs, cs = t.stride(-2), t.stride(-1)
    bs = t.stride(0) if t.dim() == 3 else 0
    if cs == 1 and (rs >= t.shape[-1] or t.shape[-2] == 1):
        return 0, max(rs, t.shape[-1]), bs
    if rs == 1 and (cs >= t.shape[-2] or t.shape[-1] == 1):
        return 1, max(cs, t.shape[-2]), bs
    raise ValueError(f"{name} needs unit stride along its rows or its columns")


def gemm_batched(model: str, fmt: str, A, B, C=None, out=None, fingerprint: bool = True, store_d: bool = True):
    """Batched D[b] = C[b] + A[b] B[b], each entry with the K-chained
    arithmetic of gemm.  A: [batch, M, K] or [M, K] (shared), B: [batch, K,
    N] or [K, N], as strided views: each operand needs unit stride along its
    rows or along its columns (so A.transpose(-1, -2) views of [K, M] storage
    work without copies).  C, out: [batch, M, N] with unit column stride.
    Returns (D, fp) with fp [batch, (M/16)*(N/16)]."""
    torch = _torch()
    mi, fi = _model_fmt(model, fmt)
    for t, name in ((A, "A"), (B, "B")):
        if not isinstance(t, torch.Tensor) or not t.is_cuda:
            raise TypeError(f"{name} must be a CUDA tensor")
        if t.dtype not in _in_dtypes()[fmt]:
            raise TypeError(f"{name} has dtype {t.dtype}, expected one of {_in_dtypes()[fmt]} for {fmt}")
        if t.dim() not in (2, 3):
            raise ValueError(f"{name} must be 2-D or 3-D")
    batch = max(A.shape[0] if A.dim() == 3 else 1, B.shape[0] if B.dim() == 3 else 1)
    for t, name in ((A, "A"), (B, "B")):
        if t.dim() == 3 and t.shape[0] != batch:
            raise ValueError(f"{name} batch size {t.shape[0]} != {batch}")
    M, K = A.shape[-2:]
    K2, N = B.shape[-2:]
    if K != K2:
        raise ValueError("inner dimensions differ")
    ta, lda, sa = _operand_layout(A, "A")
    tb, ldb, sb = _operand_layout(B, "B")

    def f32_layout(t, name):
        if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype not in (torch.float32, torch.int32):
            raise TypeError(f"{name} must be a CUDA fp32 tensor")
        if tuple(t.shape[-2:]) != (M, N) or (t.dim() == 3 and t.shape[0] != batch):
            raise ValueError(f"{name} must be [batch, M, N] or [M, N]")
        if t.stride(-1) != 1:
            raise ValueError(f"{name} needs unit column stride")
        return t.stride(-2), (t.stride(0) if t.dim() == 3 else 0)

    ldc, sc = f32_layout(C, "C") if C is not None else (N, 0)
    if not store_d:
        if not fingerprint:
            raise ValueError("store_d=False needs fingerprint=True")
        out = None
    elif out is None:
        out = torch.empty((batch, M, N), dtype=torch.float32, device=A.device)
    ldd, sd = f32_layout(out, "out") if out is not None else (N, 0)
    if out is not None and batch > 1 and sd == 0:
        raise ValueError("out entries of a batch must not overlap")
    tiles_per = (M // 16) * (N // 16)
    fp = torch.empty((batch, tiles_per), dtype=torch.int32, device=A.device) if fingerprint else None
    with _on_device(_device_of(A, B, C, out, fp)):
        _check(lib().mmaemu_gemm_strided_batched(
            mi, fi, ta, tb, M, N, K, batch,
            A.data_ptr(), lda, sa, B.data_ptr(), ldb, sb,
            C.data_ptr() if C is not None else None, ldc, sc,
            out.data_ptr() if out is not None else None, ldd, sd,
            fp.data_ptr() if fp is not None else None, tiles_per), "mmaemu_gemm_strided_batched")
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
    with _on_device(_device_of(t)):
        _check(lib().mmaemu_xorsum(t.data_ptr(), nbytes // 4, ctypes.byref(res)), "mmaemu_xorsum")
    return int(res.value)


def gemm_host(model: str, fmt: str, A_host, B_host, C_host=None, fingerprint: bool = True, device=None,
              out=None, fp_out=None, store_d: bool = True):
    """End-to-end call from host memory (mmaemu_gemm_host): host A, B (and C)
    in, host D and fingerprints out, with the transfers overlapped with the
    arithmetic inside the library.  Host tensors should be page-locked
    (``tensor.pin_memory()``) for the overlap.  ``device`` selects the CUDA
    device (default: the current one).  ``out`` / ``fp_out`` take the results
    in caller-owned host tensors (contiguous, 32-bit elements: [M, N] and
    [(M/16)*(N/16)]; fp_out implies fingerprint); otherwise page-locked
    ones are allocated per call.  store_d=False is the fingerprint-only
    mode: D is neither written nor copied back (None).  Returns CPU tensors
    (D, fp)."""
    torch = _torch()
    mi, fi = _model_fmt(model, fmt)
    for t, name in ((A_host, "A"), (B_host, "B")):
        if not isinstance(t, torch.Tensor) or t.is_cuda or not t.is_contiguous():
            raise TypeError(f"{name} must be a contiguous CPU tensor")
        if t.dtype not in _in_dtypes()[fmt]:
            raise TypeError(f"{name} has dtype {t.dtype}, expected one of {_in_dtypes()[fmt]} for {fmt}")
    if A_host.dim() != 2 or B_host.dim() != 2 or A_host.shape[1] != B_host.shape[0]:
        raise ValueError("A must be [M,K] and B [K,N]")
    M, K = A_host.shape
    N = B_host.shape[1]
    if C_host is not None:
        if C_host.is_cuda or not C_host.is_contiguous() or tuple(C_host.shape) != (M, N) or \
                C_host.dtype not in (torch.float32, torch.int32, torch.uint32):
            raise TypeError("C must be a contiguous CPU fp32 tensor [M,N]")
    words = (torch.float32, torch.int32, torch.uint32)
    if not store_d:
        if not fingerprint and fp_out is None:
            raise ValueError("store_d=False needs fingerprint=True")
        if out is not None:
            raise ValueError("store_d=False writes no D: out must be None")
        D_host = None
    elif out is not None:
        if not isinstance(out, torch.Tensor) or out.is_cuda or not out.is_contiguous() or \
                tuple(out.shape) != (M, N) or out.dtype not in words:
            raise TypeError("out must be a contiguous CPU tensor [M,N] of 32-bit elements")
        D_host = out
    else:
        D_host = torch.empty((M, N), dtype=torch.float32, pin_memory=True)
    if fp_out is not None:
        if not isinstance(fp_out, torch.Tensor) or fp_out.is_cuda or not fp_out.is_contiguous() or \
                fp_out.numel() != (M // 16) * (N // 16) or fp_out.dtype not in words[1:]:
            raise TypeError("fp_out must be a contiguous CPU int32 tensor of (M/16)*(N/16) elements")
        fp_host = fp_out
    else:
        fp_host = torch.empty(((M // 16) * (N // 16),), dtype=torch.int32, pin_memory=True) if fingerprint else None
    with torch.cuda.device(device if device is not None else torch.cuda.current_device()):
        set_stream(torch.cuda.current_stream())
        fn = lib().mmaemu_gemm_host
        fn.argtypes = [ctypes.c_int] * 5 + [ctypes.c_void_p] * 5
        fn.restype = ctypes.c_int
        _check(fn(mi, fi, M, N, K, A_host.data_ptr(), B_host.data_ptr(),
                  C_host.data_ptr() if C_host is not None else None,
                  D_host.data_ptr() if D_host is not None else None,
                  fp_host.data_ptr() if fp_host is not None else None), "mmaemu_gemm_host")
    return D_host, fp_host


def tiles_host(model: str, fmt: str, A_host, B_host, C_host=None, device=None, out=None):
    """End-to-end tile batch from host memory (mmaemu_tiles_host): host A, B
    (and C) [ntiles,16,16] in, host D out, streamed in chunks with the copies
    in both directions overlapped with the arithmetic.  Host tensors should
    be page-locked (``tensor.pin_memory()``).  ``out`` takes D in a
    caller-owned contiguous CPU tensor of ntiles*256 32-bit elements;
    otherwise a page-locked one is allocated.  Returns the CPU tensor D."""
    torch = _torch()
    mi, fi = _model_fmt(model, fmt)
    for t, name in ((A_host, "A"), (B_host, "B")):
        if not isinstance(t, torch.Tensor) or t.is_cuda or not t.is_contiguous():
            raise TypeError(f"{name} must be a contiguous CPU tensor")
        if t.dtype not in _in_dtypes()[fmt]:
            raise TypeError(f"{name} has dtype {t.dtype}, expected one of {_in_dtypes()[fmt]} for {fmt}")
    nt = A_host.numel() // 256
    if A_host.numel() != nt * 256 or B_host.numel() != nt * 256:
        raise ValueError("A and B must hold ntiles x 16 x 16 elements each")
    words = (torch.float32, torch.int32, torch.uint32)
    if C_host is not None and (not isinstance(C_host, torch.Tensor) or C_host.is_cuda or
                               not C_host.is_contiguous() or C_host.numel() != nt * 256 or C_host.dtype not in words):
        raise TypeError("C must be a contiguous CPU fp32 tensor of ntiles x 16 x 16 elements")
    if out is not None:
        if not isinstance(out, torch.Tensor) or out.is_cuda or not out.is_contiguous() or \
                out.numel() != nt * 256 or out.dtype not in words:
            raise TypeError("out must be a contiguous CPU tensor of ntiles x 16 x 16 32-bit elements")
        D_host = out
    else:
        D_host = torch.empty((nt, 16, 16), dtype=torch.float32, pin_memory=True)
    with torch.cuda.device(device if device is not None else torch.cuda.current_device()):
        set_stream(torch.cuda.current_stream())
        fn = lib().mmaemu_tiles_host
        fn.argtypes = [ctypes.c_int] * 2 + [ctypes.c_void_p] * 4 + [ctypes.c_size_t]
        fn.restype = ctypes.c_int
        _check(fn(mi, fi, A_host.data_ptr(), B_host.data_ptr(), C_host.data_ptr() if C_host is not None else None,
                  D_host.data_ptr(), nt), "mmaemu_tiles_host")
    return D_host


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
    with _on_device(_device_of(t)):
        _check(fn(t.data_ptr(), nbytes // 4, ctypes.byref(res)), "mmaemu_xorsum_noalloc")
    return int(res.value)


NOALLOC_MAX_WORDS = 1 << 27  # MMAEMU_XORSUM_NOALLOC_MAX_WORDS


def trim_workspace():
    """Return the current device's unused GEMM workspace (cached decoded
    operands of earlier calls, see set_workspace_cache) to the device."""
    _check(lib().mmaemu_trim_workspace(), "mmaemu_trim_workspace")


def set_workspace_cache(enable: bool):
    """Opt in (or out) of keeping the GEMM workspace between calls on the
    current device.  Off by default: each GEMM's decoded-operand workspace
    goes back to the device at the next synchronisation, so the library
    holds no device memory between calls.  On, repeated GEMMs reuse it and
    skip the allocation; turning it off trims what is held."""
    _check(lib().mmaemu_set_workspace_cache(1 if enable else 0), "mmaemu_set_workspace_cache")


def workspace_reserved() -> int:
    """Bytes of device memory the library's workspace pool holds on the
    current device right now."""
    v = ctypes.c_size_t(0)
    _check(lib().mmaemu_workspace_reserved(ctypes.byref(v)), "mmaemu_workspace_reserved")
    return int(v.value)


STATUS_TIMEOUT, STATUS_BOUNDS = 1, 2


def device_status(clear: bool = True) -> int:
    """Bits the kernels recorded on the current device since the last clear
    (waits for torch's current stream): STATUS_TIMEOUT -- a bounded wait
    gave up; STATUS_BOUNDS -- the bounds-checking build found an index
    outside its buffer.  Returns the bits (0: nothing recorded)."""
    torch = _torch()
    bits = ctypes.c_uint32(0)
    set_stream(torch.cuda.current_stream())
    rc = lib().mmaemu_device_status(1 if clear else 0, ctypes.byref(bits))
    if rc not in (0, -3, -6):  # OK, ETIMEOUT, EBOUNDS carry the bits
        _check(rc, "mmaemu_device_status")
    return int(bits.value)


def selftest_wait_timeout(spins: int) -> bool:
    """Run a kernel whose bounded wait can never complete (nothing ever
    arrives) with a bound of ``spins`` tries; returns whether it completed
    (always False).  The timeout is recorded in device_status."""
    torch = _torch()
    done = ctypes.c_int(0)
    set_stream(torch.cuda.current_stream())
    _check(lib().mmaemu_selftest_wait_timeout(spins, ctypes.byref(done)), "mmaemu_selftest_wait_timeout")
    return bool(done.value)


def bounds_checking() -> bool:
    """True when the loaded library is the bounds-checking build."""
    return bool(lib().mmaemu_bounds_checking())
