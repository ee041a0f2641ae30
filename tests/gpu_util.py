"""Helpers for the GPU parity tests: numpy bit patterns <-> CUDA tensors."""

import numpy as np


def dev_in(x: np.ndarray):
    import torch

    x = np.ascontiguousarray(x)
    if x.dtype == np.uint8:
        return torch.from_numpy(x).cuda()
    return torch.from_numpy(x.view(np.int16)).cuda()


def dev_f32(x: np.ndarray):
    import torch

    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.uint32).view(np.int32)).cuda()


def host_bits(t) -> np.ndarray:
    import torch

    return t.contiguous().view(torch.int32).cpu().numpy().view(np.uint32)


def first_mismatch(got: np.ndarray, want: np.ndarray) -> str:
    bad = np.argwhere(got != want)
    if bad.size == 0:
        return "equal"
    idx = tuple(bad[0])
    return f"{bad.shape[0]} mismatches; first at {idx}: got {got[idx]:08X} want {want[idx]:08X}"


# Guard words around output buffers: a kernel that writes outside its output
# changes them (a substitute for a memory checker, which this pool does not
# run).  The inner view starts 256 bytes into the buffer, so it keeps the
# 16-byte alignment the library requires.
GUARD = 0x5A5AA5A5
GUARD_WORDS = 64


def guarded(shape, dtype="float32"):
    """(buffer, inner view): a CUDA buffer of 32-bit words filled with GUARD
    and a contiguous view of `shape` inside it, GUARD_WORDS words from each
    end."""
    import torch

    n = int(np.prod(shape))
    buf = torch.full((n + 2 * GUARD_WORDS,), GUARD, dtype=torch.int32, device="cuda")
    inner = buf[GUARD_WORDS:GUARD_WORDS + n].view(*shape)
    return buf, (inner.view(torch.float32) if dtype == "float32" else inner)


def guards_intact(buf) -> bool:
    w = buf.cpu().numpy().view(np.uint32)
    return bool((w[:GUARD_WORDS] == GUARD).all() and (w[-GUARD_WORDS:] == GUARD).all())


def fullsize_digests(D: np.ndarray, fp: np.ndarray) -> dict:
    """The digests tests/golden/make_fullsize.py stores for the oracle's
    result (loaded from that script so both sides hash the same way)."""
    import importlib.util
    import os

    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "make_fullsize.py")
    spec = importlib.util.spec_from_file_location("make_fullsize", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.digests(D, fp)
