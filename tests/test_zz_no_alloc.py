"""The allocation-free xorsum gives the same value as mmaemu_xorsum and the oracle.

mmaemu_xorsum_noalloc exists for callers that cannot allocate device memory
at the point where they need a fingerprint (a check that runs after the
device ran out of memory, or a process whose device memory is wholly
reserved by another allocator).  Its scratch is a fixed array in the library
image, shared by every call, so two calls in a row must each still give the
right answer whatever the previous call left there.  Both entry points are
called through the C ABI, and the value is also checked against the oracle's
xorsum of the same words.  Once warmed up on a device, a call takes no device
memory: the free memory the driver reports is the same before and after.
"""

import ctypes

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

MAX_WORDS = 1 << 27  # MMAEMU_XORSUM_NOALLOC_MAX_WORDS


def _abi():
    import bit_exact_tensor_b200 as mmaemu

    L = mmaemu.lib()
    for name in ("mmaemu_xorsum", "mmaemu_xorsum_noalloc"):
        f = getattr(L, name)
        f.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.POINTER(ctypes.c_uint32)]
        f.restype = ctypes.c_int
    return L


def _both(L, t, n):
    import torch

    torch.cuda.synchronize()
    a, b = ctypes.c_uint32(0), ctypes.c_uint32(0)
    assert L.mmaemu_set_stream(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0
    assert L.mmaemu_xorsum(t.data_ptr(), n, ctypes.byref(a)) == 0
    assert L.mmaemu_xorsum_noalloc(t.data_ptr(), n, ctypes.byref(b)) == 0
    return a.value, b.value


@pytest.mark.parametrize("n", [1, 3, 4, 8191, 8192, 8193, 1_000_003, MAX_WORDS])
def test_noalloc_equals_xorsum_two_calls_in_a_row(cref, n):
    import torch

    L = _abi()
    rng = np.random.default_rng(n)
    for call in range(2):  # the second call sees the first call's leftovers
        w = rng.integers(0, 1 << 32, size=n, dtype=np.uint64).astype(np.uint32)
        t = torch.from_numpy(w.view(np.int32)).cuda()
        ref, got = _both(L, t, n)
        assert got == ref, (n, call)
        assert got == cref.xorsum(w), (n, call)
        del t


def test_noalloc_takes_no_device_memory_once_warm(cref):
    import torch

    L = _abi()
    w = np.arange(1 << 20, dtype=np.uint32) * np.uint32(2654435761)
    t = torch.from_numpy(w.view(np.int32)).cuda()
    out = ctypes.c_uint32(0)
    torch.cuda.synchronize()
    assert L.mmaemu_xorsum_noalloc(t.data_ptr(), w.size, ctypes.byref(out)) == 0  # warm-up
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        assert L.mmaemu_xorsum_noalloc(t.data_ptr(), w.size, ctypes.byref(out)) == 0
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert out.value == cref.xorsum(w)


def test_noalloc_shrinking_sizes_reuse_the_scratch():
    """A large call then a small one: the small call must not pick up the
    large call's partial words."""
    import torch

    L = _abi()
    for n in (5_000_000, 20_000, 4):
        t = torch.randint(-(1 << 31), 1 << 31, (n,), dtype=torch.int32, device="cuda")
        ref, got = _both(L, t, n)
        assert got == ref, n


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import torch

    L = _abi()
    t = torch.zeros(16, dtype=torch.int32, device="cuda")
    out = ctypes.c_uint32(0)
    assert L.mmaemu_xorsum_noalloc(t.data_ptr(), MAX_WORDS + 1, ctypes.byref(out)) == -1  # MMAEMU_EINVAL
    assert L.mmaemu_xorsum_noalloc(t.data_ptr(), 0, ctypes.byref(out)) == 0 and out.value == 0
