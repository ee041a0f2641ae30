"""The C-ABI library loads, exports what include/mmaemu.h declares and rejects
bad arguments before touching a device (CPU only; no compute calls)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mmaemu.h")


def header_text():
    """All of include/*.h (the C ABI: mmaemu.h and mmaemu_probe.h)."""
    import glob

    return "\n".join(open(h).read() for h in sorted(glob.glob(os.path.join(os.path.dirname(HEADER), "*.h"))))


def declared_functions():
    src = re.sub(r"/\*.*?\*/", "", header_text(), flags=re.S)
    return sorted(set(re.findall(r"\b(mmaemu_[a-z_0-9]+)\s*\(", src)))


def declared_constants():
    consts = {}
    for name, val in re.findall(r"#define\s+(MMAEMU_[A-Z_0-9]+)\s+\(?(-?\d+)\)?", header_text()):
        consts[name] = int(val)
    for body in re.findall(r"enum\s*\{([^}]*)\}", re.sub(r"/\*.*?\*/", "", header_text(), flags=re.S)):
        for name, val in re.findall(r"(MMAEMU_[A-Z_0-9]+)\s*=\s*(-?\d+)", body):
            consts[name] = int(val)
    return consts


@pytest.fixture(scope="module")
def L():
    import bit_exact_tensor_b200 as m
    from bit_exact_tensor_b200 import _build

    _build.build_library()
    return m.lib()


def test_header_declares_the_boundary():
    assert declared_functions() == ["mmaemu_bounds_checking", "mmaemu_device_status", "mmaemu_gemm",
                                    "mmaemu_gemm_host", "mmaemu_gemm_strided_batched", "mmaemu_gemm_verify",
                                    "mmaemu_mma_emulated", "mmaemu_mma_native", "mmaemu_model_describe",
                                    "mmaemu_model_identify", "mmaemu_native_tiles",
                                    "mmaemu_probe_alignment_rounding", "mmaemu_probe_floor", "mmaemu_probe_neutral",
                                    "mmaemu_probe_normalization", "mmaemu_probe_precision", "mmaemu_probe_subnormal",
                                    "mmaemu_probe_writeback_rounding", "mmaemu_selftest_wait_timeout",
                                    "mmaemu_set_stream", "mmaemu_set_workspace_cache", "mmaemu_strerror",
                                    "mmaemu_tiles", "mmaemu_tiles_host", "mmaemu_trim_workspace",
                                    "mmaemu_workspace_reserved",
                                    "mmaemu_xorsum", "mmaemu_xorsum_noalloc"]


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
        assert ctypes.cast(getattr(L, name), ctypes.c_void_p).value
    assert L.mmaemu_bounds_checking() == 0


def test_checking_build_exports_every_declared_symbol(L):
    from bit_exact_tensor_b200 import _build

    C = ctypes.CDLL(_build.LIB_CHECK)
    for name in declared_functions():
        assert hasattr(C, name), name
    C.mmaemu_bounds_checking.restype = ctypes.c_int
    assert C.mmaemu_bounds_checking() == 1


def test_constants_match_python_binding():
    import bit_exact_tensor_b200 as m

    c = declared_constants()
    assert c["MMAEMU_AMPERE"] == m.MODELS["ampere"] and c["MMAEMU_HOPPER"] == m.MODELS["hopper"]
    assert c["MMAEMU_FP16"] == m.FORMATS["fp16"] and c["MMAEMU_BF16"] == m.FORMATS["bf16"]
    assert c["MMAEMU_E4M3"] == m.FORMATS["e4m3"]
    assert (c["MMAEMU_OK"], c["MMAEMU_EINVAL"], c["MMAEMU_ECUDA"], c["MMAEMU_ETIMEOUT"],
            c["MMAEMU_EUNSUPPORTED"], c["MMAEMU_ECALLBACK"], c["MMAEMU_EBOUNDS"]) == (0, -1, -2, -3, -4, -5, -6)
    from bit_exact_tensor_b200 import probe

    for code, name in probe.ROUNDING.items():
        assert c["MMAEMU_ROUND_" + name.upper().replace("-", "_")] == code


def test_strerror_and_set_stream(L):
    for code in (0, -1, -2, -3, -4, -5, -6, 7):
        assert L.mmaemu_strerror(code)
    assert L.mmaemu_set_stream(None) == 0


def test_invalid_arguments_rejected_before_any_device_work(L):
    EINVAL = -1
    buf = ctypes.create_string_buffer(4096 + 16)
    p = (ctypes.addressof(buf) + 15) & ~15
    # bad enums, Ampere x E4M3, bad shapes, NULL and misaligned pointers
    assert L.mmaemu_gemm(3, 0, 16, 16, 16, p, p, None, p, None) == EINVAL
    assert L.mmaemu_gemm(2, 2, 16, 16, 16, p, p, None, p, None) == EINVAL  # B200 x E4M3 is not modelled
    assert L.mmaemu_gemm(0, 3, 16, 16, 16, p, p, None, p, None) == EINVAL
    assert L.mmaemu_gemm(0, 2, 16, 16, 16, p, p, None, p, None) == EINVAL
    assert L.mmaemu_gemm(1, 0, 16, 24, 16, p, p, None, p, None) == EINVAL
    assert L.mmaemu_gemm(1, 0, 0, 16, 16, p, p, None, p, None) == EINVAL
    assert L.mmaemu_gemm(1, 0, 16, 16, -16, p, p, None, p, None) == EINVAL
    assert L.mmaemu_gemm(1, 0, 16, 16, 16, None, p, None, p, None) == EINVAL
    assert L.mmaemu_gemm(1, 0, 16, 16, 16, p + 2, p, None, p, None) == EINVAL
    assert L.mmaemu_gemm(1, 0, 65535 * 64, 16, 16, p, p, None, p, None) == EINVAL  # grid rows
    assert L.mmaemu_gemm(1, 0, 16, 16, 16, p, p, None, None, None) == EINVAL  # nothing to produce
    # verify mode: the claimed D and the mismatch words are required
    assert L.mmaemu_gemm_verify(1, 0, 16, 16, 16, p, p, None, None, None, p) == EINVAL
    assert L.mmaemu_gemm_verify(1, 0, 16, 16, 16, p, p, None, p, None, None) == EINVAL
    assert L.mmaemu_gemm_verify(0, 2, 16, 16, 16, p, p, None, p, None, p) == EINVAL
    assert L.mmaemu_gemm_verify(1, 0, 16, 16, 16, p, p, None, p + 8, None, p) == EINVAL

    def sb(ta=0, tb=0, M=16, N=16, K=16, batch=1, lda=16, sa=0, ldb=16, sbb=0, C=None, ldc=16, sc=0, D=p, ldd=16,
           sd=0, fp=None, sf=0, A=p):
        f = L.mmaemu_gemm_strided_batched
        f.argtypes = [ctypes.c_int] * 8 + [ctypes.c_void_p, ctypes.c_longlong, ctypes.c_longlong] * 4 + [
            ctypes.c_void_p, ctypes.c_longlong]
        return f(1, 0, ta, tb, M, N, K, batch, A, lda, sa, p, ldb, sbb, C, ldc, sc, D, ldd, sd, fp, sf)

    assert sb(ta=2) == EINVAL
    assert sb(tb=-1) == EINVAL
    assert sb(lda=8) == EINVAL                 # lda < K
    assert sb(ta=1, lda=8) == EINVAL           # lda < M
    assert sb(lda=20) == EINVAL                # vector-loaded rows need lda % 8 == 0
    assert sb(sa=4, batch=2, sd=256) == EINVAL  # ... and stride_a % 8 == 0
    assert sb(tb=1, ldb=24 + 4) == EINVAL      # transposed B rows are vector-loaded too
    assert sb(ldd=18) == EINVAL                # ldd % 4
    assert sb(ldd=8) == EINVAL                 # ldd < N
    assert sb(C=p, ldc=16, sc=2, batch=2, sd=256) == EINVAL
    assert sb(batch=0) == EINVAL
    assert sb(batch=65536, sd=256) == EINVAL
    assert sb(sa=-8) == EINVAL
    assert sb(D=None, fp=None) == EINVAL
    assert sb(D=None, fp=p + 2) == EINVAL      # fingerprints are 4-byte aligned
    assert sb(D=None, fp=p, batch=2, sf=0) == EINVAL  # fingerprint regions overlap
    assert sb(A=p + 8) == EINVAL
    assert L.mmaemu_tiles(0, 2, p, p, None, p, 1) == EINVAL
    assert L.mmaemu_tiles(0, 0, p, p, None, None, 1) == EINVAL
    assert L.mmaemu_tiles(0, 0, p, p, p + 4, p, 1) == EINVAL
    assert L.mmaemu_tiles(0, 0, p, p, None, p, 0) == 0  # empty batch is a no-op
    assert L.mmaemu_xorsum(p, 4, None) == EINVAL
    assert L.mmaemu_xorsum(p + 4, 4, ctypes.byref(ctypes.c_uint32())) == EINVAL


def test_product_path_never_imports_the_oracle():
    """The library package must not route through the CPU oracle."""
    pkg = os.path.join(ROOT, "bit_exact_tensor_b200")
    pat = re.compile(r"\b(import|from)\s+oracle\b|liborc|mmaemu_ref|\bcref\b|\borc_[a-z]")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert not pat.search(text), f


class _FakeTensor:
    def __init__(self, device):
        import torch

        self.device = torch.device(device)


def test_binding_refuses_operands_on_different_devices():
    """Every wrapper runs with its operands' device current; operands on two
    devices (or off the GPU) are refused on the host, before any launch."""
    import bit_exact_tensor_b200 as mm

    assert str(mm._device_of(_FakeTensor("cuda:1"), None, _FakeTensor("cuda:1"))) == "cuda:1"
    with pytest.raises(ValueError):
        mm._device_of(_FakeTensor("cuda:0"), _FakeTensor("cuda:1"))
    with pytest.raises(TypeError):
        mm._device_of(_FakeTensor("cpu"))


def test_gemm_host_refuses_bad_output_buffers():
    """gemm_host's caller-owned outputs are checked on the host, before the
    library is called: D must be a contiguous CPU [M, N] tensor of 32-bit
    elements, the fingerprints (M/16)*(N/16) 32-bit integers."""
    import torch

    import bit_exact_tensor_b200 as mm

    M, N, K = 32, 48, 16
    A = torch.zeros((M, K), dtype=torch.int16)
    B = torch.zeros((K, N), dtype=torch.int16)
    good_d = torch.zeros((M, N), dtype=torch.float32)
    for bad in (torch.zeros((M, N + 16), dtype=torch.float32), torch.zeros((M, N), dtype=torch.float64),
                torch.zeros((N, M), dtype=torch.float32).t()):
        with pytest.raises(TypeError, match="out must be"):
            mm.gemm_host("ampere", "fp16", A, B, None, out=bad)
    for bad in (torch.zeros(((M // 16) * (N // 16) + 1,), dtype=torch.int32),
                torch.zeros(((M // 16) * (N // 16),), dtype=torch.float32)):
        with pytest.raises(TypeError, match="fp_out must be"):
            mm.gemm_host("ampere", "fp16", A, B, None, out=good_d, fp_out=bad)


def test_tiles_host_refuses_bad_buffers():
    """tiles_host checks its host tensors before the library is called."""
    import torch

    import bit_exact_tensor_b200 as mm

    A = torch.zeros((3, 16, 16), dtype=torch.int16)
    B = torch.zeros((3, 16, 16), dtype=torch.int16)
    with pytest.raises(ValueError, match="ntiles"):
        mm.tiles_host("ampere", "fp16", A, torch.zeros((2, 16, 16), dtype=torch.int16))
    with pytest.raises(TypeError, match="A has dtype"):
        mm.tiles_host("ampere", "fp16", A.float(), B)
    with pytest.raises(TypeError, match="C must be"):
        mm.tiles_host("ampere", "fp16", A, B, torch.zeros((3, 16, 16), dtype=torch.float64))
    with pytest.raises(TypeError, match="out must be"):
        mm.tiles_host("ampere", "fp16", A, B, None, out=torch.zeros((2, 16, 16), dtype=torch.float32))
