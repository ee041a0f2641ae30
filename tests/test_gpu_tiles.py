"""mmaemu_tiles on the GPU against the C oracle, bit for bit."""

import numpy as np
import pytest

from bit_exact_tensor_b200 import workloads as wl
from gpu_util import dev_f32, dev_in, first_mismatch, guarded, guards_intact, host_bits

pytestmark = pytest.mark.gpu


def run_tiles(model, fmt, A, B, C):
    """The tile batch through the binding, D written into a guarded buffer
    whose guard words must survive."""
    import bit_exact_tensor_b200 as mmaemu

    dbuf, D = guarded((A.shape[0], 16, 16))
    mmaemu.tiles(model, fmt, dev_in(A), dev_in(B), dev_f32(C) if C is not None else None, out=D)
    assert guards_intact(dbuf), "D guard words overwritten"
    return host_bits(D)


def test_config1_ampere_fp16_all_4096_tiles(cref):
    A, B, C = wl.config1()
    got = run_tiles("ampere", "fp16", A, B, C)
    want = cref.tiles("ampere", "fp16", A, B, C)
    assert np.array_equal(got, want), first_mismatch(got, want)


@pytest.mark.parametrize("model,fmt", wl.PAIRS)
def test_config2_100k_tiles(cref, model, fmt):
    A, B, C, cls = wl.config2(fmt)
    got = run_tiles(model, fmt, A, B, C)
    want = cref.tiles(model, fmt, A, B, C)
    assert np.array_equal(got, want), first_mismatch(got, want)
    # every adversarial class is present and exercised
    assert set(np.unique(cls)) == {0, 1, 2, 3, 4}


@pytest.mark.parametrize("model,fmt", wl.PAIRS)
def test_special_values(cref, model, fmt):
    A, B, C = wl.tiles_specials(fmt)
    got = run_tiles(model, fmt, A, B, C)
    want = cref.tiles(model, fmt, A, B, C)
    assert np.array_equal(got, want), first_mismatch(got, want)


@pytest.mark.parametrize("ntiles", [1, 3, 8, 9, 77, 1000])
def test_ragged_counts_and_null_c(cref, ntiles):
    A, B, C = wl.tiles_random_normal(ntiles, "bf16", seed=ntiles, subnormal_frac=0.2)
    got = run_tiles("ampere", "bf16", A, B, None)
    want = cref.tiles("ampere", "bf16", A, B, None)
    assert np.array_equal(got, want), first_mismatch(got, want)


def test_in_place_and_empty(cref):
    import bit_exact_tensor_b200 as mmaemu

    A, B, C = wl.tiles_random_normal(40, "fp16", seed=5)
    Ct = dev_f32(C)
    mmaemu.tiles("hopper", "fp16", dev_in(A), dev_in(B), Ct, out=Ct)  # D == C
    assert np.array_equal(host_bits(Ct), cref.tiles("hopper", "fp16", A, B, C))
    empty = mmaemu.tiles("hopper", "fp16", dev_in(A[:0]), dev_in(B[:0]))
    assert empty.shape == (0, 16, 16)


def test_deterministic_repeat():
    A, B, C, _ = wl.config2("e4m3", ntiles=5000, seed=9)
    r1 = run_tiles("hopper", "e4m3", A, B, C)
    r2 = run_tiles("hopper", "e4m3", A, B, C)
    assert np.array_equal(r1, r2)


def test_worst_case_magnitudes(cref):
    """Max-magnitude operands everywhere: the 17-term Hopper group and the
    Ampere stages reach their largest sums (no int32 overflow); with the
    B200 model's 25 fraction bits the sum needs 33 bits."""
    for fmt, top in (("fp16", 0x7BFF), ("bf16", 0x7F7F), ("e4m3", 0x7E)):
        A = np.full((4, 16, 16), top, dtype=wl.in_dtype(fmt))
        B = np.full((4, 16, 16), top, dtype=wl.in_dtype(fmt))
        B[1] |= 0x80 if fmt == "e4m3" else 0x8000
        C = np.full((4, 16, 16), 0x7F7FFFFF, dtype=np.uint32)
        C[2] = 0xFF7FFFFF
        for model in ("ampere", "hopper", "b200"):
            if (model, fmt) not in wl.PAIRS:
                continue
            got = run_tiles(model, fmt, A, B, C)
            assert np.array_equal(got, cref.tiles(model, fmt, A, B, C)), (model, fmt)


@pytest.mark.parametrize("model,fmt", wl.PAIRS)
def test_full_width_group_sums(cref, model, fmt):
    """Sixteen products with the largest significand at one exponent 2e and
    a C of (2 - 2^-23) 2^(2e): every term is on the group's top exponent, so
    the aligned sum is as wide as it gets -- 33 bits with the B200 model's
    25 fraction bits.  Signs vary per tile."""
    import numpy as np

    top = {"fp16": 0x5BFF, "bf16": 0x44FF, "e4m3": 0x5F}[fmt]  # 255.875, 2040, 30
    e2 = {"fp16": 14, "bf16": 20, "e4m3": 8}[fmt]              # exponent of their squares
    sign = 0x80 if fmt == "e4m3" else 0x8000
    rng = np.random.default_rng(13)
    nt = 64
    A = np.full((nt, 16, 16), top, dtype=wl.in_dtype(fmt))
    B = np.full((nt, 16, 16), top, dtype=wl.in_dtype(fmt))
    A[nt // 2:] |= sign  # negative products in half the tiles
    A[rng.random(A.shape) < 0.05] ^= sign
    c = np.float32((2 - 2**-23) * 2.0**e2).view(np.uint32)
    C = np.full((nt, 16, 16), c, dtype=np.uint32)
    C[nt // 4: 3 * nt // 4] |= 0x80000000
    got = run_tiles(model, fmt, A, B, C)
    want = cref.tiles(model, fmt, A, B, C)
    assert np.array_equal(got, want), first_mismatch(got, want)


def _host(x, pinned=True):
    import torch

    v = x.view(np.uint8) if x.dtype == np.uint8 else x.view(np.int16) if x.dtype == np.uint16 else x.view(np.int32)
    t = torch.from_numpy(np.ascontiguousarray(v))
    return t.pin_memory() if pinned else t


@pytest.mark.parametrize("pinned", [True, False])
def test_config2_from_host_memory(cref, pinned):
    """mmaemu_tiles_host, the end-to-end tile call: 100,000 tiles streamed
    in 8 chunks of 12,500 from host memory, the same bits as the oracle."""
    import bit_exact_tensor_b200 as mmaemu

    A, B, C, _ = wl.config2("fp16")
    D = mmaemu.tiles_host("ampere", "fp16", _host(A, pinned), _host(B, pinned), _host(C, pinned))
    got = D.view(-1).numpy().view(np.uint32).reshape(A.shape[0], 16, 16)
    want = cref.tiles("ampere", "fp16", A, B, C)
    assert np.array_equal(got, want), first_mismatch(got, want)


@pytest.mark.parametrize("model,fmt,ntiles", [("hopper", "e4m3", 12305), ("ampere", "bf16", 4097), ("b200", "fp16", 1)])
def test_ragged_chunks_from_host_memory(cref, model, fmt, ntiles):
    """Chunk counts and ragged last chunks (12,305 tiles: three chunks of
    4,102, 4,102 and 4,101; 4,097 tiles: one chunk), C = NULL, and D written
    into a caller-owned buffer."""
    import torch

    import bit_exact_tensor_b200 as mmaemu

    A, B, _ = wl.tiles_random_normal(ntiles, fmt, seed=ntiles, subnormal_frac=0.1)
    out = torch.full((ntiles * 256,), -1, dtype=torch.int32).pin_memory()
    D = mmaemu.tiles_host(model, fmt, _host(A), _host(B), None, out=out)
    assert D is out
    got = out.numpy().view(np.uint32).reshape(ntiles, 16, 16)
    want = cref.tiles(model, fmt, A, B, None)
    assert np.array_equal(got, want), first_mismatch(got, want)


def test_tiles_from_host_memory_empty_and_invalid_pair():
    """An empty batch is a no-op; an invalid model/format pair (Ampere has
    no E4M3) is refused with MMAEMU_EINVAL before anything is copied."""
    import torch

    import bit_exact_tensor_b200 as mmaemu

    empty = torch.zeros((0, 16, 16), dtype=torch.int16)
    assert mmaemu.tiles_host("hopper", "fp16", empty, empty).numel() == 0
    A = torch.zeros((2, 16, 16), dtype=torch.uint8)
    with pytest.raises(mmaemu.MmaEmuError) as err:
        mmaemu.tiles_host("ampere", "e4m3", A, A)
    assert err.value.code == -1
