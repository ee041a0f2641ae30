"""Verify mode (recompute and compare with a claimed D) and fingerprint-only
mode of the GEMM, against the C oracle.

The claimed results are the oracle's D with planted bit changes, so the
expected mismatch count and first index are known exactly.  At full size the
claimed D is the GPU's own stored D (itself checked against the oracle on
samples by test_gpu_gemm), with planted changes.
"""

import numpy as np
import pytest

from bit_exact_tensor_b200 import workloads as wl
from gpu_util import dev_f32, dev_in, host_bits
from test_gpu_gemm import normal_inputs

pytestmark = pytest.mark.gpu

NONE = (1 << 64) - 1


def verify(model, fmt, A, B, C, Dc, fingerprint=True):
    import bit_exact_tensor_b200 as mmaemu

    mism, fp = mmaemu.gemm_verify(model, fmt, dev_in(A), dev_in(B), dev_f32(C) if C is not None else None,
                                  dev_f32(Dc), fingerprint=fingerprint)
    count, first = (int(v) & ((1 << 64) - 1) for v in mism.cpu().tolist())
    return count, first, (host_bits(fp) if fp is not None else None)


def plant(D, rng, n, always=()):
    """Flip one random bit in n random elements (plus the given flat
    indices); returns the changed copy and the sorted flat indices."""
    Dc = D.copy().reshape(-1)
    idx = set(int(i) for i in rng.choice(Dc.size, size=n, replace=False)) | set(always)
    for i in idx:
        Dc[i] ^= np.uint32(1) << np.uint32(rng.integers(0, 32))
    return Dc.reshape(D.shape), sorted(idx)


@pytest.mark.parametrize("model,fmt", wl.PAIRS)
def test_verify_counts_exactly_the_planted_mismatches(cref, model, fmt):
    M, N, K = 80, 272, 64
    A, B, C = normal_inputs(M, N, K, fmt, seed=41)
    want = cref.gemm(model, fmt, A, B, C)
    count, first, fp = verify(model, fmt, A, B, C, want)
    assert (count, first) == (0, NONE)
    assert np.array_equal(fp, cref.tile_fingerprints(want))
    rng = np.random.default_rng(42)
    for n, always in ((1, ()), (7, ()), (0, (0,)), (0, (M * N - 1,)), (200, (M * N - 1,))):
        Dc, idx = plant(want, rng, n, always)
        count, first, fp = verify(model, fmt, A, B, C, Dc)
        assert (count, first) == (len(idx), idx[0])
        assert np.array_equal(fp, cref.tile_fingerprints(want))  # fingerprints of the recomputed D


def test_verify_compares_every_bit(cref):
    """NaN payloads and zero signs count: the comparison is of bit patterns."""
    M, N, K = 32, 32, 32
    A, B, C = normal_inputs(M, N, K, "fp16", seed=43)
    A[0, 0] = 0x7E00  # NaN in row 0 -> row 0 of D is the canonical NaN
    B &= 0x7FFF  # B >= 0 ...
    A[1, :] = 0x8000  # ... so row 1's products are all -0 ...
    C[1, :] = 0x80000000  # ... and with C = -0, D's row 1 is -0
    want = cref.gemm("ampere", "fp16", A, B, C)
    assert (want[0] == 0x7FC00000).all() and (want[1] == 0x80000000).all()
    Dc = want.copy()
    Dc[0, 5] = 0x7FC00001  # another NaN
    Dc[1, 7] = 0x00000000  # +0 for -0
    count, first, _ = verify("ampere", "fp16", A, B, C, Dc, fingerprint=False)
    assert (count, first) == (2, 5)


@pytest.mark.parametrize("model,fmt", [("ampere", "fp16"), ("hopper", "bf16"), ("hopper", "e4m3")])
def test_fingerprint_only_mode(cref, model, fmt):
    import bit_exact_tensor_b200 as mmaemu

    A, B, C = normal_inputs(64, 400, 48, fmt, seed=44)
    D, fp = mmaemu.gemm(model, fmt, dev_in(A), dev_in(B), dev_f32(C), store_d=False)
    assert D is None
    assert np.array_equal(host_bits(fp), cref.tile_fingerprints(cref.gemm(model, fmt, A, B, C)))


def test_verify_full_size_e4m3():
    """The 8192 x 4096 x 14336 E4M3-Hopper workload: the GPU's stored D
    verifies clean; planted changes are found exactly; the fingerprint-only
    and verify-mode fingerprints equal those of the storing run."""
    import torch

    import bit_exact_tensor_b200 as mmaemu

    A, B, C = wl.config5()
    Ad, Bd = dev_in(A), dev_in(B)
    D, fp = mmaemu.gemm("hopper", "e4m3", Ad, Bd, None)
    mism, fp_v = mmaemu.gemm_verify("hopper", "e4m3", Ad, Bd, None, D, fingerprint=True)
    assert mism.cpu().tolist() == [0, mmaemu.NO_MISMATCH]
    assert torch.equal(fp_v, fp)
    _, fp_only = mmaemu.gemm("hopper", "e4m3", Ad, Bd, None, store_d=False)
    assert torch.equal(fp_only, fp)
    M, N = D.shape
    flat = D.view(torch.int32).view(-1)
    picks = sorted({0, M * N - 1, 12345 * 16 + 7, (M // 2) * N + N // 3})
    for i in picks:
        flat[i] ^= 1 << 20
    mism, _ = mmaemu.gemm_verify("hopper", "e4m3", Ad, Bd, None, D)
    assert mism.cpu().tolist() == [len(picks), picks[0]]
    flat[0] ^= 1 << 20
    mism, _ = mmaemu.gemm_verify("hopper", "e4m3", Ad, Bd, None, D)
    assert mism.cpu().tolist() == [len(picks) - 1, picks[1]]


@pytest.mark.parametrize("model,fmt", [("ampere", "fp16"), ("hopper", "bf16"), ("hopper", "e4m3")])
def test_corrupted_input_byte_is_localised_by_the_fingerprints(cref, model, fmt):
    """Fault injection on the host (the silent-data-corruption check the
    fingerprints exist for): one exponent bit of one A element is flipped.
    The recomputed per-tile fingerprints differ from the clean run's in that
    element's row of tiles only, and equal the oracle's for the corrupted
    input; one flipped bit in a host copy of D changes the whole-tensor
    xorsum by exactly that bit."""
    import bit_exact_tensor_b200 as mmaemu

    M, N, K = 96, 160, 64
    A, B, C = normal_inputs(M, N, K, fmt, seed=45)
    D0, fp0 = mmaemu.gemm(model, fmt, dev_in(A), dev_in(B), dev_f32(C))
    fp0 = host_bits(fp0).reshape(M // 16, N // 16)
    m, k = 37, 21
    bad = A.copy()
    bad[m, k] ^= 0x40 if fmt == "e4m3" else 0x2000  # an exponent bit: the element's magnitude changes by 2^8 or more
    _, fp1 = mmaemu.gemm(model, fmt, dev_in(bad), dev_in(B), dev_f32(C))
    fp1 = host_bits(fp1).reshape(M // 16, N // 16)
    assert np.array_equal(fp1.reshape(-1), cref.tile_fingerprints(cref.gemm(model, fmt, bad, B, C)))
    rows = sorted(set(np.argwhere(fp1 != fp0)[:, 0].tolist()))
    assert rows == [m // 16]
    # one bit of D flipped on the host: the tensor's xorsum changes by that bit
    d = host_bits(D0).reshape(-1).copy()
    x0 = int(np.bitwise_xor.reduce(d))
    d[1234] ^= np.uint32(1 << 17)
    assert mmaemu.xorsum(dev_f32(d.reshape(M, N))) == x0 ^ (1 << 17)
