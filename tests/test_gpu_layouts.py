"""Transposed, padded and strided-batched GEMM layouts against the C oracle.

Every case stores the operands in the layout under test on the device and
gives the oracle the same logical matrices as dense row-major copies; the
arithmetic must be identical bit for bit (the layout only changes where
elements are read from and written to).
"""

import numpy as np
import pytest

from bit_exact_tensor_b200 import workloads as wl
from gpu_util import dev_f32, dev_in, first_mismatch, host_bits
from test_gpu_gemm import normal_inputs

pytestmark = pytest.mark.gpu


def stored(x: np.ndarray, trans: bool, pad: int) -> np.ndarray:
    """Storage for logical matrix x ([rows, cols]): x itself or its transpose,
    with pad extra (garbage) elements at the end of every stored row."""
    s = np.ascontiguousarray(x.T if trans else x)
    if pad:
        fill = np.full((s.shape[0], pad), 0x7E if s.dtype == np.uint8 else 0x7E00, dtype=s.dtype)
        s = np.concatenate([s, fill], axis=1)
    return s


def view(t, rows, cols, trans: bool):
    """The logical [rows, cols] view of a device storage tensor."""
    return t[:, :rows].transpose(0, 1) if trans else t[:, :cols]


@pytest.mark.parametrize("model,fmt", wl.PAIRS)
@pytest.mark.parametrize("ta,tb", [(0, 0), (1, 0), (0, 1), (1, 1)])
def test_transposed_and_padded_operands(cref, model, fmt, ta, tb):
    import bit_exact_tensor_b200 as mmaemu

    M, N, K = 80, 144, 48
    A, B, C = normal_inputs(M, N, K, fmt, seed=50 + 2 * ta + tb)
    want = cref.gemm(model, fmt, A, B, C)
    As = dev_in(stored(A, bool(ta), pad=8 if ta else 16))
    Bs = dev_in(stored(B, bool(tb), pad=16 if tb else 8))
    Av = view(As, M, K, bool(ta)) if ta else As[:, :K]
    Bv = view(Bs, K, N, bool(tb)) if tb else Bs[:, :N]
    D, fp = mmaemu.gemm_batched(model, fmt, Av, Bv, dev_f32(C))
    got = host_bits(D[0])
    assert np.array_equal(got, want), first_mismatch(got, want)
    assert np.array_equal(host_bits(fp[0]), cref.tile_fingerprints(want))


@pytest.mark.parametrize("model,fmt", [("ampere", "fp16"), ("hopper", "bf16"), ("hopper", "e4m3")])
def test_strided_batch_with_shared_operand_and_padded_outputs(cref, model, fmt):
    """Three problems: A per entry (transposed storage), one B shared by all
    (stride 0), C and D with padded rows and gaps between entries."""
    import torch

    import bit_exact_tensor_b200 as mmaemu

    batch, M, N, K = 3, 48, 96, 64
    rng = np.random.default_rng(60)
    As, Cs = [], []
    for b in range(batch):
        A, B, C = normal_inputs(M, N, K, fmt, seed=61 + b)
        As.append(A)
        Cs.append(C)
    B = normal_inputs(M, N, K, fmt, seed=70)[1]
    # A: [batch, K, M] storage, viewed as [batch, M, K]
    Ad = dev_in(np.stack([a.T for a in As])).transpose(1, 2)
    Bd = dev_in(B)
    # C and D: rows padded to N + 12, entries 7 rows apart beyond M
    ldc, rows = N + 12, M + 7
    Cbuf = np.full((batch, rows, ldc), 0x7FC00000, dtype=np.uint32)
    for b in range(batch):
        Cbuf[b, :M, :N] = Cs[b]
    Cd = dev_f32(Cbuf)[:, :M, :N]
    Dbuf = torch.full((batch, rows, ldc), 0x12345678, dtype=torch.int32, device="cuda")
    Dd = Dbuf[:, :M, :N]
    _, fp = mmaemu.gemm_batched(model, fmt, Ad, Bd, Cd, out=Dd)
    got_all = host_bits(Dbuf)
    for b in range(batch):
        want = cref.gemm(model, fmt, As[b], B, Cs[b])
        assert np.array_equal(got_all[b, :M, :N], want), (b, first_mismatch(got_all[b, :M, :N], want))
        assert np.array_equal(host_bits(fp[b]), cref.tile_fingerprints(want))
    # nothing outside the logical outputs was written
    pad = got_all.copy()
    pad[:, :M, :N] = 0x12345678
    assert (pad == 0x12345678).all()


def test_batched_fingerprint_only_and_in_place(cref):
    import bit_exact_tensor_b200 as mmaemu

    batch, M, N, K = 2, 32, 64, 32
    data = [normal_inputs(M, N, K, "fp16", seed=80 + b) for b in range(batch)]
    A = dev_in(np.stack([d[0] for d in data]))
    B = dev_in(np.stack([d[1] for d in data]))
    C = dev_f32(np.stack([d[2] for d in data]))
    wants = [cref.gemm("hopper", "fp16", *d) for d in data]
    D, fp = mmaemu.gemm_batched("hopper", "fp16", A, B, C, store_d=False)
    assert D is None
    for b in range(batch):
        assert np.array_equal(host_bits(fp[b]), cref.tile_fingerprints(wants[b]))
    mmaemu.gemm_batched("hopper", "fp16", A, B, C, out=C, fingerprint=False)  # in place
    for b in range(batch):
        assert np.array_equal(host_bits(C[b]), wants[b])
