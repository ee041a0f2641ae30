"""The probe API on the GPU: the emulation recovers its own models, and
B200's own tensor cores are characterised with the same target tests.

Page: "Hawkeye: Reproducing GPU-Level Non-Determinism (MLSys 2026)" (reading
notes): "Target Tests" table, Algorithm 4, and the future-work item of
running the same target tests on Blackwell.
"""

import json

import numpy as np
import pytest

from bit_exact_tensor_b200 import workloads as wl
from gpu_util import dev_f32, dev_in, host_bits

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fmt", ["fp16", "bf16", "e4m3"])
def test_native_tiles_layout_is_exact_on_small_integers(fmt):
    """Integer operands in [-3, 3] and integer C: every product and partial
    sum is exact, so B200's MMA must return the exact dot product.  This
    checks the fragment layouts of the native kernel, not its rounding."""
    import torch

    from bit_exact_tensor_b200 import probe

    L = probe._lib()
    rng = np.random.default_rng(7)
    nt = 37
    a = rng.integers(-3, 4, size=(nt, 16, 16)).astype(np.float64)
    b = rng.integers(-3, 4, size=(nt, 16, 16)).astype(np.float64)
    c = rng.integers(-50, 51, size=(nt, 16, 16)).astype(np.float64)
    A, B, C = wl.to_bits(a, fmt), wl.to_bits(b, fmt), wl.f32_bits(c)
    D = torch.empty((nt, 16, 16), dtype=torch.int32, device="cuda")
    Ad, Bd, Cd = dev_in(A), dev_in(B), dev_f32(C)
    assert L.mmaemu_native_tiles({"fp16": 0, "bf16": 1, "e4m3": 2}[fmt], Ad.data_ptr(), Bd.data_ptr(),
                                 Cd.data_ptr(), D.data_ptr(), nt) == 0
    got = host_bits(D).view(np.float32).astype(np.float64)
    want = c + np.einsum("tmk,tkn->tmn", a, b)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("model,fmt", wl.PAIRS)
def test_emulation_recovers_its_models(model, fmt):
    """The target tests, run on this library's own emulation on the GPU,
    recover the models they emulate: the characterise and simulate halves
    agree."""
    from bit_exact_tensor_b200 import probe

    r = probe.characterize(probe.emulator(model), fmt, exhaustive=True)
    assert r["fraction_bits"] == (23 if model == "ampere" else 24)
    assert r["alignment_rounding"] == "toward-zero"
    assert r["writeback_rounding"] == "toward-zero"
    assert r["normalization"] == "delayed"
    assert r["subnormal_products"] == (None if fmt == "bf16" else "not renormalized")
    assert r["neutral_subgroups"] == ([tuple(range(9))] if model == "ampere" else [])


@pytest.mark.parametrize("fmt", ["fp16", "bf16", "e4m3"])
def test_characterize_b200_tensor_cores(fmt):
    """The same target tests on B200's mma.sync (fp32 accumulate).  The
    pages give no expected answer for Blackwell; the test checks that every
    probe produces a definite reading and prints the result."""
    from bit_exact_tensor_b200 import probe

    r = probe.characterize(probe.native(), fmt, exhaustive=True)
    print("B200 native", json.dumps(r, default=list))
    assert 15 <= r["fraction_bits"] <= 27
    assert r["alignment_rounding"] in probe.ROUNDING.values()
    assert r["writeback_rounding"] in probe.ROUNDING.values()
    assert r["normalization"] in (None, "delayed", "normalized first")
    assert isinstance(r["neutral_subgroups"], list)
