"""Bounded waits and the device status word.

Every wait in the kernels has a bound; a wait that runs out records a
timeout in the device status word and the kernel winds down instead of
hanging.  The self-test kernel waits on an mbarrier that nothing ever
completes (a flag nobody sets) with a small bound: the wait must give up,
the status word must report it (MMAEMU_ETIMEOUT through mmaemu_device_status),
clearing must reset it, and the device must stay usable afterwards.
"""

import numpy as np
import pytest

from gemm_inputs import normal_inputs
from gpu_util import dev_f32, dev_in, host_bits

pytestmark = pytest.mark.gpu


def test_wait_that_never_completes_is_reported_and_the_device_stays_usable(cref):
    import torch

    import bit_exact_tensor_b200 as mmaemu

    assert mmaemu.device_status(clear=True) in (0, mmaemu.STATUS_TIMEOUT)  # start clean
    assert mmaemu.device_status() == 0
    completed = mmaemu.selftest_wait_timeout(2000)
    assert completed is False
    assert mmaemu.device_status(clear=False) & mmaemu.STATUS_TIMEOUT
    L = mmaemu.lib()
    import ctypes

    bits = ctypes.c_uint32(0)
    assert L.mmaemu_device_status(1, ctypes.byref(bits)) == -3  # MMAEMU_ETIMEOUT, and cleared
    assert bits.value & mmaemu.STATUS_TIMEOUT
    assert mmaemu.device_status() == 0
    # the context still works: a GEMM afterwards is exact and records nothing
    A, B, C = normal_inputs(64, 128, 48, "fp16", seed=2)
    D, _ = mmaemu.gemm("ampere", "fp16", dev_in(A), dev_in(B), dev_f32(C))
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(D), cref.gemm("ampere", "fp16", A, B, C))
    assert mmaemu.device_status() == 0


def test_gemms_record_nothing(cref):
    """Ordinary GEMMs and tile batches leave the status word clear (no
    bounded wait of theirs runs out)."""
    import torch

    import bit_exact_tensor_b200 as mmaemu

    mmaemu.device_status(clear=True)
    A, B, C = normal_inputs(208, 272, 160, "bf16", seed=3)
    D, _ = mmaemu.gemm("hopper", "bf16", dev_in(A), dev_in(B), dev_f32(C))
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(D), cref.gemm("hopper", "bf16", A, B, C))
    assert mmaemu.device_status() == 0
