"""mmaemu_xorsum on the GPU against the oracle's xorsum."""

import numpy as np
import pytest

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n", [1, 3, 4, 5, 255, 1024, 1000003, 33554432 + 7])
def test_xorsum_sizes(cref, n):
    import torch

    import bit_exact_tensor_b200 as mmaemu

    rng = np.random.default_rng(n)
    w = rng.integers(0, 1 << 32, size=n, dtype=np.uint64).astype(np.uint32)
    t = torch.from_numpy(w.view(np.int32)).cuda()
    assert mmaemu.xorsum(t) == cref.xorsum(w)


def test_xorsum_empty():
    import torch

    import bit_exact_tensor_b200 as mmaemu

    assert mmaemu.xorsum(torch.zeros(0, dtype=torch.int32, device="cuda")) == 0
