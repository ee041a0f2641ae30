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
