"""The plain-C oracle agrees with the Python oracle (CPU only)."""

import itertools
import random

import numpy as np
import pytest

import oracle.mma_model as mm
import pins
from bit_exact_tensor_b200 import workloads as wl

PAIRS = sorted(mm.SUPPORTED)


def py_tiles(model, fmt, A, B, C):
    M, F = mm.MODELS[model], mm.FORMATS[fmt]
    out = np.empty((A.shape[0], 16, 16), dtype=np.uint32)
    for t in range(A.shape[0]):
        out[t] = np.array(mm.mma_tile(M, F, A[t].tolist(), B[t].tolist(), C[t].tolist()), dtype=np.uint32)
    return out


def test_probes_and_golden_in_c(cref):
    for name, model, fmt, a, b, c, want in pins.PROBES:
        A = np.array([a.get(k, 0) for k in range(16)], dtype=wl.in_dtype(fmt))
        B = np.array([b.get(k, 0) for k in range(16)], dtype=wl.in_dtype(fmt))
        assert cref.mma_element(model, fmt, A, B, c) == want, name
    for model, fmt, a, b, c, want, cite in pins.load_golden():
        A = np.array([a.get(k, 0) for k in range(16)], dtype=wl.in_dtype(fmt))
        B = np.array([b.get(k, 0) for k in range(16)], dtype=wl.in_dtype(fmt))
        assert cref.mma_element(model, fmt, A, B, c) == want, cite


def test_random_elements(cref):
    rnd = random.Random(31)
    for model, fmt in PAIRS:
        for _ in range(400):
            A = [pins.random_operand(rnd, fmt) for _ in range(16)]
            B = [pins.random_operand(rnd, fmt) for _ in range(16)]
            c = pins.random_c(rnd)
            want = mm.mma_element(mm.MODELS[model], mm.FORMATS[fmt], A, B, c)
            got = cref.mma_element(model, fmt, np.array(A, dtype=wl.in_dtype(fmt)),
                                   np.array(B, dtype=wl.in_dtype(fmt)), c)
            assert got == want, (model, fmt, A, B, c)


def test_config1_subset(cref):
    A, B, C = wl.config1()
    sel = slice(0, 384)
    np.testing.assert_array_equal(cref.tiles("ampere", "fp16", A[sel], B[sel], C[sel]),
                                  py_tiles("ampere", "fp16", A[sel], B[sel], C[sel]))


@pytest.mark.parametrize("model,fmt", PAIRS)
def test_config2_subsample(cref, model, fmt):
    A, B, C, cls = wl.config2(fmt, ntiles=2000)
    idx = np.concatenate([np.flatnonzero(cls == k)[:12] for k in range(5)])
    Ds = cref.tiles(model, fmt, A[idx], B[idx], C[idx])
    np.testing.assert_array_equal(Ds, py_tiles(model, fmt, A[idx], B[idx], C[idx]))


@pytest.mark.parametrize("model,fmt", PAIRS)
def test_specials_tiles(cref, model, fmt):
    A, B, C = wl.tiles_specials(fmt, ntiles=48)
    np.testing.assert_array_equal(cref.tiles(model, fmt, A, B, C), py_tiles(model, fmt, A, B, C))


def test_gemm_chain_matches_python(cref):
    rnd = np.random.default_rng(12)
    for model, fmt in PAIRS:
        M, N, K = 32, 32, 48
        A = rnd.integers(0, 1 << (8 if fmt == "e4m3" else 16), size=(M, K)).astype(wl.in_dtype(fmt))
        B = rnd.integers(0, 1 << (8 if fmt == "e4m3" else 16), size=(K, N)).astype(wl.in_dtype(fmt))
        # keep most entries finite and moderate so the chain carries values
        fin = wl.to_bits(rnd.standard_normal((M, K)), fmt)
        A = np.where(rnd.random((M, K)) < 0.97, fin, A)
        finb = wl.to_bits(rnd.standard_normal((K, N)), fmt)
        B = np.where(rnd.random((K, N)) < 0.97, finb, B)
        C = wl.f32_bits(rnd.standard_normal((M, N)))
        D = cref.gemm(model, fmt, A, B, C)
        Dp = np.array(mm.gemm(mm.MODELS[model], mm.FORMATS[fmt], A.tolist(), B.tolist(), C.tolist()),
                      dtype=np.uint32)
        np.testing.assert_array_equal(D, Dp)
        assert cref.gemm_element(model, fmt, A, B, C, 7, 19) == D[7, 19]
        fp = cref.tile_fingerprints(D)
        assert fp.tolist() == mm.tile_fingerprints(D.tolist())


def test_gemm_region_and_k_split(cref):
    A, B, C = wl.config3(M=64, N=48, K=96)
    D = cref.gemm("ampere", "fp16", A, B, C)
    part = cref.gemm("ampere", "fp16", A, B, C, rows=(16, 32), cols=(0, 16))
    np.testing.assert_array_equal(part[16:32, 0:16], D[16:32, 0:16])
    assert not part[:16].any() and not part[32:].any()
    D1 = cref.gemm("ampere", "fp16", A[:, :48], B[:48], C)
    D2 = cref.gemm("ampere", "fp16", A[:, 48:], B[48:], D1)
    np.testing.assert_array_equal(D, D2)


def test_neutral_subgroup_exhaustive_search(cref):
    """Algorithm 4 over every subset S of the 17 terms with 2 <= |S| < 17:
    Ampere's only neutral subset is {C, P[1..8]}; Hopper has none."""
    base_a, base_b = {}, {}
    for i in range(1, 17):
        base_a[i - 1], base_b[i - 1] = pins._small(i)
    small_c = pins.f32(1.0 + 2**-20)
    nA = np.zeros((2, 16), dtype=np.uint16)
    found = {"ampere": [], "hopper": []}
    for mask in range(1 << 17):
        S = [i for i in range(17) if mask >> i & 1]
        if len(S) < 2 or len(S) == 17:
            continue
        for variant in (0, 1):  # 0 engineered, 1 zeroed
            a = dict(base_a)
            b = dict(base_b)
            c = small_c
            for i in S:
                val = 0
                if variant == 0 and i == S[0]:
                    val = 1
                elif variant == 0 and i == S[-1]:
                    val = -1
                if i == 0:
                    c = pins.f32(1024.0 * val) if val else 0
                elif val:
                    a[i - 1], b[i - 1] = (pins.X_A if val > 0 else pins.X_A | 0x8000), pins.X_B
                else:
                    a[i - 1], b[i - 1] = 0, 0
            nA[variant] = [a[k] for k in range(16)]
            if variant == 0:
                Bv0 = np.array([b[k] for k in range(16)], dtype=np.uint16)
                c0 = c
            else:
                Bv1 = np.array([b[k] for k in range(16)], dtype=np.uint16)
                c1 = c
        for model in ("ampere", "hopper"):
            if cref.mma_element(model, "fp16", nA[0], Bv0, c0) == cref.mma_element(model, "fp16", nA[1], Bv1, c1):
                found[model].append(mask)
    assert found["ampere"] == [sum(1 << i for i in range(9))]
    assert found["hopper"] == []
