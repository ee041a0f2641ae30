"""Seeded synthetic inputs shaped like the Hawkeye workloads.

This module only draws random numbers and casts them to storage formats; it
contains none of the emulated MMA arithmetic, and is the one piece of code
that both the CUDA path (tests, bench) and the CPU oracle consume.  Every
array holds raw bit patterns: uint16 for fp16/bf16, uint8 for e4m3 and
uint32 for fp32.

The pages measure on 100k random 16x16 tiles and on 4096x4096 MatMuls
("Hawkeye ... (MLSys 2026)" notes, Experiments and results); there is no
public dataset, so these generators stand in for those inputs.  Casts to the
storage formats round to nearest-even (numpy for fp16, torch for bf16 and
e4m3); generation only, both sides consume the same bytes.
"""

from __future__ import annotations

import numpy as np

FORMAT_BITS = {"fp16": (5, 10, 15), "bf16": (8, 7, 127), "e4m3": (4, 3, 7)}
PAIRS = (("ampere", "fp16"), ("ampere", "bf16"), ("hopper", "fp16"), ("hopper", "bf16"),
         ("hopper", "e4m3"), ("b200", "fp16"), ("b200", "bf16"))


def in_dtype(fmt: str):
    return np.uint8 if fmt == "e4m3" else np.uint16


# ---------------------------------------------------------------------------
# casts (round to nearest even) -> raw bits
# ---------------------------------------------------------------------------


def to_bits(x: np.ndarray, fmt: str) -> np.ndarray:
    """Cast float64/float32 values to ``fmt`` (RNE) and return the bit patterns."""
    x = np.asarray(x)
    if fmt == "fp16":
        return x.astype(np.float16).view(np.uint16)
    import torch  # generation-only dependency

    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    if fmt == "bf16":
        return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    if fmt == "e4m3":
        return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy().view(np.uint8)
    raise ValueError(fmt)


def f32_bits(x: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32)).view(np.uint32)


def from_fields(s: np.ndarray, field: np.ndarray, frac: np.ndarray, fmt: str) -> np.ndarray:
    """Assemble bit patterns from sign / exponent-field / fraction arrays."""
    eb, p, _ = FORMAT_BITS[fmt]
    bits = (s.astype(np.uint32) << (eb + p)) | (field.astype(np.uint32) << p) | frac.astype(np.uint32)
    return bits.astype(in_dtype(fmt))


def random_subnormals(rng: np.random.Generator, shape, fmt: str) -> np.ndarray:
    """Field 0, fraction uniform in [1, 2^p - 1], random sign."""
    _, p, _ = FORMAT_BITS[fmt]
    s = rng.integers(0, 2, size=shape)
    frac = rng.integers(1, 1 << p, size=shape)
    return from_fields(s, np.zeros(shape, dtype=np.int64), frac, fmt)


def log_uniform(rng: np.random.Generator, shape, lo: float, hi: float) -> np.ndarray:
    """Random sign, log2|x| uniform in [lo, hi]."""
    mag = np.exp2(rng.uniform(lo, hi, size=shape))
    return np.where(rng.integers(0, 2, size=shape) == 1, -mag, mag)


# ---------------------------------------------------------------------------
# tile batches
# ---------------------------------------------------------------------------


def tiles_random_normal(ntiles: int, fmt: str, seed: int, subnormal_frac: float = 0.1,
                        c_mode: str = "normal"):
    """Random tiles: |x| ~ |N(0,1)| with random sign, a fraction of entries
    replaced by random subnormals; C ~ N(0,1) in fp32 (or zeros).

    Draw order: A, B, C, then the subnormal choices for A and B.
    """
    rng = np.random.default_rng(seed)
    shape = (ntiles, 16, 16)
    A = to_bits(rng.standard_normal(shape), fmt)
    B = to_bits(rng.standard_normal(shape), fmt)
    C = f32_bits(rng.standard_normal(shape)) if c_mode == "normal" else np.zeros(shape, np.uint32)
    for X in (A, B):
        pick = rng.random(shape) < subnormal_frac
        sub = random_subnormals(rng, shape, fmt)
        X[pick] = sub[pick]
    return A, B, C


def config1(seed: int = 0):
    """4,096 Ampere-FP16 tiles: N(0,1) with 10% subnormal entries, C ~ N(0,1)."""
    return tiles_random_normal(4096, "fp16", seed, 0.1)


# Ranges of the "overflowing product" class, per format: log2|x| bounds.
_OVERFLOW_RANGE = {"fp16": (8.0, 15.0), "bf16": (64.0, 127.0), "e4m3": (5.0, float(np.log2(448.0)))}


def config2(fmt: str, ntiles: int = 100_000, seed: int = 1):
    """Random + adversarial tiles for one format.

    Per tile: 50% plain N(0,1); 12.5% each of
      (i)   exponent gaps: product exponents spread by g_k ~ U{0..40};
      (ii)  exact cancellation inside P[1..8] (pairs k, k' < 8 with
            a[m][k'] = -a[m][k], b[k'][n] = b[k][n]), and rows where C
            cancels what is left of the first eight products;
      (iii) subnormal operands on one or both sides;
      (iv)  products overflowing the input format.
    C per element: 50% N(0,1), 25% +0, 25% -0.
    Returns (A, B, C, cls) where cls[t] in 0..4 names the tile's class.
    """
    rng = np.random.default_rng(seed)
    shape = (ntiles, 16, 16)
    eb, p, bias = FORMAT_BITS[fmt]
    cls = np.where(rng.random(ntiles) < 0.5, 0, rng.integers(1, 5, size=ntiles))

    A = np.empty(shape, dtype=np.float64)
    B = np.empty(shape, dtype=np.float64)
    A[:] = rng.standard_normal(shape)
    B[:] = rng.standard_normal(shape)

    # (i) exponent gaps: a[m][k] ~ 2^(Ea - ga_k), b[k][n] ~ 2^(Eb - gb_k)
    # with ga_k + gb_k = g_k ~ U{0..40}; mantissas random in [1, 2).
    t1 = np.flatnonzero(cls == 1)
    if t1.size:
        g = rng.integers(0, 41, size=(t1.size, 16))
        ga = g // 2
        gb = g - ga
        top = {"fp16": 10, "bf16": 20, "e4m3": 6}[fmt]
        ma = 1.0 + rng.random((t1.size, 16, 16))
        mb = 1.0 + rng.random((t1.size, 16, 16))
        sa = np.where(rng.integers(0, 2, size=(t1.size, 16, 16)) == 1, -1.0, 1.0)
        sb = np.where(rng.integers(0, 2, size=(t1.size, 16, 16)) == 1, -1.0, 1.0)
        A[t1] = sa * ma * np.exp2(top - ga[:, None, :])
        B[t1] = sb * mb * np.exp2(top - gb[:, :, None])

    # (iv) overflow: log-uniform magnitudes in the format's top range
    t4 = np.flatnonzero(cls == 4)
    if t4.size:
        lo, hi = _OVERFLOW_RANGE[fmt]
        A[t4] = log_uniform(rng, (t4.size, 16, 16), lo, hi)
        B[t4] = log_uniform(rng, (t4.size, 16, 16), lo, hi)

    if fmt == "e4m3":
        A = np.clip(A, -448.0, 448.0)
        B = np.clip(B, -448.0, 448.0)
    Ab = to_bits(A, fmt)
    Bb = to_bits(B, fmt)

    # (iii) subnormals: one side (A or B) or both, half of the entries
    t3 = np.flatnonzero(cls == 3)
    if t3.size:
        side = rng.integers(0, 3, size=t3.size)  # 0: A, 1: B, 2: both
        sub_a = random_subnormals(rng, (t3.size, 16, 16), fmt)
        sub_b = random_subnormals(rng, (t3.size, 16, 16), fmt)
        pick_a = (rng.random((t3.size, 16, 16)) < 0.5) & (side != 1)[:, None, None]
        pick_b = (rng.random((t3.size, 16, 16)) < 0.5) & (side != 0)[:, None, None]
        Xa, Xb = Ab[t3], Bb[t3]
        Xa[pick_a] = sub_a[pick_a]
        Xb[pick_b] = sub_b[pick_b]
        Ab[t3], Bb[t3] = Xa, Xb

    # C: 50% N(0,1), 25% +0, 25% -0
    C = f32_bits(rng.standard_normal(shape))
    u = rng.random(shape)
    C[(u >= 0.5) & (u < 0.75)] = 0x00000000
    C[u >= 0.75] = 0x80000000

    # (ii) exact cancellation within k < 8: pairs (0,1), (2,3), (4,5) after a
    # random permutation of 0..7; the remaining k6 product is set to -C on
    # some rows (b[k6][n] = 1, a[m][k6] = x, C[m][n] = -x) and k7 to zero.
    t2 = np.flatnonzero(cls == 2)
    if t2.size:
        sign_bit = np.uint16(1 << (eb + p)) if fmt != "e4m3" else np.uint8(0x80)
        one = to_bits(np.ones(1), fmt)[0]
        for t in t2:
            perm = rng.permutation(8)
            for j in range(3):
                k, kk = perm[2 * j], perm[2 * j + 1]
                Ab[t, :, kk] = Ab[t, :, k] ^ sign_bit
                Bb[t, kk, :] = Bb[t, k, :]
            k6, k7 = perm[6], perm[7]
            rows = rng.random(16) < 0.5
            Bb[t, k6, :] = one
            Ab[t, :, k7] = 0
            x = Ab[t, rows, k6]
            xf = from_bits_to_f64(x, fmt)
            C[t, rows, :] = f32_bits(-np.repeat(xf[:, None], 16, axis=1))
    return Ab, Bb, C, cls


def from_bits_to_f64(bits: np.ndarray, fmt: str) -> np.ndarray:
    """Value of raw patterns (finite inputs only) -- used to build exact C
    values in the cancellation class; NaN/Inf patterns map to NaN/Inf."""
    if fmt == "fp16":
        return bits.astype(np.uint16).view(np.float16).astype(np.float64)
    import torch

    t = torch.from_numpy(np.ascontiguousarray(bits))
    if fmt == "bf16":
        return t.view(torch.int16).view(torch.bfloat16).to(torch.float64).numpy()
    return t.view(torch.float8_e4m3fn).to(torch.float64).numpy()


# ---------------------------------------------------------------------------
# GEMMs
# ---------------------------------------------------------------------------


def gemm_normal(M: int, N: int, K: int, fmt: str, seed: int, scale: float = 1.0):
    """A [M,K], B [K,N] ~ N(0,1)*scale (e4m3 saturated to +-448), C zeros."""
    rng = np.random.default_rng(seed)
    A = rng.standard_normal((M, K), dtype=np.float32) * np.float32(scale)
    B = rng.standard_normal((K, N), dtype=np.float32) * np.float32(scale)
    if fmt == "e4m3":
        np.clip(A, -448.0, 448.0, out=A)
        np.clip(B, -448.0, 448.0, out=B)
    return to_bits(A, fmt), to_bits(B, fmt), np.zeros((M, N), dtype=np.uint32)


def gemm_log_uniform(M: int, N: int, K: int, fmt: str, seed: int, lo: float, hi: float):
    """A, B with random sign and log2|x| ~ U[lo, hi]; C zeros."""
    rng = np.random.default_rng(seed)
    A = log_uniform(rng, (M, K), lo, hi)
    B = log_uniform(rng, (K, N), lo, hi)
    return to_bits(A, fmt), to_bits(B, fmt), np.zeros((M, N), dtype=np.uint32)


def config3(seed: int = 3, M: int = 4096, N: int = 4096, K: int = 4096):
    """4096^3 Ampere-FP16 GEMM inputs: A, B fp16 N(0,1), C = +0."""
    return gemm_normal(M, N, K, "fp16", seed)


def config4(seed: int = 4, M: int = 4096, N: int = 4096, K: int = 4096, wide: bool = False):
    """4096^3 Hopper-BF16 GEMM inputs: log2|x| ~ U[-60, 60]; ``wide`` uses
    U[-126, 127] so sums leave the fp32 range (parity-only variant)."""
    lo, hi = (-126.0, 127.0) if wide else (-60.0, 60.0)
    return gemm_log_uniform(M, N, K, "bf16", seed, lo, hi)


def config5(seed: int = 5, M: int = 8192, N: int = 14336, K: int = 4096):
    """LLM-layer GEMM, Hopper E4M3: N(0,1)/sqrt(K), saturated, C = +0."""
    return gemm_normal(M, N, K, "e4m3", seed, scale=1.0 / np.sqrt(K))


def config_batched(batch: int, M: int, N: int, K: int, seed: int = 7, fmt: str = "fp16"):
    """A batch of independent GEMMs (per-expert or per-head MatMuls of a
    model layer): A [batch,M,K], B [batch,K,N] ~ N(0,1), C [batch,M,N] ~
    N(0,1) in fp32."""
    rng = np.random.default_rng(seed)
    A = to_bits(rng.standard_normal((batch, M, K), dtype=np.float32), fmt)
    B = to_bits(rng.standard_normal((batch, K, N), dtype=np.float32), fmt)
    C = f32_bits(rng.standard_normal((batch, M, N), dtype=np.float32))
    return A, B, C


# ---------------------------------------------------------------------------
# special values (parity only)
# ---------------------------------------------------------------------------


def special_patterns(fmt: str) -> np.ndarray:
    """NaN, +-Inf (where the format has them), +-0, max finite, min subnormal."""
    if fmt == "fp16":
        return np.array([0x7E00, 0xFE01, 0x7C00, 0xFC00, 0x0000, 0x8000, 0x7BFF, 0x0001, 0x8001],
                        dtype=np.uint16)
    if fmt == "bf16":
        return np.array([0x7FC0, 0xFF81, 0x7F80, 0xFF80, 0x0000, 0x8000, 0x7F7F, 0x0001, 0x8001],
                        dtype=np.uint16)
    return np.array([0x7F, 0xFF, 0x00, 0x80, 0x7E, 0xFE, 0x01, 0x81], dtype=np.uint8)


def tiles_specials(fmt: str, ntiles: int = 2048, seed: int = 6, rate: float = 0.02):
    """Random tiles with special patterns sprinkled into A, B and C
    (C also gets +-Inf, NaN, +-0 and fp32 subnormals)."""
    A, B, C = tiles_random_normal(ntiles, fmt, seed, 0.05)
    rng = np.random.default_rng(seed + 1000)
    sp = special_patterns(fmt)
    for X in (A, B):
        pick = rng.random(X.shape) < rate
        X[pick] = sp[rng.integers(0, sp.size, size=int(pick.sum()))]
    csp = np.array([0x7F800000, 0xFF800000, 0x7FC00000, 0x00000000, 0x80000000, 0x00000001,
                    0x807FFFFF, 0x7F7FFFFF], dtype=np.uint32)
    pick = rng.random(C.shape) < rate
    C[pick] = csp[rng.integers(0, csp.size, size=int(pick.sum()))]
    return A, B, C
