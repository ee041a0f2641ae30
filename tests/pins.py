"""Pins for the Python oracle: facts fixed by the pages or by mathematics.

``run_battery()`` evaluates every pin against ``oracle.mma_model`` (looked up
at call time, so a test can plant a mistake in the oracle and check that some
pin catches it) and returns the list of failures.

Page: "Hawkeye: Reproducing GPU-Level Non-Determinism (MLSys 2026)" (reading
notes).  Each pin names the section it follows.
"""

from __future__ import annotations

import os
import random
from fractions import Fraction

import numpy as np

import oracle.mma_model as mm
import rational_model as rm

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "page_examples.txt")


def h16(x: float) -> int:
    """fp16 bit pattern of an exactly representable value."""
    v = np.float16(x)
    assert float(v) == x, x
    return int(v.view(np.uint16))


def f32(x: float) -> int:
    v = np.float32(x)
    assert float(v) == x, x
    return int(v.view(np.uint32))


def bf16(x: float) -> int:
    b = int(np.float32(x).view(np.uint32))
    assert b & 0xFFFF == 0, x
    return b >> 16


def elem(model: str, fmt: str, a: dict, b: dict, c: int) -> int:
    """One element through the oracle; a, b map k -> pattern (others +0)."""
    A = [a.get(k, 0) for k in range(16)]
    B = [b.get(k, 0) for k in range(16)]
    return mm.mma_element(getattr(mm, model.upper()), mm.FORMATS[fmt], A, B, c)


def load_golden():
    cases = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        head, a, b, c, d, cite = [x.strip() for x in line.split("|")]
        model, fmt = head.split()
        av = {k: int(x, 16) for k, x in enumerate(a.split())}
        bv = {k: int(x, 16) for k, x in enumerate(b.split())}
        cases.append((model, fmt, av, bv, int(c, 16), int(d, 16), cite))
    return cases


# ---------------------------------------------------------------------------
# closed-form probes (target-test table; Obs. 3)
# ---------------------------------------------------------------------------

# Each probe: (name, model, fmt, a, b, c, expected, derivation)
PROBES = [
    # Internal Precision Detection: C = 1, P1 = P2 = 2^-24.  Ampere keeps
    # 23 fraction bits below 2^0, so 2^-24 truncates away: 1.0.  Hopper keeps
    # 24, so each adds one unit: 1 + 2^-23.
    ("precision", "ampere", "fp16", {0: h16(2**-12), 1: h16(2**-12)}, {0: h16(2**-12), 1: h16(2**-12)},
     f32(1.0), 0x3F800000),
    ("precision", "hopper", "fp16", {0: h16(2**-12), 1: h16(2**-12)}, {0: h16(2**-12), 1: h16(2**-12)},
     f32(1.0), 0x3F800001),
    # Rounding Mode Detection: C = 1, P1 = -2^-24.  Truncating the magnitude
    # drops the term on Ampere (a floor shift would give 1 - 2^-23,
    # 0x3F7FFFFF); on Hopper the term is exactly one unit: 1 - 2^-24.
    ("align-rz", "ampere", "fp16", {0: h16(-2**-12)}, {0: h16(2**-12)}, f32(1.0), 0x3F800000),
    ("align-rz", "hopper", "fp16", {0: h16(-2**-12)}, {0: h16(2**-12)}, f32(1.0), 0x3F7FFFFF),
    # Toward-zero write-back: C = 2 - 2^-23, P1 = 1.5 -> exact 3.5 - 2^-23,
    # truncated to the fp32 grid at [2,4): 3.5 - 2^-22 (RNE would give 3.5).
    ("writeback-rz", "ampere", "fp16", {0: h16(1.5)}, {0: h16(1.0)}, 0x3FFFFFFF, 0x405FFFFF),
    ("writeback-rz", "hopper", "fp16", {0: h16(1.5)}, {0: h16(1.0)}, 0x3FFFFFFF, 0x405FFFFF),
    # Normalization Stage Detection (Ampere): C = 1 + 2^-23, P1 = 1.5 * -1.5
    # = -2.25 kept at exponent 0, so C is not shifted: -(1.25 - 2^-23).
    # Normalising the product first (to 1.125 * 2^1) would drop C's last bit:
    # -1.25 = 0xBFA00000.
    ("delayed-norm", "ampere", "fp16", {0: h16(1.5)}, {0: h16(-1.5)}, 0x3F800001, 0xBF9FFFFF),
    # Subnormal Behavior Detection: P1 = 2^-24 (fp16 subnormal 0x0001) x 1
    # stays at exponent -14 with significand 1; P2 = (2^-10 (1 + 2^-10))^2.
    # The max exponent is -14, P2 is shifted by 6: 2^-20 + 2^-24 + 2^-29.
    # Renormalising P1 (to exponent -24) would keep P2 whole: 0x35884008.
    ("subnormal", "ampere", "fp16", {0: 0x0001, 1: 0x1401}, {0: h16(1.0), 1: 0x1401}, 0, 0x35884000),
    ("subnormal", "hopper", "fp16", {0: 0x0001, 1: 0x1401}, {0: h16(1.0), 1: 0x1401}, 0, 0x35884000),
    # Signed zeros (reading: an IEEE toward-zero sum of zeros is -0 only when
    # every addend is -0; exact cancellation gives +0).
    ("zero-sign", "ampere", "fp16", {k: 0x8000 for k in range(16)}, {}, 0x80000000, 0x80000000),
    ("zero-sign", "hopper", "bf16", {k: 0x8000 for k in range(16)}, {}, 0x80000000, 0x80000000),
    ("zero-sign", "ampere", "fp16", {k: 0x8000 for k in range(16)}, {}, 0x00000000, 0x00000000),
    ("zero-sign", "ampere", "fp16", {k: 0x8000 for k in range(15)}, {}, 0x80000000, 0x00000000),
    ("zero-sign", "hopper", "fp16", {0: h16(2.0)}, {0: h16(-1.0)}, f32(2.0), 0x00000000),
    # One product entering each position of the second stage is exact.
    ("stage2-exact", "ampere", "fp16", {9: h16(3.0)}, {9: h16(-0.5)}, 0, f32(-1.5)),
    # FP8 E4M3 (Hopper): 448 * 448 + 448 * 448 = 401408 exactly (e4m3 0x7E).
    ("e4m3-exact", "hopper", "e4m3", {0: 0x7E, 15: 0x7E}, {0: 0x7E, 15: 0x7E}, 0, f32(401408.0)),
    # NaN and infinity handling (reading): NaN operand -> canonical NaN;
    # Inf x 0 -> NaN; +Inf + -Inf -> NaN; C = -Inf + finite -> -Inf.
    ("nan", "hopper", "fp16", {3: 0x7E00}, {3: h16(1.0)}, 0, 0x7FC00000),
    ("inf*0", "ampere", "fp16", {3: 0x7C00}, {3: 0x0000}, 0, 0x7FC00000),
    ("inf-inf", "ampere", "bf16", {1: 0x7F80, 12: 0x7F80}, {1: 0x3F80, 12: 0xBF80}, 0, 0x7FC00000),
    ("c=-inf", "hopper", "bf16", {1: 0x3F80}, {1: 0x3F80}, 0xFF800000, 0xFF800000),
    ("e4m3-nan", "hopper", "e4m3", {5: 0x7F}, {5: 0x38}, 0, 0x7FC00000),
]


def probe_failures():
    out = []
    for name, model, fmt, a, b, c, want in PROBES:
        got = elem(model, fmt, a, b, c)
        if got != want:
            out.append(f"probe {name} {model}/{fmt}: got {got:08X} want {want:08X}")
    return out


def golden_failures():
    out = []
    for model, fmt, a, b, c, want, cite in load_golden():
        got = elem(model, fmt, a, b, c)
        if got != want:
            out.append(f"golden [{cite}] {model}/{fmt}: got {got:08X} want {want:08X}")
    return out


# ---------------------------------------------------------------------------
# Algorithm 4: computationally neutral subgroups
# ---------------------------------------------------------------------------

X_A, X_B = h16(32.0), h16(32.0)  # +-1024 = +-X


def _small(i: int):
    """A distinct small product for term i (1 <= i <= 16), with bits down to
    2^-20 so that alignment against X = 1024 visibly truncates it."""
    return h16(1.0 + i * 2**-10), h16(1.0 + 2**-10)


def neutral_tile(model: str, S: frozenset, zeroed: bool) -> int:
    """Term 0 is C, term i (1..16) is P[i] (k = i - 1).  Terms outside S get
    distinct small values.  Inside S either all zero (``zeroed``) or
    engineered to sum to zero: +X on the first element, -X on the last."""
    order = sorted(S)
    a, b, c = {}, {}, f32(1.0 + 2**-20)
    for i in range(17):
        if i in S:
            if zeroed:
                val = None
            elif i == order[0]:
                val = +1
            elif i == order[-1]:
                val = -1
            else:
                val = None
            if i == 0:
                c = 0 if val is None else f32(1024.0 * val)
            elif val is not None:
                a[i - 1], b[i - 1] = (X_A if val > 0 else X_A | 0x8000), X_B
        elif i > 0:
            a[i - 1], b[i - 1] = _small(i)
    return elem(model, "fp16", a, b, c)


def is_neutral(model: str, S) -> bool:
    S = frozenset(S)
    return neutral_tile(model, S, False) == neutral_tile(model, S, True)


AMPERE_STAGE1 = frozenset(range(0, 9))  # {C, P[1..8]}


def neutral_failures():
    """Obs. 2: for Ampere FP16 only {accumulator, P[1..8]} is a nontrivial
    neutral subgroup; for Hopper (one 17-term stage) there is none.  The full
    exhaustive search over all subsets runs against the C oracle in the test
    suite; here a fixed spread of subsets is checked."""
    out = []
    rnd = random.Random(4)
    subsets = [AMPERE_STAGE1, frozenset(range(1, 9)), frozenset(range(0, 8)), frozenset(range(9, 17)),
               frozenset(range(0, 10)), frozenset({0, 1}), frozenset({8, 9}), frozenset({1, 16}),
               frozenset(range(1, 17)), frozenset({0, 16})]
    while len(subsets) < 40:
        s = frozenset(i for i in range(17) if rnd.random() < 0.5)
        if 2 <= len(s) < 17:
            subsets.append(s)
    for S in subsets:
        for model in ("ampere", "hopper"):
            want = model == "ampere" and S == AMPERE_STAGE1
            if is_neutral(model, S) != want:
                out.append(f"neutral {model} {sorted(S)}: expected neutral={want}")
    return out


# ---------------------------------------------------------------------------
# BF16 minimum contribution (recovered pipeline, BF16 paragraph)
# ---------------------------------------------------------------------------


def floor_case():
    """Fifteen products of 1.9921875 * 2^-78 times 1.9921875 * 2^-77 (each
    7.9377 units of 2^-156) and one of 1.375 * 2^-76 * 2^-76 (22 units).
    Every group max exponent is below the -133 threshold, so the grid is
    2^-156 (Ampere, F = 23) or 2^-157 (Hopper).  Ampere: the eight
    stage-1 terms truncate to 7 units each (56), the stage-2 sum is
    56 + 7*7 + 22 = 127 units < 128 = 2^-149, so the result is +0.  Hopper:
    15 * 15 + 44 = 269 half-units = 134.5 units >= 128: the smallest fp32
    subnormal, 0x00000001.  Without the threshold, Ampere would keep the
    fractions and reach 2^-149 too."""
    a = {k: bf16(1.9921875 * 2**-78) for k in range(15)}
    b = {k: bf16(1.9921875 * 2**-77) for k in range(15)}
    a[15], b[15] = bf16(1.375 * 2**-76), bf16(2**-76)
    return a, b


def floor_failures():
    a, b = floor_case()
    out = []
    for model, want in (("ampere", 0x00000000), ("hopper", 0x00000001)):
        got = elem(model, "bf16", a, b, 0)
        if got != want:
            out.append(f"floor -133 {model}: got {got:08X} want {want:08X}")
    # One unit of 2^-156 is the smallest contribution: 127 units (1.984375 *
    # 2^-75 * 2^-75) plus one product of exactly 2^-156 (2^-78 * 2^-78) make
    # 128 units = 2^-149, the smallest fp32 subnormal, in both models.
    a2 = {0: bf16(1.984375 * 2**-75), 1: bf16(2**-78)}
    b2 = {0: bf16(2**-75), 1: bf16(2**-78)}
    for model in ("ampere", "hopper"):
        got = elem(model, "bf16", a2, b2, 0)
        if got != 0x00000001:
            out.append(f"2^-156 unit {model}: got {got:08X} want 00000001")
    return out


# ---------------------------------------------------------------------------
# random elements against the independent rational restatement
# ---------------------------------------------------------------------------

_FMT_EMIN = {"fp16": -14, "bf16": -126, "e4m3": -6}


def rational_expect(model: str, fmt: str, A, B, c) -> int:
    M = getattr(mm, model.upper())
    av = [rm.real_format_value(x, fmt) for x in A]
    bv = [rm.real_format_value(x, fmt) for x in B]
    cv = rm.real_format_value(c, "fp32")
    sign_bit = 0x80 if fmt == "e4m3" else 0x8000
    res = rm.dot_reference(av, bv, cv, F=M.F, groups=M.groups, e_floor=M.e_floor,
                           emin_in=_FMT_EMIN[fmt], emin_c=-126,
                           a_negzero=[x == sign_bit for x in A], b_negzero=[x == sign_bit for x in B],
                           c_negzero=c == 0x80000000)
    if res[0] == "nan":
        return M.nan  # the model's NaN pattern (0x7FC00000 for both models on the pages)
    if res[0] == "fin":
        res = rm.round_rz(res[1], 23, -126, 127)
    return rm.encode_fp32(res)


def random_operand(rnd: random.Random, fmt: str) -> int:
    """A random pattern biased toward interesting cases."""
    nb = 8 if fmt == "e4m3" else 16
    r = rnd.random()
    if r < 0.1:
        return 0 if rnd.random() < 0.5 else 1 << (nb - 1)
    if r < 0.2:  # subnormal
        p = {"fp16": 10, "bf16": 7, "e4m3": 3}[fmt]
        return (rnd.getrandbits(1) << (nb - 1)) | rnd.randrange(1, 1 << p)
    if r < 0.25:
        return rnd.getrandbits(nb)  # anything, specials included
    # moderate magnitudes so that terms interact
    x = rnd.choice((-1, 1)) * (1 + rnd.random()) * 2.0 ** rnd.randint(-6, 6)
    if fmt == "fp16":
        return int(np.float16(x).view(np.uint16))
    if fmt == "bf16":
        return int(np.float32(x).view(np.uint32)) >> 16
    import torch

    return int(torch.tensor([x], dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)[0])


def random_c(rnd: random.Random) -> int:
    r = rnd.random()
    if r < 0.1:
        return rnd.choice((0, 0x80000000))
    if r < 0.15:
        return rnd.getrandbits(32)
    if r < 0.2:
        return rnd.randrange(1, 1 << 23) | (rnd.getrandbits(1) << 31)
    return int(np.float32(rnd.choice((-1, 1)) * (1 + rnd.random()) * 2.0 ** rnd.randint(-8, 8)).view(np.uint32))


def rational_failures(n_per_pair: int = 60, seed: int = 11):
    rnd = random.Random(seed)
    out = []
    for model, fmt in sorted(mm.SUPPORTED):
        for _ in range(n_per_pair):
            A = [random_operand(rnd, fmt) for _ in range(16)]
            B = [random_operand(rnd, fmt) for _ in range(16)]
            c = random_c(rnd)
            want = rational_expect(model, fmt, A, B, c)
            got = mm.mma_element(getattr(mm, model.upper()), mm.FORMATS[fmt], A, B, c)
            if got != want:
                out.append(f"rational {model}/{fmt}: got {got:08X} want {want:08X} A={A} B={B} c={c:08X}")
                break
    return out


# ---------------------------------------------------------------------------
# tile indexing: D[m][n] = C[m][n] + sum_k A[m][k] B[k][n]
# ---------------------------------------------------------------------------


def tile_failures():
    """A tile whose every element has a distinct closed form: A[m][k] = 1
    only at k = m, B[k][n] = (n + 1) * 2^k ... small integers, exact."""
    out = []
    one = h16(1.0)
    A = [[0] * 16 for _ in range(16)]
    B = [[0] * 16 for _ in range(16)]
    C = [[0] * 16 for _ in range(16)]
    for m in range(16):
        A[m][(m * 5) % 16] = one  # row m selects k = 5m mod 16
        for n in range(16):
            C[m][n] = f32(float(m * 16 + n))
    for k in range(16):
        for n in range(16):
            B[k][n] = h16(float(1000 + 16 * k + n))
    for model in (mm.AMPERE, mm.HOPPER):
        D = mm.mma_tile(model, mm.FP16, A, B, C)
        for m in range(16):
            for n in range(16):
                k = (m * 5) % 16
                want = f32(float(m * 16 + n + 1000 + 16 * k + n))
                if D[m][n] != want:
                    out.append(f"tile index {model.name} ({m},{n}): got {D[m][n]:08X} want {want:08X}")
                    return out
    return out


def run_battery(rational_n: int = 60):
    return (golden_failures() + probe_failures() + neutral_failures() + floor_failures()
            + tile_failures() + rational_failures(rational_n))
