"""Exhaustive check of the oracle on tiny formats.

The oracle is parametric in the storage format and in the accumulation
model, so a toy configuration small enough to enumerate completely exercises
every branch of GroupSum, the stage hand-over and the toward-zero cast
(including overflow to infinity and gradual underflow).  The comparison side
is the exact-rational restatement in ``rational_model.py``.
"""

import itertools
import random

import pytest

import oracle.mma_model as mm
import rational_model as rm

E2M1 = mm.Fmt("e2m1", 2, 1, 1)          # inputs: 0, 0.5, 1, 1.5, 2, 3, Inf, NaN
E2M2 = mm.Fmt("e2m2", 2, 2, 1)          # accumulator input C
E3M2 = mm.Fmt("e3m2", 3, 2, 3)          # output: emin -2, emax 3, subnormal step 2^-4

R_IN = rm.TinyFormat(2, 1, 1)
R_C = rm.TinyFormat(2, 2, 1)
R_OUT = rm.TinyFormat(3, 2, 3)

MODELS = [
    mm.Model("two-stage-floored", 2, ((0,), (1,)), e_floor=1),
    mm.Model("one-stage", 3, ((0, 1),), e_floor=None),
    mm.Model("two-stage", 2, ((0,), (1,)), e_floor=None),
]
MODELS4 = [
    mm.Model("two-stage-4", 2, ((0, 1), (2, 3)), e_floor=None),
    mm.Model("one-stage-4", 4, ((0, 1, 2, 3),), e_floor=0),
]


def _out_table():
    table = {}
    for bits in range(1 << R_OUT.nbits):
        v = R_OUT.value(bits)
        if not isinstance(v, float) and v != 0:
            table[v] = bits
    return table


OUT_BITS = _out_table()


def expected(model, a_bits, b_bits, c_bits):
    av = [R_IN.value(x) for x in a_bits]
    bv = [R_IN.value(x) for x in b_bits]
    cv = R_C.value(c_bits)
    res = rm.dot_reference(av, bv, cv, F=model.F, groups=model.groups, e_floor=model.e_floor,
                           emin_in=R_IN.emin, emin_c=R_C.emin,
                           a_negzero=[R_IN.negative_zero(x) for x in a_bits],
                           b_negzero=[R_IN.negative_zero(x) for x in b_bits],
                           c_negzero=R_C.negative_zero(c_bits))
    if res[0] == "fin":
        res = rm.round_rz(res[1], R_OUT.p, 1 - R_OUT.bias, 6 - R_OUT.bias)
    sign_shift = R_OUT.nbits - 1
    if res[0] == "nan":
        return ((1 << 3) - 1) << 2 | 1 << 1
    if res[0] == "inf":
        return res[1] << sign_shift | ((1 << 3) - 1) << 2
    if res[0] == "zero":
        return res[1] << sign_shift
    return OUT_BITS[res[1]]


FINITE_IN = [b for b in range(16) if not isinstance(R_IN.value(b), float)]
C_SET = [0b00000, 0b10000, 0b00001, 0b00100, 0b10110, 0b01011, 0b11111 & 0b10011, 0b01100, 0b11101]


@pytest.mark.parametrize("model", MODELS, ids=lambda m: m.name)
def test_exhaustive_two_products(model):
    """All finite (a0, b0, a1, b1) with a spread of C values, K = 2."""
    n = 0
    for a0, b0, a1, b1 in itertools.product(FINITE_IN, repeat=4):
        for c in C_SET:
            got = mm.mma_element(model, E2M1, [a0, a1], [b0, b1], c, cfmt=E2M2, out=E3M2)
            want = expected(model, [a0, a1], [b0, b1], c)
            assert got == want, (model.name, (a0, b0, a1, b1, c), got, want)
            n += 1
    assert n == len(FINITE_IN) ** 4 * len(C_SET)


@pytest.mark.parametrize("model", MODELS4, ids=lambda m: m.name)
def test_random_four_products_with_specials(model):
    """K = 4 with grouping (c, p1, p2) + (p3, p4) or one stage; all 16 input
    patterns (Inf and NaN included) and all 32 C patterns, sampled."""
    rnd = random.Random(7)
    for _ in range(20000):
        a = [rnd.randrange(16) for _ in range(4)]
        b = [rnd.randrange(16) for _ in range(4)]
        c = rnd.randrange(32)
        got = mm.mma_element(model, E2M1, a, b, c, cfmt=E2M2, out=E3M2)
        assert got == expected(model, a, b, c), (model.name, a, b, c)
