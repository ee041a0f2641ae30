"""An independent restatement of the MMA model in exact rationals.

Used only by the tests to pin the integer oracle.  It does not reuse any
oracle code: values come from the IEEE definition (or numpy/torch casts for
the real formats), exponents from floor(log2|x|), and each aligned term from
trunc(x / 2^(e_max - F)) in ``fractions.Fraction`` arithmetic.  Special
values follow IEEE float semantics (Python floats), which is what the
oracle's reading of NaN/Inf handling amounts to.
"""

from __future__ import annotations

import math
from fractions import Fraction

import numpy as np

INF = float("inf")
NAN = float("nan")


def flog2(q: Fraction) -> int:
    """floor(log2 |q|) for q != 0."""
    n, d = abs(q.numerator), q.denominator
    k = n.bit_length() - d.bit_length()
    if k >= 0:
        if n < (d << k):
            k -= 1
    elif (n << -k) < d:
        k -= 1
    return k


def trunc(q: Fraction) -> int:
    """Round toward zero."""
    n, d = q.numerator, q.denominator
    return n // d if n >= 0 else -((-n) // d)


class TinyFormat:
    """A format given by its field widths; values from the IEEE definition."""

    def __init__(self, ebits, p, bias, ieee=True):
        self.ebits, self.p, self.bias, self.ieee = ebits, p, bias, ieee
        self.nbits = 1 + ebits + p

    def value(self, bits: int):
        neg = (bits >> (self.ebits + self.p)) & 1
        E = (bits >> self.p) & ((1 << self.ebits) - 1)
        f = bits & ((1 << self.p) - 1)
        top = (1 << self.ebits) - 1
        if self.ieee and E == top:
            if f:
                return NAN
            return -INF if neg else INF
        if not self.ieee and E == top and f == (1 << self.p) - 1:
            return NAN
        if E == 0:
            v = Fraction(f, 1 << self.p) * Fraction(2) ** (1 - self.bias)
        else:
            v = (1 + Fraction(f, 1 << self.p)) * Fraction(2) ** (E - self.bias)
        return -v if neg else v

    def negative_zero(self, bits):
        return bits == 1 << (self.nbits - 1)

    @property
    def emin(self):
        return 1 - self.bias


def real_format_value(bits: int, fmt: str):
    """Value of a real-format pattern via numpy / torch (not via the oracle)."""
    if fmt == "fp32":
        x = float(np.array([bits], dtype=np.uint32).view(np.float32)[0])
    elif fmt == "fp16":
        x = float(np.array([bits], dtype=np.uint16).view(np.float16)[0])
    else:
        import torch

        if fmt == "bf16":
            x = float(torch.tensor([bits], dtype=torch.int32).to(torch.int16).view(torch.bfloat16)[0])
        else:
            x = float(torch.tensor([bits], dtype=torch.uint8).view(torch.float8_e4m3fn)[0])
    if math.isnan(x) or math.isinf(x):
        return x
    return Fraction(x)


REAL_EMIN = {"fp16": -14, "bf16": -126, "e4m3": -6, "fp32": -126}


def is_neg_zero_value(v) -> bool:
    return isinstance(v, float) and v == 0.0 and math.copysign(1.0, v) < 0


def dot_reference(a_vals, b_vals, c_val, *, F, groups, e_floor, emin_in, emin_c,
                  a_negzero, b_negzero, c_negzero):
    """Exact-rational model of one output.  Returns ('nan',), ('inf', sign),
    ('zero', sign) or ('fin', value: Fraction)."""
    K = len(a_vals)
    # specials with IEEE float semantics
    if any(isinstance(v, float) and math.isnan(v) for v in list(a_vals) + list(b_vals) + [c_val]):
        return ("nan",)
    special = any(isinstance(v, float) for v in list(a_vals) + list(b_vals) + [c_val])
    if special:
        acc = float(c_val) if isinstance(c_val, float) else 0.0
        infs = []
        if isinstance(c_val, float):
            infs.append(c_val)
        for a, b in zip(a_vals, b_vals):
            if isinstance(a, float) or isinstance(b, float):
                pr = float(a) * float(b)
                if math.isnan(pr):
                    return ("nan",)
                infs.append(pr)
        acc = sum(infs)
        if math.isnan(acc):
            return ("nan",)
        return ("inf", 1 if acc < 0 else 0)

    def ex(v, emin):
        return max(flog2(v), emin)

    prods = []
    for a, b in zip(a_vals, b_vals):
        if a == 0 or b == 0:
            prods.append(None)
        else:
            prods.append((a * b, ex(a, emin_in) + ex(b, emin_in)))
    carry = None if c_val == 0 else (c_val, ex(c_val, emin_c))
    total = None
    for gi, idx in enumerate(groups):
        items = ([carry] if carry is not None else []) + [prods[k] for k in idx if prods[k] is not None]
        if not items:
            total = None
            carry = None
            continue
        e_max = max(e for _, e in items)
        if e_floor is not None:
            e_max = max(e_max, e_floor)
        grid = Fraction(2) ** (e_max - F)
        S = sum(trunc(v / grid) for v, _ in items)
        total = S * grid
        if gi + 1 < len(groups):
            if S == 0:
                carry = None
            else:
                E1 = flog2(total)
                unit = Fraction(2) ** (E1 - F)
                carry = (trunc(total / unit) * unit, E1)
    if total is None or total == 0:
        all_negz = c_negzero and all(
            (a == 0 or b == 0) and ((an if a == 0 else (a < 0)) ^ (bn if b == 0 else (b < 0)))
            for a, b, an, bn in zip(a_vals, b_vals, a_negzero, b_negzero))
        return ("zero", 1 if all_negz else 0)
    return ("fin", total)


def round_rz(v: Fraction, p: int, emin: int, emax: int):
    """Round a nonzero rational toward zero onto a binary format with p
    fraction bits.  Returns ('inf', s), ('zero', s) or ('fin', value)."""
    s = 1 if v < 0 else 0
    E = flog2(v)
    if E > emax:
        return ("inf", s)
    unit = Fraction(2) ** ((E if E >= emin else emin) - p)
    q = trunc(v / unit) * unit
    if q == 0:
        return ("zero", s)
    return ("fin", q)


def encode_fp32(res) -> int:
    kind = res[0]
    if kind == "nan":
        return 0x7FC00000
    if kind == "inf":
        return (res[1] << 31) | 0x7F800000
    if kind == "zero":
        return res[1] << 31
    return int(np.array([float(res[1])], dtype=np.float32).view(np.uint32)[0])
