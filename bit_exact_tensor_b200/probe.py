"""Probe API binding (include/mmaemu_probe.h): the characterise half of
characterise-then-simulate.

The target tests and the neutral-subgroup search of "Hawkeye: Reproducing
GPU-Level Non-Determinism (MLSys 2026)" (reading notes: "Target Tests"
table; Algorithm 4) run inside libmmaemu against a tile MMA:

* :func:`emulator` -- this library's emulation of a model (on the GPU);
* :func:`native` -- B200's own tensor cores (``mma.sync``);
* :func:`from_callable` -- any Python function ``f(fmt, A, B, C) -> D`` on
  numpy bit-pattern arrays of shape [ntiles, 16, 16] (A, B uint16 or uint8,
  C and D uint32).  Probes read only the diagonal D[t, i, i].

:func:`characterize` runs them all and returns the recovered model.
Argument marshalling only: the probe logic is the library's.
"""

from __future__ import annotations

import ctypes
from itertools import combinations

import numpy as np

from . import FORMATS, MODELS, MmaEmuError, lib

__all__ = ["Target", "emulator", "native", "from_callable", "precision", "alignment_rounding",
           "writeback_rounding", "normalization", "subnormal_products", "exponent_floor", "neutral_subgroups",
           "all_subsets", "characterize", "describe", "identify", "descriptor", "ROUNDING"]

ROUNDING = {0: "toward-zero", 1: "nearest", 2: "down", 3: "up", 4: "nearest-even", 5: "other", 6: "nearest-away"}
ROUNDING_CODE = {v: k for k, v in ROUNDING.items()}
EUNSUPPORTED = -4
NO_FLOOR, FLOOR_ANY = -100000, 100000


class ModelDesc(ctypes.Structure):
    """mmaemu_model_desc"""
    _fields_ = [("fraction_bits", ctypes.c_int), ("stages", ctypes.c_int), ("stage_products", ctypes.c_int * 4),
                ("e_floor", ctypes.c_int), ("alignment_rounding", ctypes.c_int),
                ("writeback_rounding", ctypes.c_int), ("delayed_normalization", ctypes.c_int),
                ("subnormal_renormalized", ctypes.c_int), ("nan_bits", ctypes.c_uint32)]

MMA_FN = ctypes.CFUNCTYPE(ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                          ctypes.POINTER(ctypes.c_uint32), ctypes.POINTER(ctypes.c_uint32), ctypes.c_size_t)

_configured = False


def _lib():
    global _configured
    L = lib()
    if not _configured:
        vp, i32, ip = ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(ctypes.c_int)
        for name in ("mmaemu_probe_precision", "mmaemu_probe_writeback_rounding"):
            getattr(L, name).argtypes = [i32, MMA_FN, vp, ip]
        for name in ("mmaemu_probe_alignment_rounding", "mmaemu_probe_normalization", "mmaemu_probe_subnormal",
                     "mmaemu_probe_floor"):
            getattr(L, name).argtypes = [i32, MMA_FN, vp, i32, ip]
        L.mmaemu_model_describe.argtypes = [i32, ctypes.POINTER(ModelDesc)]
        L.mmaemu_model_identify.argtypes = [ctypes.POINTER(ModelDesc), ip]
        L.mmaemu_probe_neutral.argtypes = [i32, MMA_FN, vp, ctypes.POINTER(ctypes.c_uint32), ctypes.c_size_t,
                                           ctypes.POINTER(ctypes.c_uint8)]
        L.mmaemu_native_tiles.argtypes = [i32, vp, vp, vp, vp, ctypes.c_size_t]
        for name in ("mmaemu_probe_precision", "mmaemu_probe_writeback_rounding", "mmaemu_probe_alignment_rounding",
                     "mmaemu_probe_normalization", "mmaemu_probe_subnormal", "mmaemu_probe_neutral",
                     "mmaemu_probe_floor", "mmaemu_native_tiles", "mmaemu_model_describe",
                     "mmaemu_model_identify"):
            getattr(L, name).restype = i32
        _configured = True
    return L


class Target:
    """A tile MMA the probes can call: a C function pointer and its context."""

    def __init__(self, fn, ctx, name: str, keep=()):
        self.fn, self.ctx, self.name = fn, ctx, name
        self._keep = keep  # objects the pointers refer to

    def __repr__(self):
        return f"Target({self.name})"


def emulator(model: str) -> Target:
    """The library's emulation of ``model`` ("ampere" or "hopper")."""
    L = _lib()
    ctx = ctypes.c_int(MODELS[model])
    fn = MMA_FN(ctypes.cast(L.mmaemu_mma_emulated, ctypes.c_void_p).value)
    return Target(fn, ctypes.cast(ctypes.pointer(ctx), ctypes.c_void_p), f"emulated {model}", (ctx,))


def native() -> Target:
    """B200's own tensor cores (mma.sync with fp32 accumulation)."""
    L = _lib()
    fn = MMA_FN(ctypes.cast(L.mmaemu_mma_native, ctypes.c_void_p).value)
    return Target(fn, None, "native")


def from_callable(f, name: str = "callable") -> Target:
    """Wrap ``f(fmt, A, B, C) -> D`` (numpy bit-pattern arrays)."""
    fmt_names = {v: k for k, v in FORMATS.items()}

    def cb(_ctx, fmt, A, B, C, D, ntiles):
        try:
            name_ = fmt_names[fmt]
            dt = np.uint8 if name_ == "e4m3" else np.uint16
            nbytes = ntiles * 256 * np.dtype(dt).itemsize
            a = np.frombuffer((ctypes.c_char * nbytes).from_address(A), dtype=dt).reshape(ntiles, 16, 16)
            b = np.frombuffer((ctypes.c_char * nbytes).from_address(B), dtype=dt).reshape(ntiles, 16, 16)
            c = np.ctypeslib.as_array(C, shape=(ntiles, 16, 16))
            d = np.ctypeslib.as_array(D, shape=(ntiles, 16, 16))
            d[...] = np.asarray(f(name_, a.copy(), b.copy(), c.copy()), dtype=np.uint32).reshape(ntiles, 16, 16)
            return 0
        except Exception:  # reported to the probe as a callback failure
            import traceback

            traceback.print_exc()
            return 1

    fn = MMA_FN(cb)
    return Target(fn, None, name, (cb,))


def _check(rc: int, where: str):
    if rc != 0:
        raise MmaEmuError(rc, where)


def precision(target: Target, fmt: str) -> int:
    """Fraction bits F kept below the group's largest exponent (the internal
    significand is F + 1 bits wide)."""
    out = ctypes.c_int()
    _check(_lib().mmaemu_probe_precision(FORMATS[fmt], target.fn, target.ctx, ctypes.byref(out)),
           "mmaemu_probe_precision")
    return out.value


def alignment_rounding(target: Target, fmt: str, fraction_bits: int) -> str:
    out = ctypes.c_int()
    _check(_lib().mmaemu_probe_alignment_rounding(FORMATS[fmt], target.fn, target.ctx, fraction_bits,
                                                  ctypes.byref(out)), "mmaemu_probe_alignment_rounding")
    return ROUNDING[out.value]


def writeback_rounding(target: Target, fmt: str) -> str:
    out = ctypes.c_int()
    _check(_lib().mmaemu_probe_writeback_rounding(FORMATS[fmt], target.fn, target.ctx, ctypes.byref(out)),
           "mmaemu_probe_writeback_rounding")
    return ROUNDING[out.value]


def normalization(target: Target, fmt: str, fraction_bits: int) -> str:
    out = ctypes.c_int()
    _check(_lib().mmaemu_probe_normalization(FORMATS[fmt], target.fn, target.ctx, fraction_bits,
                                             ctypes.byref(out)), "mmaemu_probe_normalization")
    return "delayed" if out.value else "normalized first"


def subnormal_products(target: Target, fmt: str, fraction_bits: int):
    """"renormalized", "not renormalized", or None where the probe cannot be
    built (BF16)."""
    out = ctypes.c_int()
    rc = _lib().mmaemu_probe_subnormal(FORMATS[fmt], target.fn, target.ctx, fraction_bits, ctypes.byref(out))
    if rc == EUNSUPPORTED:
        return None
    _check(rc, "mmaemu_probe_subnormal")
    return "renormalized" if out.value else "not renormalized"


def exponent_floor(target: Target, fmt: str, fraction_bits: int):
    """BF16 only: the floor on each group's max exponent (an int), "none"
    (meaning none at or above F - 158, the bottom of the probed range), or
    None for other formats."""
    out = ctypes.c_int()
    rc = _lib().mmaemu_probe_floor(FORMATS[fmt], target.fn, target.ctx, fraction_bits, ctypes.byref(out))
    if rc == EUNSUPPORTED:
        return None
    _check(rc, "mmaemu_probe_floor")
    return "none" if out.value == NO_FLOOR else out.value


def all_subsets():
    """Every bit mask over {C, P1..P16} with 2 <= |S| <= 16 (131,053)."""
    m = np.arange(1 << 17, dtype=np.uint32)
    sizes = np.bitwise_count(m)
    return m[(sizes >= 2) & (sizes <= 16)]


def neutral_subgroups(target: Target, fmt: str, subsets=None):
    """Algorithm 4: the subsets (as sorted tuples of term indices, 0 = C,
    i = P[i]) whose engineered cancellation is bitwise invisible.  All
    2 <= |S| <= 16 subsets by default (the exhaustive search)."""
    if subsets is None:
        masks = all_subsets()
    else:
        masks = np.array([sum(1 << i for i in s) for s in subsets], dtype=np.uint32)
    flags = np.zeros(masks.size, dtype=np.uint8)
    _check(_lib().mmaemu_probe_neutral(FORMATS[fmt], target.fn, target.ctx,
                                       masks.ctypes.data_as(ctypes.POINTER(ctypes.c_uint32)), masks.size,
                                       flags.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8))), "mmaemu_probe_neutral")
    return [tuple(i for i in range(17) if (int(m) >> i) & 1) for m, f in zip(masks, flags) if f]


def sampled_subsets(n_random: int = 400, seed: int = 0):
    """Contiguous runs from C or from P1 (the candidates for accumulation
    stages) plus random subsets: a fast, non-exhaustive search."""
    out = set()
    for lo in (0, 1):
        for hi in range(lo + 1, 17):
            if 2 <= hi - lo + 1 <= 16:
                out.add(tuple(range(lo, hi + 1)))
    for a, b in combinations(range(17), 2):
        out.add((a, b))
    rng = np.random.default_rng(seed)
    while n_random > 0:
        s = tuple(int(i) for i in np.flatnonzero(rng.random(17) < 0.5))
        if 2 <= len(s) <= 16:
            out.add(s)
            n_random -= 1
    return sorted(out)


def characterize(target: Target, fmt: str, exhaustive: bool = True) -> dict:
    """All target tests on one format; the result reads as a model."""
    F = precision(target, fmt)
    res = {"target": target.name, "format": fmt, "fraction_bits": F, "significand_bits": F + 1,
           "alignment_rounding": alignment_rounding(target, fmt, F),
           "writeback_rounding": writeback_rounding(target, fmt)}
    res["normalization"] = normalization(target, fmt, F) if F >= 23 else None
    res["subnormal_products"] = subnormal_products(target, fmt, F)
    res["e_floor"] = exponent_floor(target, fmt, F) if F >= 23 else None
    neutral = neutral_subgroups(target, fmt, None if exhaustive else sampled_subsets())
    res["neutral_subgroups"] = neutral
    res["neutral_search"] = "exhaustive" if exhaustive else "sampled"
    return res


def _desc_dict(d: ModelDesc) -> dict:
    return {"fraction_bits": d.fraction_bits, "stage_products": [d.stage_products[i] for i in range(d.stages)],
            "e_floor": {NO_FLOOR: "none", FLOOR_ANY: "any"}.get(d.e_floor, d.e_floor),
            "alignment_rounding": ROUNDING[d.alignment_rounding], "writeback_rounding": ROUNDING[d.writeback_rounding],
            "delayed_normalization": bool(d.delayed_normalization),
            "subnormal_renormalized": bool(d.subnormal_renormalized), "nan_bits": d.nan_bits}


def describe(model: str) -> dict:
    """The parameters of a built-in model (mmaemu_model_describe)."""
    d = ModelDesc()
    _check(_lib().mmaemu_model_describe(MODELS[model], ctypes.byref(d)), "mmaemu_model_describe")
    return _desc_dict(d)


def descriptor(r: dict):
    """A descriptor from :func:`characterize` output, or None when the
    neutral subgroups do not read as consecutive stages (every neutral set
    must be a prefix {C, P[1..k]}; each k ends a stage)."""
    ends = []
    for s in r["neutral_subgroups"]:
        if tuple(s) != tuple(range(len(s))):
            return None
        ends.append(len(s) - 1)
    bounds = [0] + sorted(ends) + [16]
    stages = [b - a for a, b in zip(bounds, bounds[1:])]
    if len(stages) > 4 or r["normalization"] is None:
        return None
    floor = r.get("e_floor")
    return {"fraction_bits": r["fraction_bits"], "stage_products": stages,
            "e_floor": "any" if floor is None else floor, "alignment_rounding": r["alignment_rounding"],
            "writeback_rounding": r["writeback_rounding"],
            "delayed_normalization": r["normalization"] == "delayed",
            "subnormal_renormalized": r["subnormal_products"] == "renormalized", "nan_bits": 0}


def identify(desc: dict):
    """The built-in model name with these parameters, or None."""
    d = ModelDesc()
    d.fraction_bits = desc["fraction_bits"]
    d.stages = len(desc["stage_products"])
    for i, n in enumerate(desc["stage_products"][:4]):
        d.stage_products[i] = n
    floor = desc["e_floor"]
    d.e_floor = NO_FLOOR if floor == "none" else FLOOR_ANY if floor == "any" else int(floor)
    for key in ("alignment_rounding", "writeback_rounding"):
        if desc[key] not in ROUNDING_CODE:
            return None
        setattr(d, key, ROUNDING_CODE[desc[key]])
    d.delayed_normalization = int(desc["delayed_normalization"])
    d.subnormal_renormalized = int(desc["subnormal_renormalized"])
    d.nan_bits = desc.get("nan_bits", 0)
    out = ctypes.c_int()
    rc = _lib().mmaemu_model_identify(ctypes.byref(d), ctypes.byref(out))
    if rc == EUNSUPPORTED:
        return None
    _check(rc, "mmaemu_model_identify")
    return {0: "ampere", 1: "hopper", 2: "b200"}[out.value]
