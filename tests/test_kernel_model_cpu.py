"""The GEMM and tile kernels' arithmetic, restated on the host, against the oracle.

``kernel_model.c`` repeats the CUDA kernels' own steps -- packed exponent
codes, the grid base taken from a packed code, the carried value and every
product added by one round-toward-zero fused multiply-add, the sign-pair
count, the exact group value recovered by one subtraction, 24-bit truncation
by masking, and the scaled ("checked") state with its overflow, underflow,
signed-zero and Inf/NaN paths -- on the host FPU.  Every result must equal the
oracle's bit for bit, in both the unchecked and the checked form, so that the
design is checked on the CPU, independently of a GPU run.  Planted mistakes in
the model must be caught.
"""

import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest

from bit_exact_tensor_b200 import workloads as wl
from gemm_inputs import accumulator_edge_inputs, normal_inputs, special_inputs, worst_case_inputs

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "kernel_model.c")
MODEL = {"ampere": 0, "hopper": 1, "b200": 2}
FMT = {"fp16": 0, "bf16": 1, "e4m3": 2}
_libs = {}


def model_lib(tmp_dir, *defines):
    key = defines
    if key in _libs:
        return _libs[key]
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    with open("/proc/cpuinfo") as f:
        if " fma" not in f.read():
            pytest.skip("the host CPU has no FMA instruction")
    so = os.path.join(str(tmp_dir), "km" + "".join(d.lower() for d in defines) + ".so")
    subprocess.run(["gcc", "-O2", "-mfma", "-frounding-math", "-shared", "-fPIC", *[f"-D{d}" for d in defines],
                    SRC, "-o", so, "-lm"], check=True)
    lib = ctypes.CDLL(so)
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    lib.km_gemm.argtypes = [i32, i32, i32, i32, i32, vp, vp, vp, vp, i32]
    _libs[key] = lib
    return lib


@pytest.fixture(scope="module")
def km(tmp_path_factory):
    return model_lib(tmp_path_factory.mktemp("km"))


def run_model(lib, model, fmt, A, B, C, checked):
    A, B = np.ascontiguousarray(A), np.ascontiguousarray(B)
    M, K = A.shape
    N = B.shape[1]
    D = np.zeros((M, N), dtype=np.uint32)
    Cp = None if C is None else np.ascontiguousarray(C, dtype=np.uint32)
    rc = lib.km_gemm(MODEL[model], FMT[fmt], M, N, K, A.ctypes.data, B.ctypes.data,
                     None if Cp is None else Cp.ctypes.data, D.ctypes.data, int(checked))
    assert rc == 0
    return D


def mismatch(got, want):
    bad = np.argwhere(got != want)
    if bad.size == 0:
        return "equal"
    i = tuple(bad[0])
    return f"{bad.shape[0]} mismatches; first at {i}: got {got[i]:08X} want {want[i]:08X}"


CASES = {
    "normal-80x96x64": lambda fmt: normal_inputs(80, 96, 64, fmt, seed=31),
    "specials": lambda fmt: special_inputs(48, 64, 80, fmt),
    "edges": lambda fmt: accumulator_edge_inputs(fmt, seed=23),
    "worst": lambda fmt: worst_case_inputs(fmt),
    "wide-log-uniform": lambda fmt: (wl.gemm_log_uniform(32, 64, 96, fmt, seed=41, lo=-126.0, hi=127.0)
                                     if fmt == "bf16" else normal_inputs(32, 64, 96, fmt, seed=41)),
}


@pytest.mark.parametrize("checked", [False, True], ids=["unchecked", "checked"])
@pytest.mark.parametrize("case", list(CASES))
@pytest.mark.parametrize("model,fmt", wl.PAIRS)
def test_kernel_design_equals_oracle(cref, km, model, fmt, case, checked):
    A, B, C = CASES[case](fmt)
    want = cref.gemm(model, fmt, A, B, C)
    got = run_model(km, model, fmt, A, B, C, checked)
    assert np.array_equal(got, want), mismatch(got, want)


@pytest.mark.parametrize("model,fmt", wl.PAIRS)
def test_kernel_design_on_tile_classes(cref, km, model, fmt):
    """Tiles of every class of the random + adversarial tile workload (gaps,
    cancellation, subnormals, overflowing products; C with signed zeros),
    each a K = 16 GEMM."""
    A, B, C, cls = wl.config2(fmt, ntiles=400, seed=9)
    for t in range(A.shape[0]):
        want = cref.gemm(model, fmt, A[t], B[t], C[t])
        got = run_model(km, model, fmt, A[t], B[t], C[t], checked=bool(t & 1))
        assert np.array_equal(got, want), (t, int(cls[t]), mismatch(got, want))


@pytest.mark.parametrize("mistake", ["MISTAKE_NO_COUNT", "MISTAKE_NO_SKEW", "MISTAKE_NO_MASK", "MISTAKE_NO_FLOOR",
                                     "MISTAKE_SUBNORMAL_CODE", "MISTAKE_NEAREST_WRITEBACK",
                                     "MISTAKE_HOPPER_UNTRUNCATED"])
def test_planted_mistakes_in_the_design_are_caught(cref, tmp_path, mistake):
    lib = model_lib(tmp_path, mistake)
    caught = False
    for case in CASES:
        for model, fmt in wl.PAIRS:
            A, B, C = CASES[case](fmt)
            for checked in (False, True):
                if not np.array_equal(run_model(lib, model, fmt, A, B, C, checked), cref.gemm(model, fmt, A, B, C)):
                    caught = True
                    break
            if caught:
                break
        if caught:
            break
    assert caught, mistake
