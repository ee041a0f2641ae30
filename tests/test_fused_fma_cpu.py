"""The identity behind the GEMM's product pass, checked on the host's FMA unit.

The GEMM adds every product of a group with one round-toward-zero fused
multiply-add into a double whose low mantissa bits hold the group sum on the
grid 2^(e_max - F).  ``fused_fma_check.c`` compares that, for random groups in
FP16, BF16 and E4M3 at F = 23, 24 and 25 (zeros, subnormals, the -133 floor),
with exact integer truncation of each product ("Hawkeye: Reproducing
GPU-Level Non-Determinism (MLSys 2026)", Obs. 3), and each planted mistake
must be caught.
"""

import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "fused_fma_check.c")


def run_check(tmp_path, *defines):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    try:
        with open("/proc/cpuinfo") as f:
            if " fma" not in f.read():
                pytest.skip("the host CPU has no FMA instruction")
    except OSError:
        pytest.skip("cannot read the host CPU flags")
    exe = os.path.join(str(tmp_path), "check" + "".join(d.lower() for d in defines))
    cmd = ["gcc", "-O2", "-mfma", "-frounding-math", *[f"-D{d}" for d in defines], SRC, "-o", exe, "-lm"]
    subprocess.run(cmd, check=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout.split()
    return int(out[0]), int(out[1])


def test_fused_round_toward_zero_fma_is_the_truncating_group_sum(tmp_path):
    bad, cases = run_check(tmp_path)
    assert cases == 360_000
    assert bad == 0


@pytest.mark.parametrize("mistake", ["NO_GROWTH", "NO_COUNT", "ROUND_NEAREST"])
def test_each_ingredient_is_needed(tmp_path, mistake):
    bad, cases = run_check(tmp_path, mistake)
    assert bad > cases // 4, (mistake, bad, cases)
