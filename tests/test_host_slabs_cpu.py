"""The row slabs in which mmaemu_gemm_host streams A, C and D (the library's
csrc/host_slabs.h, compiled here for the host): for every shape and GPU size
tried, the slabs cover the rows in order, start on tile boundaries, the first
holds exactly one wave of GEMM tiles, the last is 1/16 of the row blocks and
the ones between are balanced.  The 4096 x 4096 schedule on 148 SMs is the
one the end-to-end benchmark runs."""

import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "host_slabs_check.cpp")
INC = os.path.join(os.path.dirname(HERE), "bit_exact_tensor_b200", "csrc")


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    if shutil.which("g++") is None:
        pytest.skip("g++ not available")
    exe = str(tmp_path_factory.mktemp("slabs") / "host_slabs_check")
    subprocess.run(["g++", "-O2", "-std=c++17", "-I", INC, SRC, "-o", exe], check=True)
    return exe


def run(checker, *shapes):
    args = [str(v) for shape in shapes for v in shape]
    return subprocess.run([checker, *args], check=True, capture_output=True, text=True).stdout.splitlines()


def test_slab_properties_hold_for_every_shape(checker):
    bad, cases = map(int, run(checker)[0].split())
    assert cases > 100_000
    assert bad == 0


def test_schedules_of_the_benchmarked_and_tested_shapes(checker):
    lines = run(checker, (4096, 4096, 148), (1040, 4096, 148), (1040, 400, 148), (8192, 4096, 148))[1:]
    assert lines[0] == "0 640 1472 2304 3072 3840 4096"  # one wave, four middle slabs, 256 rows
    assert lines[1] == "0 640 768 896 960 1024 1040"  # the GPU test's multi-slab shape
    assert lines[2] == "0 1040"  # fewer tiles than one wave: one slab
    assert lines[3] == "0 640 2432 4224 5952 7680 8192"
