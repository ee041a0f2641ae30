"""bench.py's check of the timed result against the stored oracle digests,
on the CPU: the oracle's own D for the 4,096-tile workload passes, and a D
with one flipped bit (planted in the oracle's output, on the host) is
rejected.  So a timed run can only report ``verified: true`` for a result
equal to the oracle's element by element."""

import sys

import numpy as np
import pytest

from bit_exact_tensor_b200 import workloads as wl


@pytest.fixture(scope="module")
def bench_mod():
    saved = sys.argv
    sys.argv = ["bench.py"]
    try:
        import bench
    finally:
        sys.argv = saved
    return bench


@pytest.fixture(scope="module")
def oracle_d(cref):
    A, B, C = wl.config1()
    return np.ascontiguousarray(cref.tiles("ampere", "fp16", A, B, C), dtype=np.uint32)


def test_oracle_result_verifies(bench_mod, oracle_d):
    rec = bench_mod.verify_against_oracle("tiles-ampere-fp16-4096", oracle_d.view(np.float32), None)
    assert rec["verified"] is True and rec["d_sha256_equal"] is True


def test_one_flipped_bit_is_rejected(bench_mod, oracle_d):
    bad = oracle_d.copy()
    bad.reshape(-1)[12345] ^= 1
    with pytest.raises(RuntimeError, match="differs from the oracle"):
        bench_mod.verify_against_oracle("tiles-ampere-fp16-4096", bad.view(np.float32), None)


def test_unknown_workload_is_not_claimed_verified(bench_mod, oracle_d):
    rec = bench_mod.verify_against_oracle("no-such-workload", oracle_d.view(np.float32), None)
    assert rec["verified"] is None


def test_every_benchmark_workload_has_stored_oracle_digests(bench_mod):
    """Each workload bench.py can time (its modes -fponly, -verify and -wt
    share their base workload's result) maps to a record of oracle digests,
    so no timed result goes unchecked."""
    import json

    with open(bench_mod.GOLDEN) as fh:
        golden = json.load(fh)
    for name in sorted(bench_mod.WORKLOAD_NAMES):
        base = name
        for suffix in ("-fponly", "-verify", "-wt"):
            if base.endswith(suffix):
                base = base[: -len(suffix)]
        assert base in bench_mod.GOLDEN_NAMES, name
        sec, key = bench_mod.GOLDEN_NAMES[base]
        rec = golden[sec][key]
        assert len(rec["d_sha256"]) == 64, name
        if sec == "workloads":
            assert len(rec["fp_sha256"]) == 64, name
