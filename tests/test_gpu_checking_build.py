"""The bounds-checking build on the GPU.

libmmaemu_check.so is the same library compiled with MMAEMU_BOUNDS_CHECK:
every global index a kernel computes (operand loads, decoded-panel writes and
copies, C/D/claimed-D/fingerprint accesses) is checked against the extent of
its buffer, and a violation is recorded in the device status word and the
access skipped (no trap, no fault).  A child process loads that build
(MMAEMU_LIB=check), runs GEMMs of every layout and mode and tile batches on
small and ragged shapes, compares them with the oracle, and requires the
status word to stay clear -- a substitute for a memory checker, which this
pool does not run.  A second child runs the full-size workloads (device and
host-memory GEMMs, the batched GEMM, streamed tiles) against the oracle's
stored digests under the same build.
"""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

CHILD = r"""
import sys
sys.path.insert(0, ROOT); sys.path.insert(0, HERE)
import numpy as np, torch
import bit_exact_tensor_b200 as mmaemu
from bit_exact_tensor_b200 import workloads as wl
from oracle import cref
from gemm_inputs import normal_inputs, special_inputs, accumulator_edge_inputs
from gpu_util import dev_in, dev_f32, host_bits

assert mmaemu.bounds_checking(), "not the checking build"
mmaemu.device_status(clear=True)
checked = 0
for model, fmt in wl.PAIRS:
    for (M, N, K) in ((16, 16, 16), (80, 144, 48), (208, 272, 160)):
        A, B, C = normal_inputs(M, N, K, fmt, seed=M + N + K)
        D, fp = mmaemu.gemm(model, fmt, dev_in(A), dev_in(B), dev_f32(C))
        want = cref.gemm(model, fmt, A, B, C)
        assert np.array_equal(host_bits(D), want), (model, fmt, M, N, K)
        assert np.array_equal(host_bits(fp), cref.tile_fingerprints(want))
        checked += 1
    A, B, C = special_inputs(48, 64, 80, fmt)
    D, _ = mmaemu.gemm(model, fmt, dev_in(A), dev_in(B), dev_f32(C))
    assert np.array_equal(host_bits(D), cref.gemm(model, fmt, A, B, C)), (model, fmt, "specials")
    A, B, C = accumulator_edge_inputs(fmt, seed=23)
    D, _ = mmaemu.gemm(model, fmt, dev_in(A), dev_in(B), dev_f32(C))
    assert np.array_equal(host_bits(D), cref.gemm(model, fmt, A, B, C)), (model, fmt, "edges")
    At, Bt, Ct, _ = wl.config2(fmt, ntiles=777, seed=4)
    Dt = mmaemu.tiles(model, fmt, dev_in(At), dev_in(Bt), dev_f32(Ct))
    assert np.array_equal(host_bits(Dt), cref.tiles(model, fmt, At, Bt, Ct)), (model, fmt, "tiles")
# transposed, strided-batched, fingerprint-only and verify modes
A, B, C = wl.config_batched(3, 80, 144, 64, seed=11)
Ad, Bd, Cd = dev_in(A), dev_in(B), dev_f32(C)
D, fp = mmaemu.gemm_batched("ampere", "fp16", Ad.transpose(-1, -2).contiguous().transpose(-1, -2),
                            Bd.transpose(-1, -2).contiguous().transpose(-1, -2), Cd)
for b in range(3):
    assert np.array_equal(host_bits(D[b]), cref.gemm("ampere", "fp16", A[b], B[b], C[b])), ("batched", b)
_, fp2 = mmaemu.gemm("ampere", "fp16", Ad[0], Bd[0], Cd[0], store_d=False)
assert np.array_equal(host_bits(fp2), host_bits(fp[0]))
mism, _ = mmaemu.gemm_verify("ampere", "fp16", Ad[0], Bd[0], Cd[0], D[0].contiguous())
assert mism.cpu().tolist()[0] == 0
torch.cuda.synchronize()
bits = mmaemu.device_status()
assert bits == 0, f"status word {bits:#x}"
print("CHECKED", checked)
"""


def test_checking_build_runs_clean_and_exact():
    env = dict(os.environ, MMAEMU_LIB="check")
    code = "ROOT = %r\nHERE = %r\n" % (ROOT, HERE) + CHILD
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "CHECKED 21" in r.stdout


FULL_CHILD = r"""
import sys, json, hashlib
sys.path.insert(0, ROOT); sys.path.insert(0, HERE)
import numpy as np, torch
import bit_exact_tensor_b200 as mmaemu
from bit_exact_tensor_b200 import workloads as wl

assert mmaemu.bounds_checking(), "not the checking build"
mmaemu.device_status(clear=True)
G = json.load(open(GOLDEN))
sha = lambda x: hashlib.sha256(np.ascontiguousarray(x, dtype="<u4").tobytes()).hexdigest()

def host(x):
    v = x.view(np.uint8) if x.dtype == np.uint8 else x.view(np.int16) if x.dtype == np.uint16 else x.view(np.int32)
    return torch.from_numpy(np.ascontiguousarray(v)).pin_memory()

A, B, C = wl.config3()
rec = G["workloads"]["cfg3-ampere-fp16-4096"]
D, fp = mmaemu.gemm("ampere", "fp16", host(A).cuda(), host(B).cuda(), host(C).cuda())
assert sha(D.cpu().numpy().view(np.uint32)) == rec["d_sha256"] and sha(fp.cpu().numpy().view(np.uint32)) == rec["fp_sha256"]
Dh, fph = mmaemu.gemm_host("ampere", "fp16", host(A), host(B), host(C))
assert sha(Dh.numpy().view(np.uint32)) == rec["d_sha256"] and sha(fph.numpy().view(np.uint32)) == rec["fp_sha256"]
A, B, C = wl.config_batched(8, 1024, 4096, 4096)
rec = G["workloads"]["batched-ampere-fp16-8x1024x4096x4096"]
D, fp = mmaemu.gemm_batched("ampere", "fp16", host(A).cuda(), host(B).cuda(), host(C).cuda())
assert sha(D.cpu().numpy().view(np.uint32).reshape(-1, 4096)) == rec["d_sha256"]
assert sha(fp.cpu().numpy().view(np.uint32)) == rec["fp_sha256"]
A, B, C, _ = wl.config2("fp16")
Dt = mmaemu.tiles_host("ampere", "fp16", host(A), host(B), host(C))
assert sha(Dt.numpy().view(np.uint32)) == G["tiles"]["tiles-ampere-fp16-100k"]["d_sha256"]
torch.cuda.synchronize()
bits = mmaemu.device_status()
assert bits == 0, f"status word {bits:#x}"
print("FULL CHECKED")
"""


def test_checking_build_at_full_size():
    """The same build on the full-size workloads: the 4096^3 FP16-Ampere GEMM
    from device and from host memory (row slabs on two compute streams), the
    batched GEMM and 100,000 tiles streamed from host memory in chunks.  Every
    result equals the oracle's stored digests and no index leaves its
    buffer."""
    env = dict(os.environ, MMAEMU_LIB="check")
    golden = os.path.join(HERE, "golden", "fullsize_gemm.json")
    code = "ROOT = %r\nHERE = %r\nGOLDEN = %r\n" % (ROOT, HERE, golden) + FULL_CHILD
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "FULL CHECKED" in r.stdout
