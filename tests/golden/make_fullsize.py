"""Write the oracle's results for the full-size GEMM workloads.

Runs the plain-C oracle (``oracle/mmaemu_ref.c`` through ``oracle.cref``)
on every output element of the large K-chained GEMMs and stores, per
workload, digests that let a GPU test check the whole result without the
oracle having to run again:

  * ``d_sha256``   -- SHA-256 of D (M x N fp32 bit patterns, little-endian,
                      row-major): equal digests mean every element is equal;
  * ``fp_sha256``  -- SHA-256 of the per-16x16-tile xorsum fingerprints
                      (the AEGIS fingerprint, tiles in row-major grid order);
  * ``slab_sha16`` -- the first 16 hex digits of the SHA-256 of each 16-row
                      slab of D, so that a mismatch can be located;
  * ``xorsum`` and counts of special results (+-Inf, NaN, +-0) as readable
    properties.

The workloads are the pages' MatMul experiments ("Hawkeye: Reproducing
GPU-Level Non-Determinism (MLSys 2026)" notes, Experiments and results:
4096 x 4096 MatMuls in each model/format pair) plus the LLM-layer E4M3 GEMM,
with the seeded synthetic inputs of ``bit_exact_tensor_b200/workloads.py``.
Only the oracle and the input generators are called here; nothing comes from
the CUDA library.  The oracle's wall time for each full workload is stored
beside the digests (``oracle_seconds``, ``oracle_threads``).

  python tests/golden/make_fullsize.py [--only NAME ...] [--threads T]
  python tests/golden/make_fullsize.py --tiles     # digests of the tile workloads
  python tests/golden/make_fullsize.py --time-only NAME --threads 1
  python tests/golden/make_fullsize.py --time-python-tiles  # Python oracle, 4,096 tiles
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import platform
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

OUT = os.path.join(HERE, "fullsize_gemm.json")


def workloads():
    from bit_exact_tensor_b200 import workloads as wl

    return {
        "cfg3-ampere-fp16-4096": ("ampere", "fp16", wl.config3),
        "cfg4-hopper-bf16-4096": ("hopper", "bf16", wl.config4),
        "cfg4b-hopper-bf16-4096-wide": ("hopper", "bf16", lambda: wl.config4(wide=True)),
        "cfg5-hopper-e4m3-8192x4096x14336": ("hopper", "e4m3", wl.config5),
        # B200's own FP16 MMA as measured with the pages' target tests: the
        # 4096^3 inputs of config 3 under that model
        "cfg3-b200-fp16-4096": ("b200", "fp16", wl.config3),
        # 8 independent 1024 x 4096 x 4096 problems (the layouts' batched
        # GEMM): D stacked as [8 * 1024, 4096], fingerprints batch-major
        "batched-ampere-fp16-8x1024x4096x4096": ("ampere", "fp16", lambda: wl.config_batched(8, 1024, 4096, 4096)),
    }


def digests(D, fp) -> dict:
    """Digests of a result D ([M, N] uint32) and its tile fingerprints; the
    GPU tests compute the same from the GPU's arrays (a plain function of the
    bytes, no emulation arithmetic)."""
    import numpy as np

    D = np.ascontiguousarray(D, dtype="<u4")
    fp = np.ascontiguousarray(fp, dtype="<u4")
    M = D.shape[0]
    slabs = [hashlib.sha256(D[i:i + 16].tobytes()).hexdigest()[:16] for i in range(0, M, 16)]
    return {"d_sha256": hashlib.sha256(D.tobytes()).hexdigest(),
            "fp_sha256": hashlib.sha256(fp.tobytes()).hexdigest(),
            "slab_sha16": slabs}


def special_counts(D) -> dict:
    import numpy as np

    mag = D & 0x7FFFFFFF
    return {"pos_inf": int((D == 0x7F800000).sum()), "neg_inf": int((D == 0xFF800000).sum()),
            "nan": int((mag > 0x7F800000).sum()), "pos_zero": int((D == 0).sum()),
            "neg_zero": int((D == 0x80000000).sum()), "subnormal": int(((mag > 0) & (mag < 0x00800000)).sum())}


def run_one(name: str, threads: int) -> dict:
    from oracle import cref

    model, fmt, make = workloads()[name]
    A, B, C = make()
    t0 = time.perf_counter()
    if A.ndim == 3:  # a batch of independent problems, one oracle run each
        parts = [cref.gemm(model, fmt, A[b], B[b], C[b], nthreads=threads) for b in range(A.shape[0])]
        fp = np.concatenate([cref.tile_fingerprints(Db) for Db in parts])
        D = np.concatenate(parts, axis=0)
        batch = A.shape[0]
    else:
        D = cref.gemm(model, fmt, A, B, C, nthreads=threads)
        fp = cref.tile_fingerprints(D)
        batch = 1
    dt = time.perf_counter() - t0
    M, K = A.shape[-2:]
    N = B.shape[-1]
    rec = {"model": model, "fmt": fmt, "M": M, "N": N, "K": K, "xorsum": cref.xorsum(D),
           "specials": special_counts(D), "oracle_seconds": round(dt, 2), "oracle_threads": threads,
           "oracle_macs_per_s": batch * M * N * K / dt}
    if batch > 1:
        rec["batch"] = batch
    rec.update(digests(D, fp))
    return rec


def host_info() -> dict:
    cpu = platform.processor() or ""
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    cpu = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu": cpu, "logical_cpus_available": len(os.sched_getaffinity(0))}


def tile_workloads():
    """The pages' random-tile experiments: 4,096 Ampere-FP16 tiles with
    subnormals, and 100,000 random + adversarial tiles per model/format
    pair."""
    from bit_exact_tensor_b200 import workloads as wl

    out = {"tiles-ampere-fp16-4096": ("ampere", "fp16", wl.config1)}
    for model, fmt in wl.PAIRS:
        out[f"tiles-{model}-{fmt}-100k"] = (model, fmt, lambda fmt=fmt: wl.config2(fmt)[:3])
    return out


def run_tiles(threads: int) -> dict:
    """SHA-256 of the oracle's D for every tile workload."""
    from oracle import cref

    recs = {}
    for name, (model, fmt, make) in tile_workloads().items():
        A, B, C = make()
        t0 = time.perf_counter()
        D = cref.tiles(model, fmt, A, B, C, nthreads=threads)
        dt = time.perf_counter() - t0
        D = np.ascontiguousarray(D, dtype="<u4")
        recs[name] = {"model": model, "fmt": fmt, "ntiles": int(A.shape[0]),
                      "d_sha256": hashlib.sha256(D.tobytes()).hexdigest(),
                      "specials": special_counts(D), "oracle_seconds": round(dt, 2), "oracle_threads": threads}
        print(name, recs[name]["oracle_seconds"], "s", flush=True)
    return recs


def time_python_tiles() -> dict:
    """Wall time of the Python oracle (arbitrary-precision integers, one
    element at a time) on the 4,096 Ampere-FP16 tiles of the small tile
    workload, single-threaded."""
    from bit_exact_tensor_b200 import workloads as wl
    from oracle import mma_model as mm

    A, B, C = wl.config1()
    model, fmt = mm.MODELS["ampere"], mm.FORMATS["fp16"]
    t0 = time.perf_counter()
    for t in range(A.shape[0]):
        mm.mma_tile(model, fmt, A[t].tolist(), B[t].tolist(), C[t].tolist())
    dt = time.perf_counter() - t0
    return {"workload": "4,096 Ampere-FP16 tiles (16.8 M MACs)", "seconds": round(dt, 1), "threads": 1,
            "macs_per_s": A.shape[0] * 4096 / dt}


def main() -> int:
    from oracle import cref

    ap = argparse.ArgumentParser()
    ap.add_argument("--only", nargs="*", default=None)
    ap.add_argument("--threads", type=int, default=cref.default_threads())
    ap.add_argument("--time-only", default=None, help="time one workload, store only its timing")
    ap.add_argument("--time-python-tiles", action="store_true")
    ap.add_argument("--tiles", action="store_true", help="store the tile workloads' digests")
    args = ap.parse_args()

    updates = {"workloads": {}, "timings": {}, "tiles": {}}
    if args.tiles:
        updates["tiles"].update(run_tiles(args.threads))
    elif args.time_python_tiles:
        updates["timings"]["python_oracle_tiles_4096"] = dict(time_python_tiles(), host=host_info())
    elif args.time_only:
        rec = run_one(args.time_only, args.threads)
        want = load().get("workloads", {}).get(args.time_only)
        if want is not None and want["d_sha256"] != rec["d_sha256"]:
            raise SystemExit(f"{args.time_only}: result differs from the stored digest")
        updates["timings"][f"{args.time_only}-{args.threads}threads"] = {
            "seconds": rec["oracle_seconds"], "threads": args.threads, "macs_per_s": rec["oracle_macs_per_s"],
            "host": host_info()}
    else:
        for name in args.only or list(workloads()):
            rec = run_one(name, args.threads)
            rec["host"] = host_info()
            print(name, rec["oracle_seconds"], "s", rec["specials"], flush=True)
            save({"workloads": {name: rec}})
    save(updates)
    return 0


def load() -> dict:
    if os.path.exists(OUT):
        with open(OUT) as fh:
            return json.load(fh)
    return {}


def save(updates: dict) -> None:
    """Merge into the file as it is now (other runs may have written to it
    meanwhile)."""
    data = load()
    for sec, recs in updates.items():
        data.setdefault(sec, {}).update(recs)
    with open(OUT, "w") as fh:
        json.dump(data, fh, indent=1, sort_keys=True)
        fh.write("\n")


if __name__ == "__main__":
    sys.exit(main())
