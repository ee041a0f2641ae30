"""Benchmark: emulated MACs/s of the 4096^3 FP16-Ampere bit-exact GEMM.

One step = one mmaemu_gemm call on the 4096x4096x4096 Ampere-FP16 workload
(A, B fp16 ~ N(0,1), C = +0, per-16x16-tile xorsum fingerprints), i.e. the
whole hot path: operand staging and decode, exact products, per-group max
exponent, truncating alignment and signed sum, Ampere stage hand-over,
toward-zero write-back, the 256-chunk K chain and the fused fingerprint
epilogue.  Inputs are resident in HBM before timing starts; the 192 MiB
working set (A 32 MiB, B 32 MiB, C 64 MiB, D 64 MiB) is larger than the
126 MB L2.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

With --gpus N > 1 launch it under torchrun: every rank runs its own
4096^3 problem on its own GPU (weak scaling, the work partitions into
independent problems, no data-path collective); the reported time is the max
over ranks and ``value`` counts the MACs of all ranks.

``--impl reference`` times the CPU oracle (the plain C restatement of the
model) on the host cores on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

M = N = K = 4096
MACS_PER_STEP = M * N * K
# algorithmic integer ops per emulated MAC in the integer formulation of the
# model (exponent add, max, shift amount, significand product, truncating
# shift, sign, accumulate): the INT32-ALU roofline the metric names
OPS_PER_MAC = 7
METRIC = "emulated MACs/s for 4096^3 FP16-Ampere GEMM; % of INT32-ALU roofline; bit-exact"
UNIT = "MAC/s"
# Pages' CPU simulator, same workload: 50.8 s per 4096x4096 FP16-Ampere MatMul
# (K = 4096) on an Apple M4 Pro -> 68.72e9 / 50.8 MAC/s.  Context, not a target.
PAGES_MACS_PER_S = MACS_PER_STEP / 50.8
SMS, MAX_SM_MHZ = 148, 1965.0
# Nominal unit counts, for context only: the rooflines use the issue rates
# that libmmaemu_peaks measures on the GPU in the same run (lanes per SM per
# clock, see --pipe-rates and profiles/pipe_rates_b200.md).
NOMINAL_FP64_LANES, NOMINAL_INT32_LANES = 64, 128
H2D_BYTES = M * K * 2 + K * N * 2 + M * N * 4
D2H_BYTES = M * N * 4 + (M // 16) * (N // 16) * 4
ALGO_BYTES = H2D_BYTES + D2H_BYTES  # A, B, C read and D, fingerprints written once
WORKLOAD = "gemm M=N=K=4096, Ampere FP16 model, fp32 C=0 and D, fused per-16x16-tile xorsum"
# DRAM bytes per launch of the GEMM kernel (dram__bytes_read.sum + dram__bytes_write.sum)
# from one ncu capture (its summary is committed under profiles/), valid only
# for the kernel sources it was taken on, identified by their hash.
TRAFFIC_CAPTURE = {"source_sha16": "6a57c870d1eafe47", "bytes": 1634566400}
KERNEL_SOURCES = ("bit_exact_tensor_b200/csrc/mmaemu.cu", "bit_exact_tensor_b200/csrc/mmaemu_core.cuh",
                  "include/mmaemu.h")
GOLDEN = os.path.join(ROOT, "tests", "golden", "fullsize_gemm.json")
# workload name -> record name of the stored oracle digests
GOLDEN_NAMES = {"gemm-ampere-fp16-4096": ("workloads", "cfg3-ampere-fp16-4096"),
                "gemm-hopper-bf16-4096": ("workloads", "cfg4-hopper-bf16-4096"),
                "gemm-hopper-bf16-4096-wide": ("workloads", "cfg4b-hopper-bf16-4096-wide"),
                "gemm-hopper-e4m3-8192x4096x14336": ("workloads", "cfg5-hopper-e4m3-8192x4096x14336"),
                "gemm-b200-fp16-4096": ("workloads", "cfg3-b200-fp16-4096")}
PEAK_OPS = {"dfma": 0, "dadd": 1, "add_min_s16x2": 2, "lop3": 3, "imad": 4, "iadd": 5, "popc_xor": 6, "prmt": 7,
            "imnmx": 8, "ffma": 9,
            # pairs on independent chains (rate in pairs): do two pipes work at the same time?
            "pair_dfma_lop3": 10, "pair_dfma_imad": 11, "pair_dfma_ffma": 12, "pair_dfma_add_min_s16x2": 13,
            "pair_lop3_imad": 14, "pair_lop3_ffma": 15}


def hbm_peak_gbs():
    """The driver's measured copy bandwidth (MEASURED_PEAKS.json), else the
    pool's earlier measurement."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            return float(json.load(fh)["hbm_gbs"]), "MEASURED_PEAKS.json hbm_gbs (measured copy)"
    except (OSError, KeyError, ValueError):
        return 6650.0, "fallback 6.65 TB/s (earlier measurement on this pool)"
DEFAULT_WORKLOAD = "gemm-ampere-fp16-4096"
PAIRS = (("ampere", "fp16"), ("ampere", "bf16"), ("hopper", "fp16"), ("hopper", "bf16"), ("hopper", "e4m3"),
         ("b200", "fp16"), ("b200", "bf16"))
GOLDEN_NAMES.update({"tiles-ampere-fp16-4096": ("tiles", "tiles-ampere-fp16-4096")})
GOLDEN_NAMES.update({f"tiles-{m}-{f}-100k": ("tiles", f"tiles-{m}-{f}-100k") for m, f in PAIRS})
E4M3_LAYER = "gemm-hopper-e4m3-8192x4096x14336"
# variants of the E4M3 layer GEMM: fingerprints only (no D written), verify
# a claimed D instead of storing it, weights stored [N][K] (B transposed)
GEMM_MODES = ("fponly", "verify", "wt")
BATCHED = "gemm-batched-ampere-fp16-8x1024x4096x4096"
GOLDEN_NAMES[BATCHED] = ("workloads", "batched-ampere-fp16-8x1024x4096x4096")
WORKLOAD_NAMES = ({DEFAULT_WORKLOAD, "gemm-hopper-bf16-4096", "gemm-hopper-bf16-4096-wide", E4M3_LAYER,
                   "tiles-ampere-fp16-4096", BATCHED, "gemm-b200-fp16-4096"}
                  | {f"{E4M3_LAYER}-{m}" for m in GEMM_MODES}
                  | {f"tiles-{m}-{f}-100k" for m, f in PAIRS})


def workload_spec(name: str) -> dict:
    """Inputs and byte/MAC counts of a named workload (the configurations of
    the Hawkeye workloads: random 16x16x16 tiles and large GEMMs)."""
    from bit_exact_tensor_b200 import workloads as wl

    def gemm(model, fmt, make, M_, N_, K_, desc):
        eb = 1 if fmt == "e4m3" else 2
        return {"kind": "gemm", "model": model, "fmt": fmt, "make": make, "macs": M_ * N_ * K_, "desc": desc,
                "mn": (M_, N_), "mode": "store",
                "h2d": (M_ * K_ + K_ * N_) * eb + M_ * N_ * 4, "d2h": M_ * N_ * 4 + (M_ // 16) * (N_ // 16) * 4,
                "l2": "inputs larger than L2"}

    def tiles(model, fmt, make, nt, desc):
        eb = 1 if fmt == "e4m3" else 2
        return {"kind": "tiles", "model": model, "fmt": fmt, "make": make, "macs": nt * 4096, "desc": desc,
                "h2d": nt * 256 * (2 * eb + 4), "d2h": nt * 1024,
                "l2": "inputs larger than L2" if nt * 256 * (2 * eb + 8) > 126e6 else "fits in L2"}

    for mode in GEMM_MODES:
        if name.endswith("-" + mode):
            spec = workload_spec(name[: -len(mode) - 1])
            M_, N_ = spec["mn"]
            out_d, out_fp = M_ * N_ * 4, (M_ // 16) * (N_ // 16) * 4
            if mode == "fponly":
                spec.update(d2h=out_fp, desc=spec["desc"] + ", fingerprints only (D not written)")
            elif mode == "verify":
                spec.update(h2d=spec["h2d"] + out_d, d2h=16,
                            desc=spec["desc"].replace(", fused per-tile xorsum", "")
                            + ", verify mode (claimed D read and compared, not written)")
            else:
                spec.update(desc=spec["desc"] + ", B stored [N][K] (weights layout)")
            spec["mode"] = mode
            return spec
    if name == BATCHED:
        b_, m_, n_, k_ = 8, 1024, 4096, 4096
        spec = gemm("ampere", "fp16", lambda r: wl.config_batched(b_, m_, n_, k_, seed=7 + 1000 * r), m_, n_, k_,
                    f"batched gemm, {b_} independent problems M={m_} N={n_} K={k_} (A, B, C per problem), "
                    "Ampere FP16 model, N(0,1), fused per-tile xorsum")
        spec.update(macs=b_ * spec["macs"], h2d=b_ * spec["h2d"], d2h=b_ * spec["d2h"], mode="batched")
        return spec
    if name == DEFAULT_WORKLOAD:
        return gemm("ampere", "fp16", lambda r: wl.config3(seed=3 + 1000 * r), M, N, K, WORKLOAD)
    if name == "gemm-b200-fp16-4096":
        return gemm("b200", "fp16", lambda r: wl.config3(seed=3 + 1000 * r), 4096, 4096, 4096,
                    "gemm M=N=K=4096, B200 FP16 model (B200's own MMA, measured), A, B ~ N(0,1), C = 0, "
                    "fused per-tile xorsum")
    if name == "gemm-hopper-bf16-4096":
        return gemm("hopper", "bf16", lambda r: wl.config4(seed=4 + 1000 * r), 4096, 4096, 4096,
                    "gemm M=N=K=4096, Hopper BF16 model, log2|x| ~ U[-60, 60], fused per-tile xorsum")
    if name == "gemm-hopper-bf16-4096-wide":
        return gemm("hopper", "bf16", lambda r: wl.config4(seed=4 + 1000 * r, wide=True), 4096, 4096, 4096,
                    "gemm M=N=K=4096, Hopper BF16 model, log2|x| ~ U[-126, 127], fused per-tile xorsum")
    if name == E4M3_LAYER:
        return gemm("hopper", "e4m3", lambda r: wl.config5(seed=5 + 1000 * r), 8192, 14336, 4096,
                    "gemm M=8192 K=4096 N=14336, Hopper E4M3 model, N(0,1)/sqrt(K), fused per-tile xorsum")
    if name == "tiles-ampere-fp16-4096":
        return tiles("ampere", "fp16", lambda r: wl.config1(seed=0 + 1000 * r), 4096,
                     "4,096 tiles 16x16x16, Ampere FP16 model, 10% subnormal entries")
    for m, f in PAIRS:
        if name == f"tiles-{m}-{f}-100k":
            def make(r, f=f):
                A_, B_, C_, _ = wl.config2(f, seed=1 + 1000 * r)
                return A_, B_, C_
            return tiles(m, f, make, 100_000,
                         f"100,000 random + adversarial tiles, {m.capitalize() if m != 'b200' else 'B200'} "
                         f"{f.upper()} model")
    raise ValueError(name)


def kernel_source_sha16() -> str:
    import hashlib

    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic():
    return TRAFFIC_CAPTURE["bytes"] if kernel_source_sha16() == TRAFFIC_CAPTURE["source_sha16"] else None


def measure_rates(ops=("dfma", "iadd"), iters=20000):
    """Issue rates (lanes per SM per clock) of instruction classes, measured
    on the current GPU by libmmaemu_peaks (see csrc/peaks.cu)."""
    import ctypes

    from bit_exact_tensor_b200 import _build

    L = ctypes.CDLL(_build.LIB_PEAKS)
    L.mmaemu_peak_rate.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_double),
                                   ctypes.POINTER(ctypes.c_double)]
    L.mmaemu_peak_rate.restype = ctypes.c_int
    out = {}
    for op in ops:
        lanes, secs = ctypes.c_double(0), ctypes.c_double(0)
        rc = L.mmaemu_peak_rate(PEAK_OPS[op], iters, ctypes.byref(lanes), ctypes.byref(secs))
        if rc != 0:
            raise RuntimeError(f"mmaemu_peak_rate({op}) failed: {rc}")
        out[op] = lanes.value
    return out


def verify_against_oracle(name, D_host, fp_host):
    """Compare the timed call's result with the oracle's digests stored in
    tests/golden/fullsize_gemm.json (written by tests/golden/make_fullsize.py
    from a run of the oracle on every output element).  Returns the record
    for the JSON line; raises on any difference."""
    import hashlib

    import numpy as np

    if name not in GOLDEN_NAMES or not os.path.exists(GOLDEN):
        return {"verified": None, "against": "no stored oracle digest for this workload"}
    sec, key = GOLDEN_NAMES[name]
    with open(GOLDEN) as fh:
        rec = json.load(fh).get(sec, {}).get(key)
    if rec is None:
        return {"verified": None, "against": "no stored oracle digest for this workload"}
    d = np.ascontiguousarray(D_host.view(np.uint32), dtype="<u4")
    got_d = hashlib.sha256(d.tobytes()).hexdigest()
    out = {"against": f"oracle digests, tests/golden/fullsize_gemm.json [{sec}][{key}]",
           "d_sha256_equal": got_d == rec["d_sha256"]}
    if fp_host is not None and "fp_sha256" in rec:
        fp = np.ascontiguousarray(fp_host.view(np.uint32), dtype="<u4")
        out["fp_sha256_equal"] = hashlib.sha256(fp.tobytes()).hexdigest() == rec["fp_sha256"]
    out["verified"] = all(v for k, v in out.items() if k.endswith("_equal"))
    if not out["verified"]:
        raise RuntimeError(f"{name}: the timed result differs from the oracle's ({out})")
    return out


def verify_fp_against_oracle(name, fp_host):
    """The fingerprint-only mode's result against the oracle's stored
    fingerprint digest; raises on a difference."""
    import hashlib

    import numpy as np

    if not GOLDEN_NAMES.get(name) or not os.path.exists(GOLDEN):
        return {"verified": None, "against": "no stored oracle digest for this workload"}
    sec, key = GOLDEN_NAMES[name]
    with open(GOLDEN) as fh:
        want = json.load(fh)[sec][key]["fp_sha256"]
    got = hashlib.sha256(np.ascontiguousarray(fp_host.view(np.uint32), dtype="<u4").tobytes())
    out = {"verified": got.hexdigest() == want, "against": f"oracle fingerprint digest [{sec}][{key}]"}
    if not out["verified"]:
        raise RuntimeError("fingerprints differ from the oracle's")
    return out


def run_pipe_rates():
    """Print the measured issue rates of the instruction classes the kernels
    use, with the SM clock sampled during the probes."""
    import torch

    torch.cuda.init()
    with ClockSampler(0) as cs:
        rates = measure_rates(tuple(PEAK_OPS), iters=100000)
    clocks = cs.summary()
    mhz = clocks.get("sm_mhz") or MAX_SM_MHZ
    line = {"pipe_rates_lanes_per_sm_clk": {k: round(v, 2) for k, v in rates.items()},
            "sms": torch.cuda.get_device_properties(0).multi_processor_count, "clocks": clocks,
            "dfma_peak_t_per_s_at_max_clock": rates["dfma"] * SMS * MAX_SM_MHZ * 1e6 / 1e12,
            "dfma_peak_t_per_s_at_sampled_clock": rates["dfma"] * SMS * mhz * 1e6 / 1e12,
            "note": "1 block of 1024 threads per SM, 8 independent chains per thread; "
                    "add_min_s16x2 counts one packed add-and-min per lane, popc_xor an xor and a popc; "
                    "pair_* run both kinds on separate chains and count pairs"}
    print(json.dumps(line), flush=True)
    return 0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing leg")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOAD_NAMES),
                    help="which workload to time (default: the headline 4096^3 FP16-Ampere GEMM)")
    ap.add_argument("--pipe-rates", action="store_true",
                    help="measure the issue rates of the instruction classes the kernels use, and exit")
    return ap.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


# ---------------------------------------------------------------------------
# clocks sampling during the timed region
# ---------------------------------------------------------------------------
CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"mmaemu_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={CLOCK_FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu), "-lms", "100"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[4], parts[5:9]))
            except ValueError:
                continue
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[4]) if v.lower() == "active"})
        loaded = [r for r in rows if r[2] > 200.0] or rows
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": max(r[2] for r in rows), "samples": len(rows), "reasons": reasons}


def clocks_bad(cl):
    if any(r in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown") for r in cl.get("reasons", [])):
        return True
    if cl.get("sm_mhz") and cl.get("sm_max_mhz") and not cl.get("reasons"):
        return cl["sm_mhz"] < 0.6 * cl["sm_max_mhz"]
    return False


# ---------------------------------------------------------------------------
# CPU oracle timing (baseline leg and reference arm)
# ---------------------------------------------------------------------------
def oracle_rows(rows: int, nthreads: int, inputs=None):
    from oracle import cref
    from bit_exact_tensor_b200 import workloads as wl

    A, B, C = inputs if inputs is not None else wl.config3()
    t0 = time.perf_counter()
    cref.gemm("ampere", "fp16", A, B, C, rows=(0, rows), nthreads=nthreads)
    return time.perf_counter() - t0


def sample_rows(seconds: float, nthreads: int, inputs) -> int:
    """Output rows the oracle computes in about `seconds` on nthreads threads.
    The oracle hands out whole rows to its threads, so the probe runs two
    rows per thread (every thread busy) and the answer is a multiple of
    nthreads."""
    probe = 2 * nthreads
    per_row = oracle_rows(probe, nthreads, inputs) / probe
    rows = int(seconds / max(per_row, 1e-9)) // nthreads * nthreads
    return int(max(nthreads, min(M, rows)))


def cpu_baseline(target_s: float = 15.0, inputs=None):
    """Time the oracle as it stands on a bounded sample: the first R output
    rows of the same GEMM (R x 4096 x 4096 MACs), R sized for ~target_s."""
    from oracle import cref

    nthreads = cref.default_threads()
    rows = sample_rows(target_s, nthreads, inputs)
    dt = oracle_rows(rows, nthreads, inputs)
    macs = rows * N * K
    return {"value": macs / dt, "unit": UNIT, "cores": nthreads, "kind": "oracle",
            "sample": f"output rows [0,{rows}) of the 4096^3 FP16-Ampere GEMM ({macs:.3e} MACs) "
                      f"by the plain-C oracle, {nthreads} threads, {dt:.1f} s"}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    from oracle import cref
    from bit_exact_tensor_b200 import workloads as wl

    inputs = wl.config3()
    nthreads = cref.default_threads()
    steps, warmup = args.steps, args.warmup
    budget = 150.0  # seconds for the whole run
    rows = sample_rows(budget / (steps + warmup), nthreads, inputs)
    for _ in range(warmup):
        oracle_rows(rows, nthreads, inputs)
    times = [oracle_rows(rows, nthreads, inputs) for _ in range(steps)]
    tot = sum(times)
    macs = rows * N * K * steps
    value = macs / tot
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": steps, "warmup": warmup, "ms_per_step": 1e3 * tot / steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": value / PAGES_MACS_PER_S, "dtype": "int64",
            "data": "synthetic", "config": {"workload": WORKLOAD, "sample_rows_per_step": rows},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": nthreads, "kind": "oracle",
                             "sample": f"output rows [0,{rows}) per step of the 4096^3 FP16-Ampere GEMM"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# multi-rank host logic
# ---------------------------------------------------------------------------
def reduce_max(x: float, dist=None, device=None) -> float:
    """Max of a per-rank float over all ranks (identity without a process
    group).  Works with NCCL (device tensor) and gloo (CPU tensor)."""
    if dist is None:
        return x
    import torch

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def any_rank(flag: bool, dist=None, device=None) -> bool:
    """True on every rank when the flag is set on any rank."""
    return reduce_max(1.0 if flag else 0.0, dist, device) > 0.0


def aggregate_value(step_ms_max: float, world: int, macs_per_step: int = MACS_PER_STEP) -> float:
    """Whole-job emulated MACs/s: every rank runs one full problem per step
    (weak scaling), timed by the slowest rank."""
    return macs_per_step * world / (step_ms_max / 1e3)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def run_gpu(args):
    import numpy as np
    import torch

    import bit_exact_tensor_b200 as mmaemu
    from bit_exact_tensor_b200 import workloads as wl

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if dist is not None:
            dist.barrier()

    def max_over_ranks(x: float) -> float:
        return reduce_max(x, dist, dev)

    spec = workload_spec(args.workload)
    mode = spec.get("mode")
    A_np, B_np, C_np = spec["make"](rank)
    in_view = np.uint8 if spec["fmt"] == "e4m3" else np.int16
    if mode == "wt":  # weights layout: B stored as [N][K]
        B_np = np.ascontiguousarray(B_np.T)
    A = torch.from_numpy(A_np.view(in_view)).to(dev)
    B = torch.from_numpy(B_np.view(in_view)).to(dev)
    C = torch.from_numpy(C_np.view(np.int32)).to(dev)
    stream = torch.cuda.current_stream(dev)
    model, fmt = spec["model"], spec["fmt"]
    # opt in to keeping the GEMM's decoded-operand workspace between calls
    # (the library's default hands it back after every call); declared in
    # the JSON line's config
    mmaemu.set_workspace_cache(True)
    # kernels of ours per timed step: decode B, decode A, MMA for a GEMM call;
    # one tile kernel for a tile batch
    launches_per_step = 3 if spec["kind"] == "gemm" else 1
    if spec["kind"] == "gemm":
        D = torch.empty(C.shape, dtype=torch.float32, device=dev)
        fp = torch.empty(((C.shape[-2] // 16) * (C.shape[-1] // 16),), dtype=torch.int32, device=dev)
        if mode == "store":
            def step():
                mmaemu.gemm(model, fmt, A, B, C, out=D, fp_out=fp)
        elif mode == "fponly":
            def step():
                mmaemu.gemm(model, fmt, A, B, C, fp_out=fp, store_d=False)
        elif mode == "verify":
            mmaemu.gemm(model, fmt, A, B, C, out=D, fingerprint=False)  # the claim to verify
            mism = torch.empty((2,), dtype=torch.int64, device=dev)

            def step():
                mmaemu.gemm_verify(model, fmt, A, B, C, D, mismatch_out=mism)
        elif mode == "wt":
            D3 = D.view(1, *D.shape)

            def step():
                mmaemu.gemm_batched(model, fmt, A, B.t(), C, out=D3)
        else:  # batched
            def step():
                mmaemu.gemm_batched(model, fmt, A, B, C, out=D)
    else:
        D = torch.empty(C.shape, dtype=torch.float32, device=dev)

        def step():
            mmaemu.tiles(spec["model"], spec["fmt"], A, B, C, out=D)

    def timed():
        """W untimed warm-up steps right before the timed ones (the clock
        sampler has just started and left the GPU idle), then K steps between
        a barrier and a synchronisation, timed by events around the whole run
        (the value), then K more with an event pair around each call (each
        launch's duration, for the roofline).  The first timed pass records
        nothing between steps: for the short tile batches the per-step event
        records cost enough host time to leave the GPU idle between calls."""
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize(dev)
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize(dev)
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        torch.cuda.synchronize(dev)
        for s, e in ev:
            s.record(stream)
            step()
            e.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        per = [s.elapsed_time(e) for s, e in ev]
        return t0.elapsed_time(t1), per

    with ClockSampler(local) as cs:
        total_ms, per_ms = timed()
    clocks = cs.summary()
    # re-measured on every rank when any rank's clock record is bad (the
    # timed steps hold barriers, so all ranks take them together)
    if any_rank(clocks_bad(clocks), dist, dev):
        with ClockSampler(local) as cs:
            total_ms, per_ms = timed()
        clocks = cs.summary()
        clocks["remeasured"] = True
    total_ms = max_over_ranks(total_ms)
    kern_ms = max_over_ranks(sum(per_ms) / len(per_ms))

    if mode == "verify":  # on every rank, the claim must verify clean
        count, first = mism.cpu().tolist()
        if count != 0:
            raise RuntimeError(f"verify mode found {count} mismatches (first at {first}) in its own result")
    if rank != 0:
        # every rank draws its own inputs (seed + 1000 rank); the stored
        # oracle digests describe rank 0's, so rank 0 alone compares with them
        verified = {"verified": None, "against": "checked on rank 0 (the stored digests are of its inputs)"}
    elif mode == "verify":
        # and the claim itself (computed by the library) against the oracle's D
        verified = verify_against_oracle(args.workload.rsplit("-verify", 1)[0], D.cpu().numpy(), None)
        verified["against"] += "; the timed verify calls found 0 mismatches in that claim"
    elif mode in ("store", "wt", "batched", None) or spec["kind"] == "tiles":
        # the last timed call's result against the oracle's stored digests
        # (only the plain GEMM call writes fingerprints here)
        base = args.workload[:-3] if mode == "wt" else args.workload  # B stored [N][K]: the same GEMM
        verified = verify_against_oracle(base, D.cpu().numpy(),
                                         fp.cpu().numpy() if spec["kind"] == "gemm" and mode == "store" else None)
    elif mode == "fponly":
        verified = verify_fp_against_oracle(args.workload.rsplit("-fponly", 1)[0], fp.cpu().numpy())
    else:
        verified = {"verified": None, "against": "no stored oracle digest for this workload"}
    # issue rates of the FP64 pipe and of the fastest INT32 instruction,
    # measured now on this GPU (lanes per SM per clock)
    rates = measure_rates(("dfma", "iadd"))

    # end to end through the public API from pinned host buffers
    A_h = torch.from_numpy(A_np.view(in_view)).pin_memory()
    B_h = torch.from_numpy(B_np.view(in_view)).pin_memory()
    C_h = torch.from_numpy(C_np.view(np.int32)).pin_memory()
    if mode == "verify":
        Dclaim_h = D.cpu().pin_memory()
    if spec["kind"] == "tiles":
        Dt_out_h = torch.empty(C_h.shape, dtype=torch.float32, pin_memory=True)
    if mode in ("store", "fponly"):  # the results land in page-locked buffers owned by the caller
        D_out_h = torch.empty(C_h.shape, dtype=torch.float32, pin_memory=True) if mode == "store" else None
        fp_out_h = torch.empty(((C_h.shape[-2] // 16) * (C_h.shape[-1] // 16),), dtype=torch.int32,
                               pin_memory=True)

    def to_host(t):
        h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        h.copy_(t, non_blocking=True)
        return h

    def e2e_step():
        if mode == "store":
            return mmaemu.gemm_host(model, fmt, A_h, B_h, C_h, device=dev, out=D_out_h, fp_out=fp_out_h)
        if mode == "fponly":  # from host memory, fingerprints only: no D written or copied
            return mmaemu.gemm_host(model, fmt, A_h, B_h, C_h, device=dev, fp_out=fp_out_h, store_d=False)
        if spec["kind"] == "gemm":
            Ad, Bd, Cd = (t.to(dev, non_blocking=True) for t in (A_h, B_h, C_h))
            if mode == "verify":
                Dd = Dclaim_h.to(dev, non_blocking=True)
                out = (to_host(mmaemu.gemm_verify(model, fmt, Ad, Bd, Cd, Dd)[0]), None)
            elif mode == "wt":
                Dd, fpd = mmaemu.gemm_batched(model, fmt, Ad, Bd.t(), Cd)
                out = (to_host(Dd), to_host(fpd))
            else:
                Dd, fpd = mmaemu.gemm_batched(model, fmt, Ad, Bd, Cd)
                out = (to_host(Dd), to_host(fpd))
            torch.cuda.current_stream(dev).synchronize()
            return out
        # tiles: streamed in chunks by the library, copies overlapped
        return mmaemu.tiles_host(model, fmt, A_h, B_h, C_h, device=dev, out=Dt_out_h), None

    for _ in range(max(3, args.warmup)):  # warm-up, as for the device-timed steps
        last = e2e_step()
    last = None
    barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    last = None
    e0.record(stream)
    for _ in range(args.e2e_steps):
        # the previous result is released first, so that its page-locked
        # buffers go back to the host allocator's cache for this call
        last = None
        last = e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps)
    barrier()
    # the last end-to-end call's result, in host memory, against the same
    # oracle digests (rank 0, after the timed region)
    e2e_verified = None
    if rank == 0 and last is not None:
        Dh, fph = last
        if mode == "verify":
            count = int(Dh.view(-1)[0])
            e2e_verified = count == 0
            if count != 0:
                raise RuntimeError(f"the end-to-end verify call found {count} mismatches in the oracle-equal claim")
        elif mode == "fponly":
            e2e_verified = verify_fp_against_oracle(args.workload.rsplit("-fponly", 1)[0], fph.numpy())["verified"]
        else:
            base = args.workload[:-3] if mode == "wt" else args.workload
            e2e_verified = verify_against_oracle(
                base, Dh.numpy(), fph.numpy() if spec["kind"] == "gemm" and mode in ("store", "batched") and fph is not None
                else None)["verified"]

    if rank == 0:
        macs = spec["macs"]
        value = aggregate_value(total_ms / args.steps, world, macs)
        h2d, d2h = spec["h2d"], spec["d2h"]
        mhz = clocks.get("sm_mhz") or MAX_SM_MHZ
        # one round-toward-zero FP64 fused multiply-add per emulated MAC: the
        # bound is the FP64 pipe, at its measured issue rate and the SM clock
        # sampled during the timed region
        fp64_peak = rates["dfma"] * SMS * mhz * 1e6 / 1e12
        achieved = macs / (kern_ms / 1e3) / 1e12
        kernel = (f"gemm_kernel<{spec['model']},{spec['fmt']}> with its two decode kernels (one call, timed whole; "
                  "the MMA kernel is about 99% of it, profiles/gemm_ampere_fp16_4096_launches.md)"
                  if spec["kind"] == "gemm" else f"tiles_kernel<{spec['model']},{spec['fmt']}>")
        roof = {"bound": "fp64", "achieved": achieved, "peak": fp64_peak, "unit": "T FMA/s",
                "frac": achieved / fp64_peak, "kernel": kernel, "fma_per_mac": 1,
                "peak_basis": (f"DFMA issue rate measured in this run: {rates['dfma']:.1f} lanes/SM/clk "
                               f"(libmmaemu_peaks; profiles/pipe_rates_b200.md) x {SMS} SMs x {mhz:.0f} MHz "
                               f"(median SM clock sampled while timing); nominal 64 lanes/SM/clk"),
                # the metric's INT32-ALU roofline: what the integer formulation
                # of the model would need (7 integer ops per MAC) against the
                # measured INT32 issue rate of the fastest integer instruction;
                # the kernels run one FP64 FMA per MAC instead, so this is an
                # equivalent, not what binds them
                "int32_equiv": {"ops_per_mac_integer_form": OPS_PER_MAC,
                                "peak_tops": rates["iadd"] * SMS * mhz * 1e6 / 1e12,
                                "peak_basis": f"IADD issue rate measured in this run: {rates['iadd']:.1f} lanes/SM/clk",
                                "frac": OPS_PER_MAC * achieved / (rates["iadd"] * SMS * mhz * 1e6 / 1e12)}}
        roof.update({"traffic": measured_traffic() if args.workload == DEFAULT_WORKLOAD else None,
                     "traffic_unit": "bytes per launch", "algorithmic_bytes": h2d + d2h})
        if spec["kind"] == "tiles":  # mixed bound: also report HBM against the measured copy bandwidth
            hbm = (h2d + d2h) / (kern_ms / 1e3) / 1e9
            hbm_peak, hbm_basis = hbm_peak_gbs()
            roof.update({"hbm_achieved_gbs": hbm, "hbm_peak_gbs": hbm_peak, "hbm_frac": hbm / hbm_peak,
                         "hbm_peak_basis": hbm_basis})
        line = {
            "metric": METRIC if args.workload == DEFAULT_WORKLOAD else f"emulated MACs/s, {spec['desc']}",
            "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": value / PAGES_MACS_PER_S if args.workload == DEFAULT_WORKLOAD else None,
            "dtype": "f64", "data": "synthetic",
            "config": {"workload": spec["desc"], "name": args.workload, "emulated_arch": spec["model"],
                       "input_format": spec["fmt"], "global_batch": world,
                       "parallelism": f"independent x{world}", "l2": spec["l2"],
                       "workspace_cache": "on: mmaemu_set_workspace_cache(1) keeps the decoded-operand "
                                          "workspace between calls (the library default releases it)"},
            "verified": verified,
            "roofline": roof,
            "clocks": clocks,
            "e2e": {"value": macs * world / (e2e_ms / 1e3), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "verified": e2e_verified},
            "gpu_launches": launches_per_step * args.steps,
        }
        if world == 1 and not args.no_cpu_baseline and args.workload == DEFAULT_WORKLOAD:
            line["cpu_baseline"] = cpu_baseline(inputs=(A_np, B_np, C_np))
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.pipe_rates:
        return run_pipe_rates()
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
