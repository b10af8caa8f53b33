"""Benchmark: KS matmul throughput on B200 as a fraction of its roofline.

Workload (default): the seeded sweep of 258 KS patterns
(a, d in {1,...,64}; (b, c) in {(48,48),...,(256,256),(192,48),(256,64)};
a*b*d, a*c*d <= 16384) at batch 25088, in fp32 and in bf16 -- 516 runs.  It
stands in for the "600 KS patterns" of the KS-matmul abstract on the
taxoreview.com page, whose list the pages do not give.  One step is one
``ks_matmul`` launch per run (inputs resident in HBM, L2 flushed by a 256 MiB
write before every timed launch, each launch timed alone by CUDA events on its
stream).

Per run r: FLOPs_r = 2*N*a*b*c*d, bytes_r = s*(N*a*c*d + N*a*b*d + a*b*c*d),
roofline_r = min(P_peak, BW * FLOPs_r / bytes_r) with BW the measured HBM copy
bandwidth and P_peak the fp32 FMA peak for fp32 runs (measured in the same run
by the library's FMA-rate probe; 148 SMs x 128 lanes x 2 x 1965 MHz = 74.45
TFLOP/s derived, as a note), the TF32 tensor peak for TF32 runs (a torch
TF32 matmul timed in the same run) and the measured bf16 tensor peak for bf16
runs; frac_r = (FLOPs_r / t_r) / roofline_r.  ``value`` is the median of frac_r
over the runs.  One JSON line is printed (rank 0).

``--impl reference`` times the CPU oracle (the plain C loops under oracle/)
on a bounded sample of the same workload, in the same unit.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from kronecker_sparse_matrix_b200 import inputs  # noqa: E402

FP32_FMA_PEAK_TFLOPS = 148 * 128 * 2 * 1965e6 / 1e12  # 74.45: SMs x FP32 lanes x 2 flop x max SM clock (derived)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
METRIC = "KS matmul GFLOP/s and HBM GB/s at 1 B200 as fraction of roofline, pattern median"
L2_FLUSH_BYTES = 256 * 1024 * 1024


# ---------------------------------------------------------------------------- peaks
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return {"hbm_gbs": float(pk["hbm_gbs"]), "bf16_tflops": float(pk["bf16_tflops"]),
                "bf16_tflops_sustained": float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS, source="fallback")


def run_flops(p, n):
    a, b, c, d = p
    return 2.0 * n * a * b * c * d


def run_bytes(p, n, s):
    a, b, c, d = p
    return float(s) * (n * a * c * d + n * a * b * d + a * b * c * d)


def launches_per_call(p, n, dtype, variant):
    """Kernel launches one ks_matmul makes: the fp32 FMA path first writes a
    transposed copy of the values (one extra launch) when d % 8 == 0, b % 4 == 0,
    the product has >= 2^30 flop and the values fit in 64 MiB (the rule of
    ks_fma32.cu's launcher); every other path is a single kernel."""
    a, b, c, d = p
    nvals = a * b * c * d
    if variant == "fma" and dtype == "fp32" and d % 8 == 0 and b % 4 == 0 and 2 * n * nvals >= 2 ** 30 \
            and nvals * 4 <= (64 << 20):
        return 2
    return 1


def elem_bytes(dtype):
    return 2 if dtype == "bf16" else 4


def roofline_tflops(p, n, dtype, peaks):
    ai = run_flops(p, n) / run_bytes(p, n, elem_bytes(dtype))
    p_peak = {"fp32": peaks.get("fp32_fma_tflops", FP32_FMA_PEAK_TFLOPS),
              "tf32": peaks.get("tf32_tflops", peaks["bf16_tflops"] / 2),
              "bf16": peaks["bf16_tflops"]}[dtype]
    return min(p_peak, peaks["hbm_gbs"] * ai / 1e3)


def measure_fma_peak(dev, reps=5):
    """TFLOP/s of the library's FP32 FMA-rate probe (best of `reps` launches of
    about 3 ms, 4 blocks of 256 threads per SM), timed with CUDA events."""
    from kronecker_sparse_matrix_b200 import _lib
    lib = _lib.load()
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    blocks, iters = 4 * sms, 40000
    out = torch.empty(blocks, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    best = float("inf")
    for r in range(reps + 2):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        _lib.check(lib.ks_fma_rate_probe(out.data_ptr(), blocks, iters, stream.cuda_stream))
        e1.record(stream)
        e1.synchronize()
        if r >= 2:
            best = min(best, e0.elapsed_time(e1) / 1e3)
    return blocks * 256 * iters * 32 / best / 1e12


def measure_sgemm(dev, n=8192, reps=5):
    """TFLOP/s of a torch (cuBLAS) fp32 matmul n^3 on the CUDA cores (TF32
    off), best of `reps`: a lower bound for the FP32 FMA peak."""
    return measure_matmul(dev, n, reps, tf32=False)


def measure_tf32_peak(dev, n=8192, reps=5):
    """TFLOP/s of a torch (cuBLAS) fp32 matmul n^3 with TF32 tensor cores
    allowed, best of `reps`."""
    return measure_matmul(dev, n, reps, tf32=True)


def measure_matmul(dev, n, reps, tf32):
    a = torch.randn(n, n, device=dev)
    b = torch.randn(n, n, device=dev)
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = tf32
    try:
        stream = torch.cuda.current_stream(dev)
        best = float("inf")
        for r in range(reps + 2):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            torch.matmul(a, b)
            e1.record(stream)
            e1.synchronize()
            if r >= 2:
                best = min(best, e0.elapsed_time(e1) / 1e3)
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev
    del a, b
    return 2.0 * n ** 3 / best / 1e12


# ---------------------------------------------------------------------------- workloads
def workload_runs(name):
    """List of (label, pattern, batch, dtype, seed)."""
    if name == "sweep":
        pats = inputs.sweep_patterns()
        return [(f"sweep[{i}]", p, inputs.SWEEP_BATCH, dt, i) for dt in ("fp32", "bf16") for i, p in enumerate(pats)]
    if name == "sweep-fp32":
        return [(f"sweep[{i}]", p, inputs.SWEEP_BATCH, "fp32", i) for i, p in enumerate(inputs.sweep_patterns())]
    if name == "sweep-bf16":
        return [(f"sweep[{i}]", p, inputs.SWEEP_BATCH, "bf16", i) for i, p in enumerate(inputs.sweep_patterns())]
    if name == "sweep-tf32":
        return [(f"sweep[{i}]", p, inputs.SWEEP_BATCH, "tf32", i) for i, p in enumerate(inputs.sweep_patterns())]
    if name == "sweep-sample":  # every 32nd pattern in both dtypes: the sample ncu's DRAM counters are taken on
        pats = inputs.sweep_patterns()
        return [(f"sweep[{i}]", pats[i], inputs.SWEEP_BATCH, dt, i) for dt in ("fp32", "bf16")
                for i in range(0, len(pats), 32)]
    if name == "sweep-quick":  # every 8th pattern, for development only
        pats = inputs.sweep_patterns()
        return [(f"sweep[{i}]", pats[i], inputs.SWEEP_BATCH, dt, i) for dt in ("fp32", "bf16")
                for i in range(0, len(pats), 8)]
    if name.startswith("pattern:"):  # pattern:a,b,c,d:dtype[:batch] -- one run, seed 0
        parts = name.split(":")
        pat = tuple(int(v) for v in parts[1].split(","))
        batch = int(parts[3]) if len(parts) > 3 else inputs.SWEEP_BATCH
        return [(name, pat, batch, parts[2], 0)]
    if name == "vit":
        return [("vit", inputs.VIT_PATTERN, inputs.VIT_BATCH, "fp32", 0)]
    if name == "gpt2":
        return [("gpt2-fp32", inputs.GPT2_PATTERN, inputs.GPT2_BATCH, "fp32", 0),
                ("gpt2-bf16", inputs.GPT2_PATTERN, inputs.GPT2_BATCH, "bf16", 0)]
    raise ValueError(name)


WORKLOAD_TEXT = {
    "sweep": "seeded KS pattern sweep: 258 patterns x {fp32, bf16} = 516 runs, batch 25088 "
             "(a,d in {1,2,4,...,64}; (b,c) in {(48,48),(64,64),(96,96),(128,128),(192,192),(256,256),"
             "(192,48),(256,64)}; a*b*d, a*c*d <= 16384); X ~ N(0,1), values ~ N(0,1/c), seed = pattern index",
}


def torch_dtype(dt):
    return torch.float32 if dt in ("fp32", "tf32") else torch.bfloat16


def is_tf32(dt):
    return dt == "tf32"


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples during the timed region (every 200 ms)."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index, path=None):
        self.gpu_index = gpu_index
        self.path = path
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
            if self.path:
                with open(self.path, "w") as f:
                    f.write("\n".join(self.lines) + "\n")
        return False

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------- distributed
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(values, world, device):
    """Elementwise max over ranks of a list of floats (the per-run times)."""
    if world <= 1:
        return list(values)
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def rank_seed(seed, rank):
    """Weak scaling: rank r draws its own batch of rows (units are independent rows)."""
    return seed + 1_000_003 * rank


# ---------------------------------------------------------------------------- GPU arm
# Source files of each kernel family: a recorded ncu traffic figure stays
# valid only while these are unchanged.
FAMILY_SOURCES = {
    "fma-fp32": ["ks_fma32.cu", "ks_fma.cu", "ks_internal.h", "ks_epilogue.cuh"],
    "fma-bf16": ["ks_fma.cu", "ks_internal.h", "ks_epilogue.cuh"],
    "tc-bf16": ["ks_tc.cu", "ks_sm100.cuh", "ks_internal.h", "ks_epilogue.cuh"],
    "stream-fp32": ["ks_stream.cu", "ks_internal.h", "ks_epilogue.cuh"],
    "stream-bf16": ["ks_stream.cu", "ks_internal.h", "ks_epilogue.cuh"],
}


def kernel_source_hash(family):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "kronecker_sparse_matrix_b200", "csrc")
    for f in FAMILY_SOURCES.get(family, sorted(os.listdir(csrc))):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(variant_key):
    """Per-launch DRAM traffic of the dominant kernel from a committed ncu
    summary, or None when missing or taken on a different kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            tr = json.load(f)
    except (OSError, ValueError):
        return None
    ent = tr.get(variant_key)
    if not ent or ent.get("source_hash") != kernel_source_hash(variant_key):
        return None
    return ent


def gpu_arm(args, rank, world, local):
    import kronecker_sparse_matrix_b200 as ks

    dev = torch.device("cuda", local)
    peaks = load_peaks()
    runs = workload_runs(args.workload)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    results = []
    clock_path = None
    if args.save_clocks:
        clock_path = args.save_clocks if world == 1 else f"{args.save_clocks}.rank{rank}"

    # --- device-resident timing ------------------------------------------------
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(local, clock_path) as clocks:
        # the compute peaks of this device, measured in the same run; the FP32
        # peak is the larger of the library's FMA probe and cuBLAS's SGEMM
        peaks["fp32_fma_probe_tflops"] = measure_fma_peak(dev)
        peaks["fp32_sgemm_tflops"] = measure_sgemm(dev)
        peaks["fp32_fma_tflops"] = max(peaks["fp32_fma_probe_tflops"], peaks["fp32_sgemm_tflops"])
        peaks["tf32_tflops"] = measure_tf32_peak(dev)
        torch.cuda.synchronize(dev)
        barrier(world)
        for label, p, n, dt, seed in runs:
            f = inputs.factor_inputs(p, n, seed=rank_seed(seed, rank), dtype=torch_dtype(dt), device=dev)
            Y = torch.empty((n, inputs.out_features(p)), dtype=f.X.dtype, device=dev)
            tf32 = is_tf32(dt)
            variant = ks.plan(p, n, ks.ks_dtype_of(f.X, tf32))
            for _ in range(args.warmup):
                ks.matmul(f.X, f.values, p, out=Y, tf32=tf32)
            times = []
            for _ in range(args.steps):
                flush.zero_()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                ks.matmul(f.X, f.values, p, out=Y, tf32=tf32)
                e1.record(stream)
                e1.synchronize()
                times.append(e0.elapsed_time(e1) / 1e3)
            results.append({"label": label, "pattern": p, "batch": n, "dtype": dt, "variant": variant,
                            "times": times})
            del f, Y
        ks.sync_status()
    torch.cuda.synchronize(dev)
    barrier(world)

    # max over ranks, per run and step
    flat = [t for r in results for t in r["times"]]
    flat = max_over_ranks(flat, world, dev)
    k = 0
    for r in results:
        r["times"] = flat[k:k + args.steps]
        k += args.steps

    for r in results:
        p, n, dt = r["pattern"], r["batch"], r["dtype"]
        t = statistics.mean(r["times"])
        s = elem_bytes(dt)
        r["t"] = t
        r["flops"] = run_flops(p, n) * world
        r["bytes"] = run_bytes(p, n, s) * world
        r["roof_tflops"] = roofline_tflops(p, n, dt, peaks) * world
        r["tflops"] = r["flops"] / t / 1e12
        r["frac"] = r["tflops"] / r["roof_tflops"]

    # --- end to end through the public API with host buffers -------------------
    e2e = None
    if not args.no_e2e:
        e2e = e2e_measure(args, runs, rank, world, dev, peaks)

    return results, peaks, clocks.summary(), e2e


def e2e_measure(args, runs, rank, world, dev, peaks):
    """Same runs through the C-ABI call with host buffers (ks_matmul_host):
    every step copies X and values from pinned host memory to the device and Y
    back, inside the timed region."""
    import kronecker_sparse_matrix_b200 as ks

    steps = max(1, min(args.steps, args.e2e_steps))
    max_x = max(n * inputs.in_features(p) * elem_bytes(dt) for _, p, n, dt, _ in runs)
    max_y = max(n * inputs.out_features(p) * elem_bytes(dt) for _, p, n, dt, _ in runs)
    max_v = max(p[0] * p[1] * p[2] * p[3] * 4 for _, p, _, _, _ in runs)
    hx = torch.empty(max_x, dtype=torch.uint8, pin_memory=True)
    hy = torch.empty(max_y, dtype=torch.uint8, pin_memory=True)
    hv = torch.empty(max_v, dtype=torch.uint8, pin_memory=True)
    stream = torch.cuda.current_stream(dev)
    fracs = [[] for _ in runs]
    h2d = d2h = 0
    for ri, (label, p, n, dt, seed) in enumerate(runs):
        f = inputs.factor_inputs(p, n, seed=rank_seed(seed, rank), dtype=torch_dtype(dt), device=dev)
        es = f.X.element_size()
        xb, vb = f.X.numel() * es, f.values.numel() * es
        yb = n * inputs.out_features(p) * es
        hxv = hx[:xb].view(f.X.dtype).view(f.X.shape)
        hvv = hv[:vb].view(f.values.dtype).view(f.values.shape)
        hyv = hy[:yb].view(f.X.dtype).view(n, inputs.out_features(p))
        hxv.copy_(f.X)
        hvv.copy_(f.values)
        del f
        tf32 = is_tf32(dt)
        # warm-up once (untimed)
        ks.matmul_host(hxv, hvv, p, out=hyv, tf32=tf32)
        torch.cuda.synchronize(dev)
        for _ in range(steps):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            ks.matmul_host(hxv, hvv, p, out=hyv, tf32=tf32)  # H2D, product, D2H, pipelined by the library
            e1.record(stream)
            e1.synchronize()
            t = e0.elapsed_time(e1) / 1e3
            fracs[ri].append(t)
        h2d += xb + vb
        d2h += yb
    flat = max_over_ranks([t for fr in fracs for t in fr], world, dev)
    vals = []
    k = 0
    for (label, p, n, dt, seed), fr in zip(runs, fracs):
        t = statistics.mean(flat[k:k + len(fr)])
        k += len(fr)
        vals.append(run_flops(p, n) / t / 1e12 / roofline_tflops(p, n, dt, peaks))
    return {"value": statistics.median(vals), "unit": "fraction of roofline (median over runs)",
            "h2d_bytes_per_step": int(h2d * world), "d2h_bytes_per_step": int(d2h * world),
            "steps": steps, "note": "per run: ks_matmul_host on pinned host X, values and Y (the library copies "
                                    "X and values to the device and Y back, in row chunks whose copies overlap "
                                    "the products)"}


# ---------------------------------------------------------------------------- oracle (CPU) arm
def oracle_sample(runs, rows, seed_offset=0):
    """Time the CPU oracle on `rows` rows of every run; returns per-run seconds and flops."""
    import oracle

    oracle.build()
    out = []
    for label, p, n, dt, seed in runs:
        f = inputs.factor_inputs(p, rows, seed=seed + seed_offset, dtype=torch_dtype(dt), device="cpu")
        X = f.X.double().numpy()
        V = f.values.double().numpy()
        t0 = time.perf_counter()
        oracle.matmul(X, V, p)
        t = time.perf_counter() - t0
        out.append((p, dt, t, run_flops(p, rows)))
    return out, oracle.threads()


def oracle_fracs(samples, peaks, batch_for_roofline):
    fr = []
    for (p, dt, t, fl), n in zip(samples, batch_for_roofline):
        fr.append(fl / t / 1e12 / roofline_tflops(p, n, dt, peaks))
    return fr


def cpu_baseline(args, runs, peaks):
    rows = args.cpu_rows
    samples, cores = oracle_sample(runs, rows)
    fr = oracle_fracs(samples, peaks, [n for _, _, n, _, _ in runs])
    tot_t = sum(s[2] for s in samples)
    tot_f = sum(s[3] for s in samples)
    return {"value": statistics.median(fr), "unit": "fraction of roofline (median over runs)", "cores": cores,
            "kind": "oracle", "gflops": tot_f / tot_t / 1e9, "seconds": tot_t,
            "sample": f"{rows} rows of every run of the workload ({len(runs)} runs), oracle in fp64 on "
                      f"{cores} host threads; per-run throughput divided by that run's B200 roofline"}


def reference_arm(args, rank, world):
    if rank != 0:
        return None
    peaks = load_peaks()
    runs = workload_runs(args.workload)
    for _ in range(args.warmup):
        oracle_sample(runs[:4], 2)
    t_steps, fr_steps = [], []
    cores = 1
    for step in range(args.steps):
        samples, cores = oracle_sample(runs, args.ref_rows, seed_offset=step)
        t_steps.append(sum(s[2] for s in samples))
        fr_steps.append(oracle_fracs(samples, peaks, [n for _, _, n, _, _ in runs]))
    per_run = [statistics.mean(x) for x in zip(*fr_steps)]
    value = statistics.median(per_run)
    line = {"impl": "reference", "metric": METRIC, "value": value,
            "unit": "fraction of roofline (median over runs)", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(t_steps), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD_TEXT.get(args.workload, args.workload),
                       "sample_rows_per_run": args.ref_rows},
            "cpu_baseline": {"value": value, "unit": "fraction of roofline (median over runs)", "cores": cores,
                             "kind": "oracle",
                             "sample": f"{args.ref_rows} rows of every run per step, fp64 C loops"},
            "e2e": {"value": value, "unit": "fraction of roofline (median over runs)",
                    "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    return line


# ---------------------------------------------------------------------------- extra configs
def extra_configs(args, dev, peaks):
    """ViT / GPT-2 single factors and the butterfly chain, device-timed."""
    import kronecker_sparse_matrix_b200 as ks

    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def timed(fn, reps):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(reps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            e1.synchronize()
            ts.append(e0.elapsed_time(e1) / 1e3)
        return statistics.median(ts)

    out = {}
    for name, dt in [("vit", "fp32"), ("vit", "tf32"), ("gpt2", "fp32"), ("gpt2", "tf32"), ("gpt2", "bf16")]:
        f = getattr(inputs, name)(dtype=torch_dtype(dt), device=dev)
        p, n = f.pattern, f.batch
        tf32 = is_tf32(dt)
        Y = torch.empty((n, inputs.out_features(p)), dtype=f.X.dtype, device=dev)
        t = timed(lambda: ks.matmul(f.X, f.values, p, out=Y, tf32=tf32), args.steps)
        s = elem_bytes(dt)
        tf = run_flops(p, n) / t / 1e12
        roof = roofline_tflops(p, n, dt, peaks)
        bound = "hbm" if roof < (peaks["fp32_fma_tflops"] if dt == "fp32" else peaks[f"{dt}_tflops"]) else "compute"
        out[f"{name}-{dt}"] = {"pattern": list(p), "batch": n, "us": t * 1e6, "tflops": tf,
                               "gbs": run_bytes(p, n, s) / t / 1e9,
                               "frac": tf / roof, "bound": bound,
                               "variant": ks.plan(p, n, ks.ks_dtype_of(f.X, tf32))}
        del f, Y
    # the sweep in TF32 (fp32 buffers, tensor cores): median fraction of its roofline
    tf32_fr = []
    for label, p, n, dt, seed in workload_runs("sweep-tf32"):
        f = inputs.factor_inputs(p, n, seed=seed, device=dev)
        Y = torch.empty((n, inputs.out_features(p)), dtype=f.X.dtype, device=dev)
        t = timed(lambda: ks.matmul(f.X, f.values, p, out=Y, tf32=True), min(args.steps, 3))
        tf32_fr.append(run_flops(p, n) / t / 1e12 / roofline_tflops(p, n, "tf32", peaks))
        del f, Y
    out["sweep-tf32"] = {"runs": len(tf32_fr), "median_frac": statistics.median(tf32_fr),
                         "note": "the 258 sweep patterns with fp32 buffers on the TF32 tensor-core path; "
                                 "roofline min(TF32 peak, HBM x AI), all HBM-bound"}
    # fused epilogue: act(X K^T + bias) with GELU (tanh form), the MLP-up layer
    for name, dt in [("vit", "fp32"), ("gpt2", "bf16")]:
        f = getattr(inputs, name)(dtype=torch_dtype(dt), device=dev)
        p, n = f.pattern, f.batch
        bias = torch.randn(inputs.out_features(p), generator=torch.Generator(device=dev).manual_seed(2),
                           device=dev).to(f.X.dtype)
        Y = torch.empty((n, inputs.out_features(p)), dtype=f.X.dtype, device=dev)
        t = timed(lambda: ks.matmul(f.X, f.values, p, out=Y, bias=bias, act="gelu_tanh"), args.steps)
        tf = run_flops(p, n) / t / 1e12
        out[f"{name}-{dt}-bias-gelu"] = {"pattern": list(p), "batch": n, "us": t * 1e6, "tflops": tf,
                                         "frac": tf / roofline_tflops(p, n, dt, peaks)}
        del f, Y
    # KSLinear backward: dX = dY K (pattern (a, c, b, d), transposed blocks) and
    # dV (reduction over the batch); same flops and bytes as the forward product
    for name, dt in [("vit", "fp32"), ("gpt2", "fp32"), ("gpt2", "bf16")]:
        f = getattr(inputs, name)(dtype=torch_dtype(dt), device=dev)
        p, n = f.pattern, f.batch
        g = torch.Generator(device=dev).manual_seed(1)
        dy = torch.randn(n, inputs.out_features(p), generator=g, device=dev).to(f.X.dtype)
        roof = roofline_tflops(p, n, dt, peaks)
        for grad, fn in (("dx", lambda: ks.matmul_dx(dy, f.values, p)), ("dv", lambda: ks.matmul_dv(dy, f.X, p))):
            t = timed(fn, args.steps)
            tf = run_flops(p, n) / t / 1e12
            out[f"{name}-{dt}-{grad}"] = {"pattern": list(p), "batch": n, "us": t * 1e6, "tflops": tf,
                                          "frac": tf / roof}
        del f, dy
    # hierarchical butterfly factorization of a dense 4096 x 4096 product of
    # butterfly factors (the producer of the chain's factors)
    c = inputs.butterfly(device=dev)
    A = ks.chain(torch.eye(4096, device=dev), c.factors, c.patterns).t().contiguous()
    t = timed(lambda: ks.butterfly_factorize(A), args.steps)
    out["butterfly-factorize-4096-fp32"] = {"us": t * 1e6, "gbs": A.numel() * 4 / t / 1e9,
                                            "note": "rank-one fits of 4096 64x64 blocks at the top split, then "
                                                    "recursively; bytes = one read of A"}
    del A, c
    for dt in ("fp32", "bf16"):
        c = inputs.butterfly(device=dev, dtype=torch_dtype(dt))
        s = elem_bytes(dt)
        Y = torch.empty_like(c.X)
        vbytes = sum(p[0] * p[1] * p[2] * p[3] for p in c.patterns) * s
        for fused in (True, False):
            t = timed(lambda: ks.chain(c.X, c.factors, c.patterns, out=Y, fused=fused), args.steps)
            if fused:  # X once, Y once, every factor's values once
                byts = 2 * s * c.batch * c.X.shape[1] + vbytes
                note = "one fused kernel: X read once, Y written once"
            else:      # every factor's X and Y through HBM
                byts = sum(run_bytes(p, c.batch, s) for p in c.patterns)
                note = "12 launches, HBM round trip per factor"
            out[f"butterfly-chain-{dt}" + ("" if fused else "-unfused")] = {
                "factors": len(c.patterns), "batch": c.batch, "us": t * 1e6, "algorithmic_bytes": byts,
                "gbs": byts / t / 1e9, "frac": byts / t / 1e9 / peaks["hbm_gbs"], "note": note}
    return out


# ---------------------------------------------------------------------------- main
def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ks", "reference"], default="ks")
    ap.add_argument("--workload", default="sweep")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--no-extra", action="store_true")
    ap.add_argument("--cpu-rows", type=int, default=128)
    ap.add_argument("--ref-rows", type=int, default=32)
    ap.add_argument("--save-clocks", default=None, metavar="PATH",
                    help="also write the nvidia-smi clock samples of the timed region to PATH")
    ap.add_argument("--details", default=None, help="write per-run results as JSON here")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    if args.impl == "reference":
        # CPU only: rank 0 runs the oracle, the other ranks exit without work.
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        line = reference_arm(args, rank, world)
        if rank == 0:
            print(json.dumps(line), flush=True)
        return 0

    rank, world, local = dist_setup(args)
    try:

        if not torch.cuda.is_available():
            raise SystemExit("bench.py needs a CUDA device (the reference arm runs on CPU: --impl reference)")
        dev = torch.device("cuda", local)
        results, peaks, clocks, e2e = gpu_arm(args, rank, world, local)
        extra = extra_configs(args, dev, peaks) if (rank == 0 and not args.no_extra) else None
        if rank != 0:
            return 0
        fracs = [r["frac"] for r in results]
        value = statistics.median(fracs)
        per_dtype = {dt: statistics.median([r["frac"] for r in results if r["dtype"] == dt])
                     for dt in sorted({r["dtype"] for r in results})}
        ms_per_step = 1e3 * sum(r["t"] for r in results)
        tot_f = sum(r["flops"] for r in results)
        tot_b = sum(r["bytes"] for r in results)
        tot_t = sum(r["t"] for r in results)
        # dominant kernel: the (variant, dtype) family with the most device time
        fam = {}
        for r in results:
            key = f"{r['variant']}-{r['dtype']}"
            e = fam.setdefault(key, {"t": 0.0, "flops": 0.0, "bytes": 0.0, "n": 0})
            e["t"] += r["t"]
            e["flops"] += r["flops"]
            e["bytes"] += r["bytes"]
            e["n"] += 1
        dom_key = max(fam, key=lambda k: fam[k]["t"])
        dom = fam[dom_key]
        if dom_key.startswith("fma-fp32"):
            achieved = dom["flops"] / dom["t"] / 1e12
            pk = peaks["fp32_fma_tflops"]
            roof = {"bound": "alu", "achieved": achieved, "peak": pk, "unit": "TFLOP/s", "frac": achieved / pk,
                    "peak_source": "measured in this run: the larger of the library's FP32 FMA-rate probe "
                                   f"({peaks['fp32_fma_probe_tflops']:.2f}; fma.rn.f32x2 chains, CUDA events) and "
                                   f"cuBLAS SGEMM 8192^3 with TF32 off ({peaks['fp32_sgemm_tflops']:.2f}); "
                                   "derived 148 SMs x 128 lanes x 2 flop x 1965 MHz = "
                                   f"{FP32_FMA_PEAK_TFLOPS:.2f} TFLOP/s, frac against it "
                                   f"{achieved / FP32_FMA_PEAK_TFLOPS:.4f}"}
        elif dom_key.startswith("tc"):
            achieved = dom["bytes"] / dom["t"] / 1e9
            roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": achieved / peaks["hbm_gbs"], "peak_source": f"{peaks['source']} HBM copy bandwidth"}
        else:
            achieved = dom["bytes"] / dom["t"] / 1e9
            roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": achieved / peaks["hbm_gbs"], "peak_source": f"{peaks['source']} HBM copy bandwidth"}
        roof["kernel"] = dom_key
        roof["launches"] = dom["n"]
        tr = ncu_traffic(dom_key)
        roof["traffic"] = tr["bytes_per_launch"] if tr else None
        if tr:
            roof["traffic_note"] = (f"ncu DRAM read+write per launch, mean over the family's {tr['launches']} sweep "
                                    f"launches; algorithmic bytes per launch {tr['algorithmic_bytes_per_launch']:.4g} "
                                    f"(profiles/traffic.json)")
        roof["note"] = ("achieved = algorithmic flops (or bytes) summed over that family's launches / summed "
                        "CUDA-event launch time")
        line = {
            "metric": METRIC, "value": value, "unit": "fraction of roofline (median over runs)",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32+bf16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD_TEXT.get(args.workload, args.workload), "runs": len(results),
                       "batch_per_gpu": results[0]["batch"], "l2": "flushed by a 256 MiB write before every timed launch",
                       "parallelism": f"dp{world} (rows sharded, no collective)" if world > 1 else "single GPU"},
            "median_frac_by_dtype": per_dtype,
            "aggregate": {"tflops": tot_f / tot_t / 1e12, "gbs": tot_b / tot_t / 1e9},
            "roofline": roof,
            "cpu_baseline": cpu_baseline(args, workload_runs(args.workload), peaks) if world == 1 else None,
            "e2e": e2e,
            "gpu_launches": args.steps * sum(launches_per_call(r["pattern"], r["batch"], r["dtype"], r["variant"])
                                             for r in results),
            "clocks": clocks,
            "peaks": {"hbm_gbs": peaks["hbm_gbs"], "bf16_tflops": peaks["bf16_tflops"],
                      "fp32_fma_tflops": peaks["fp32_fma_tflops"], "fp32_fma_probe_tflops": peaks["fp32_fma_probe_tflops"],
                      "fp32_sgemm_tflops": peaks["fp32_sgemm_tflops"], "fp32_fma_tflops_derived": FP32_FMA_PEAK_TFLOPS,
                      "tf32_tflops": peaks["tf32_tflops"],
                      "fp32_fma_flop_per_sm_clock": (peaks["fp32_fma_tflops"] * 1e12 / 148 /
                                                     (clocks["sm_mhz"] * 1e6)) if clocks.get("sm_mhz") else None,
                      "source": f"HBM and bf16: {peaks['source']} (MEASURED_PEAKS.json); FP32 FMA and TF32: "
                                "measured in this run"},
            "extra": extra,
        }
        if args.details:
            with open(args.details, "w") as f:
                json.dump({"results": [{k: v for k, v in r.items()} for r in results], "line": line}, f, indent=1)
        print(json.dumps(line), flush=True)
        return 0
    finally:
        if world > 1:
            import torch.distributed as dist
            if dist.is_initialized():
                dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
