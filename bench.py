"""Throughput of exact Lloyd's k-means on B200 through the C ABI (libfk.so).

A step is one fk_lloyd call: one complete k-means run of `niter` Lloyd iterations (cosine
normalisation once, then assign + sort + update per iteration) over the workload's N
synthetic points, starting from the same initial centroids every step.  The metric is
points x iterations per second for the whole job.

Default workload: N = 100,000,000 points, d = 128, K = 32,768, bf16 points with fp32
accumulation and fp32 centroid sums, 3 iterations: the d = 128, K = 32,768 shape of the
Flash-KMeans article's headline run (opening paragraph: 1e9 points on an H200), scaled to
one GPU's memory.  --workload selects the others (synth.CONFIGS), e.g. the LEANN FlashLib
guide's 1M x 768, nlist 4096 coarse-quantizer build (section "性能对比").

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Under torchrun (N > 1 ranks) the run is data-parallel: every rank holds N points of its own
(its own seed; per-GPU work is fixed, weak scaling), the centroids are replicated from
rank 0, and each iteration exchanges per-cluster sums and counts with NCCL all_gather
(exact_lloyd_means_b200.dist).  The whole-job value divides all ranks' points x
iterations by the slowest rank's device time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "points·iterations/sec per Lloyd iter (assign+update) on 1 B200; % of roofline"
UNIT = "points*iter/s"
# The pages' own figure for the default workload: a 1M x 768, nlist 4096 k-means build
# (default niter 20) in 10.6 s on an H200 (another machine; context only).
PAGES_BUILD_RATE = 1_000_000 * 20 / 10.6
L2_FLUSH_BYTES = 256 << 20  # twice the B200's 126 MB L2


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=5)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--workload", default=None,
                   help="one of synth.CONFIGS (default: large_100000000x128_k32768_bf16; "
                        "with --search, ivf_1000000x768_k4096_f32_cosine, the index workload)")
    p.add_argument("--niter", type=int, default=None)
    p.add_argument("--n", type=int, default=None,
                   help="override N (smaller cases for profiling captures)")
    p.add_argument("--k", type=int, default=None,
                   help="override K, the number of clusters (cells); with --n, a small case "
                        "of the same points per cell for profiling captures")
    p.add_argument("--impl", default="fk", choices=["fk", "reference"])
    p.add_argument("--dp", action="store_true",
                   help="run the data-parallel loop (exact_lloyd_means_b200.dist) even on "
                        "one rank")
    p.add_argument("--streamed", type=int, default=0, metavar="CHUNK_ROWS",
                   help="keep X in pinned host memory and stream it every iteration in "
                        "chunks of this many rows (fk_lloyd_streamed, the out-of-core mode)")
    p.add_argument("--search", type=int, default=0, metavar="NPROBE",
                   help="IVF-Flat search instead of k-means: build the index of the workload "
                        "(its Lloyd run, then the cell lists), then time searches of a "
                        "batch of --queries queries probing NPROBE cells for --topk "
                        "neighbours (fk_ivf_search)")
    p.add_argument("--queries", type=int, default=10000)
    p.add_argument("--topk", type=int, default=10)
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=12.0)
    return p.parse_args()


# ----------------------------------------------------------------------------- helpers


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16": p["bf16_tflops"],
                "bf16_sustained": p["bf16_tflops_sustained"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


def assign_traffic_record(workload):
    """DRAM bytes per assign launch from a committed ncu summary, if one was taken on the
    current kernel source and for this workload (else None)."""
    path = os.path.join(ROOT, "profiles", "assign_traffic.json")
    src = os.path.join(ROOT, "exact_lloyd_means_b200", "csrc", "assign_sm100.cu")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        recs = json.load(f).get("records", [])
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    for rec in recs:
        if rec.get("kernel_sha") == h and rec.get("workload") == workload:
            return rec
    return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while running."""

    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = str(uuid or "").lower().replace("gpu-", "")
        self.proc = None
        self.path = os.path.join("/tmp", f"fk_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            if self.uuid and self.uuid not in parts[1].lower():
                continue
            rows.append(parts)
        os.remove(self.path)
        if not rows:
            return None
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        mx = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[j] for r in rows for j in range(4)
                          if r[5 + j].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


def cpu_baseline(X_host, C0_host, metric, precision, seconds):
    """The oracle as it stands (fp64 C + OpenMP), timed on this host's cores on a bounded
    sample: one Lloyd iteration (assign against all K centroids, CSR, update, objective)
    over S sampled points.  Returns (points*iter/s, threads, description)."""
    import oracle

    def one(S):
        Xs = X_host[:S]
        t0 = time.perf_counter()
        Xd = oracle.normalize_rows(Xs) if metric == "cosine" else oracle._f64(Xs)
        C = oracle.normalize_rows(C0_host) if metric == "cosine" else oracle._f64(C0_host)
        C = oracle.round_bf16(C) if precision == "bf16" else C
        lab, _, _ = oracle.assign(Xd, C)
        oracle.csr(lab, C.shape[0])
        oracle.update(Xd, lab, C)
        oracle.objective(Xd, C, lab)
        return time.perf_counter() - t0

    S = 64
    t = one(S)
    while t < 1.0 and S < X_host.shape[0]:
        S = min(X_host.shape[0], S * 4)
        t = one(S)
    S2 = int(min(X_host.shape[0], max(S, S * seconds / max(t, 1e-9))))
    t2 = one(S2)
    return S2 / t2, oracle.threads(), f"one oracle Lloyd iteration over the first {S2} points"


# ----------------------------------------------------------------------------- arms


def _reference_threads(oracle, world):
    """Under torchrun (N > 1) only rank 0 runs the reference arm, but torchrun starts every
    rank with one OpenMP thread: give rank 0 the host's cores back."""
    if world > 1:
        oracle.set_threads(len(os.sched_getaffinity(0)))


def reference_arm(args, spec, rank, world):
    """The oracle timed on the host as the reference arm: each step is one Lloyd iteration
    over a bounded sample of the workload's points."""
    if rank != 0:
        return
    import numpy as np
    import torch

    import oracle
    _reference_threads(oracle, world)
    from synth import gaussian_mixture, init_indices
    # a sample large enough that the per-step fixed costs (centroid normalisation and
    # rounding) are small next to the per-point work, yet about a second of CPU per step
    S = int(max(256, min(65536, 2e10 // (spec.k * spec.d))))
    n_gen = 2 * max(S, spec.k)
    X, _, _ = gaussian_mixture(n_gen, spec.d, spec.k, centers=spec.centers, sigma=spec.sigma,
                               weights=spec.weights, zipf_s=spec.zipf_s, dtype=spec.dtype,
                               seed=spec.seed)
    idx = init_indices(n_gen, spec.k, spec.seed)
    C0 = X[idx].float().numpy()
    Xh = X[:S].double().numpy() if spec.dtype == "bf16" else X[:S].numpy()
    prec = "bf16" if spec.dtype == "bf16" else "f32"

    def step():
        Xd = oracle.normalize_rows(Xh) if spec.metric == "cosine" else oracle._f64(Xh)
        C = oracle.normalize_rows(C0) if spec.metric == "cosine" else oracle._f64(C0)
        C = oracle.round_bf16(C) if prec == "bf16" else C
        lab, _, _ = oracle.assign(Xd, C)
        oracle.csr(lab, C.shape[0])
        oracle.update(Xd, lab, C)
        oracle.objective(Xd, C, lab)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = S * args.steps / dt
    sample = f"one oracle Lloyd iteration over {S} points of the workload per step"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": spec.name, "N": spec.n, "d": spec.d, "K": spec.k,
                   "metric": spec.metric, "sample_points": S},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0}}), flush=True)


def fk_arm(args, spec, rank, world, dist):
    import torch

    from exact_lloyd_means_b200 import fk
    from synth import gaussian_mixture, init_indices

    dev = torch.device("cuda", torch.cuda.current_device())
    niter = args.niter or spec.niter
    sharded = world > 1 or args.dp
    # weak scaling: every rank holds spec.n points of its own, drawn from the one mixture
    # (shard = rank); one k-means problem over all world * spec.n points when sharded
    seed = spec.seed
    X, _, _ = gaussian_mixture(spec.n, spec.d, spec.k, centers=spec.centers, sigma=spec.sigma,
                               weights=spec.weights, zipf_s=spec.zipf_s, dtype=spec.dtype,
                               seed=seed, device=dev, shard=rank)
    C0 = X[init_indices(spec.n, spec.k, seed, device=dev)].float().contiguous()
    if world > 1:
        dist.broadcast(C0, src=0)  # replicated initial centroids: rank 0's choice
    C = torch.empty_like(C0)
    labels = torch.empty(spec.n, dtype=torch.int32, device=dev)
    counts = torch.empty(spec.k, dtype=torch.int32, device=dev)
    if sharded:
        from exact_lloyd_means_b200.dist import gpu_ops, lloyd_sharded
        ops = gpu_ops(spec.n, spec.d, spec.k, X.dtype, dev)
        Xn = torch.empty_like(X) if spec.metric == "cosine" else None
    else:
        ws = fk.workspace(spec.n, spec.d, spec.k, X.dtype, spec.metric, device=dev)
    torch.cuda.synchronize()

    def run(Xin, acc, mode=True):
        """One complete k-means run from raw points and C (in place).  With acc, fk_lloyd's
        timing is added into it: mode True times every phase, "kernel" only the
        assignment's tensor-core kernel (two events per iteration)."""
        if not sharded:
            objs, tm = fk.fk_lloyd(Xin, C, niter, labels, ws, metric=spec.metric,
                                   counts=counts, timing=mode if acc is not None else False)
            if acc is not None:
                for k in ("ms_setup", "ms_prep", "ms_assign", "ms_sort", "ms_update",
                          "ms_assign_mma", "mma_timed", "screened"):
                    acc[k] = acc.get(k, 0) + tm[k]
            return objs
        Xp = Xin
        if spec.metric == "cosine":  # normalise once per run, as fk_lloyd does
            fk.fk_normalize_rows(Xin, Xn)
            fk.fk_normalize_rows(C, C)
            Xp = Xn
        objs, _ = lloyd_sharded(Xp, C, niter, ops, timing=acc)
        return objs

    def step(acc, mode=True):
        C.copy_(C0)
        return run(X, acc, mode)

    # points smaller than L2 are flushed from it between timed steps (a buffer twice the
    # L2 written outside the steps' events); larger ones cannot stay in it
    e_bytes = 4 if spec.dtype == "f32" else 2
    x_bytes = spec.n * spec.d * e_bytes
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev) \
        if x_bytes < L2_FLUSH_BYTES else None

    # the timed steps time only the assignment kernel of each step's last iteration (the
    # roofline's launches; two events per step, so that they barely perturb the steps);
    # the per-phase breakdown comes from extra steps after the timed region.  The warm-up
    # steps make the same calls as the timed ones, so fk_lloyd's cached graph of them is
    # captured before the timed region.
    mode = True if sharded else "kernel_last"
    for _ in range(args.warmup):
        step({}, mode)

    uuid = None
    try:
        uuid = torch.cuda.get_device_properties(dev).uuid
    except Exception:
        pass
    sampler = ClockSampler(uuid)
    sampler.start()
    time.sleep(0.4)
    acc = {}
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = fk.launch_count()
    if flush is None:
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            objs = step(acc, mode)
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
    else:
        marks = []
        for _ in range(args.steps):
            flush.fill_(1)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            objs = step(acc, mode)
            b.record()
            marks.append((a, b))
        torch.cuda.synchronize()
        ms = sum(a.elapsed_time(b) for a, b in marks)
    launches = fk.launch_count() - launches0
    if dist:
        dist.barrier()
    clocks = sampler.stop()
    pacc, psteps = acc, args.steps
    if not sharded:  # the phase breakdown, from steps outside the timed region
        pacc, psteps = {}, max(1, min(args.steps, 3))
        for i in range(psteps + 2):  # two untimed calls first, as for the timed steps
            if flush is not None:
                flush.fill_(1)
            step(pacc if i >= 2 else {})
        torch.cuda.synchronize()
    if dist:
        t = torch.tensor([ms], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = t.item()

    pts_iter = spec.n * niter * args.steps * world
    value = pts_iter / (ms / 1e3)

    # roofline of the dominant kernel (the assignment's tensor-core kernel), from the
    # per-launch device times fk_lloyd recorded with CUDA events on this stream during the
    # timed steps (the sharded loop times the whole assignment with torch events)
    peaks = load_peaks()
    n_assign = niter * args.steps
    flops = 2.0 * spec.n * spec.k * spec.d
    # the whole assignment phase (every kernel of it), from the phase-timed steps
    phase_ms = acc["ms_assign"] / n_assign if sharded else pacc["ms_assign"] / (niter * psteps)
    if sharded:
        mma_ms, screened = phase_ms, None
        scr = spec.dtype == "f32" and spec.d >= 256 and spec.n >= 18944
    else:
        mma_ms, screened = acc["ms_assign_mma"] / max(1, acc["mma_timed"]), acc["screened"]
        scr = screened == n_assign
    # fp32 points: the screened route's main kernel runs one bf16 product per term (peak:
    # the bf16 peak); the three-product route runs three per useful product (bf16 / 3).
    # The assign launches run at the clocks the power cap allows for their own (partial)
    # tensor load, above the clock of the seconds-long cuBLAS loop behind the sustained
    # figure, so the burst figure is the denominator; both are reported.
    div = 3.0 if (spec.dtype == "f32" and not scr) else 1.0
    peak = peaks["bf16"] / div
    peak_sus = peaks["bf16_sustained"] / div
    if spec.dtype == "f32" and scr:
        kernel = "assign_pair_kernel screening pass (fp32 points, 1 bf16 product per term)"
        peak_note = (f"measured bf16 dense peak {peaks['bf16']} TFLOP/s, burst "
                     f"({peaks['source']}); the exact re-ranking and three-product pass for "
                     "the rows that need it are in assign_phase")
    elif spec.dtype == "f32":
        kernel = "assign kernel (fp32 points, 3 bf16 products per term)"
        peak_note = ("fp32 products as 3 bf16 tensor-core products: measured bf16 dense peak "
                     f"{peaks['bf16']} TFLOP/s (burst) / 3 ({peaks['source']})")
    else:
        kernel = "assign kernel (bf16 points, 1 bf16 product per term)"
        peak_note = f"measured bf16 dense peak {peaks['bf16']} TFLOP/s, burst ({peaks['source']})"
    achieved = flops / (mma_ms / 1e3) / 1e12
    trec = assign_traffic_record(spec.name)
    roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "traffic": trec["bytes_per_launch"] if trec else None,
            "kernel": kernel, "algorithmic_flops_per_launch": flops,
            "avg_launch_ms": mma_ms, "peak_note": peak_note,
            "launches_timed": n_assign if sharded else acc["mma_timed"],
            "launches_timed_note": "the assignment kernel of each timed step's last iteration"
                                   if not sharded else "every iteration's assignment",
            "frac_of_sustained": achieved / peak_sus,
            "assign_phase": {"ms_per_iteration": phase_ms,
                             "useful_tflops": flops / (phase_ms / 1e3) / 1e12,
                             "frac_of_bf16_peak": flops / (phase_ms / 1e3) / 1e12 / peaks["bf16"],
                             "screened_iterations": screened}}
    if sharded:  # the library's sort + update run inside fk_update_partial
        upd_ms = acc["ms_partial"] / n_assign
        phases = {k: acc[k] / args.steps for k in ("ms_assign", "ms_partial", "ms_exchange",
                                                    "ms_finalize")}
    else:
        upd_ms = (pacc["ms_sort"] + pacc["ms_update"]) / (niter * psteps)
        phases = {k: pacc[k] / psteps for k in ("ms_setup", "ms_prep", "ms_assign",
                                                 "ms_sort", "ms_update")}
        phases["steps"] = psteps
        phases["note"] = ("every phase timed with CUDA events in extra steps after the "
                          "timed region")
    upd_bytes = spec.n * spec.d * e_bytes + 24.0 * spec.n

    out = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
           "higher_is_better": True, "scaling": "weak",
           "vs_baseline": value / PAGES_BUILD_RATE
           if spec.name == "ivf_1000000x768_k4096_f32_cosine" and niter == 20 else None,
           "vs_baseline_note": "pages' 1M x 768 nlist 4096 build: 10.6 s for 20 iterations "
                               "on an H200 (another machine; context)",
           "dtype": spec.dtype, "data": "synthetic",
           "config": {"workload": spec.name, "N": spec.n, "d": spec.d, "K": spec.k,
                      "metric": spec.metric, "niter_per_step": niter,
                      "parallelism": f"dp{world}" if sharded else "single GPU",
                      "points_per_rank": spec.n,
                      "l2": (f"inputs larger than L2 (X = {x_bytes / 1e9:.2f} GB per rank)"
                             if flush is None else
                             f"X ({x_bytes / 1e9:.3f} GB) smaller than L2: a "
                             f"{L2_FLUSH_BYTES >> 20} MB buffer written between timed steps,"
                             " outside their CUDA events")},
           "roofline": roof,
           "update_hbm": {"achieved_gbs": upd_bytes / (upd_ms / 1e3) / 1e9,
                          "peak_gbs": peaks["hbm_gbs"],
                          "frac": upd_bytes / (upd_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                          "frac_of_8tbs_spec": upd_bytes / (upd_ms / 1e3) / 1e9 / 8000.0,
                          "avg_ms": upd_ms},
           "phase_ms_per_step": phases,
           "gpu_launches": launches, "final_objective": objs[-1],
           "clocks": clocks}

    # the inverted lists of the finished clustering (LEANN guide, "工作原理"): CSR offsets,
    # row ids in cell order and the points gathered in that order; HBM-bound, timed apart
    # from the Lloyd steps with CUDA events on this stream
    if not sharded:
        offs = torch.empty(spec.k + 1, dtype=torch.int32, device=dev)
        rids = torch.empty(spec.n, dtype=torch.int32, device=dev)
        Xl = torch.empty_like(X)
        for _ in range(2):
            fk.fk_ivf_lists(X, labels, spec.k, offs, rids, ws, X_lists=Xl)
        torch.cuda.synchronize()
        g0 = torch.cuda.Event(enable_timing=True)
        g1 = torch.cuda.Event(enable_timing=True)
        g0.record()
        for _ in range(5):
            fk.fk_ivf_lists(X, labels, spec.k, offs, rids, ws, X_lists=Xl)
        g1.record()
        torch.cuda.synchronize()
        ivf_ms = g0.elapsed_time(g1) / 5
        # algorithmic bytes: the rows read and written once, plus the sort's label, key and
        # id traffic (about 20 B per point per radix pass)
        passes = max(1, -(-max(1, (spec.k - 1).bit_length()) // 11))
        ivf_bytes = 2.0 * spec.n * spec.d * e_bytes + 20.0 * spec.n * passes
        out["ivf_lists"] = {"ms": ivf_ms, "achieved_gbs": ivf_bytes / (ivf_ms / 1e3) / 1e9,
                            "peak_gbs": peaks["hbm_gbs"],
                            "frac": ivf_bytes / (ivf_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                            "algorithmic_bytes": ivf_bytes}
        del Xl

    # end to end through the public API with host buffers
    if not args.no_e2e:
        Xh = torch.empty(X.shape, dtype=X.dtype, pin_memory=True)
        Xh.copy_(X)
        C0h = torch.empty(C0.shape, dtype=torch.float32, pin_memory=True)
        C0h.copy_(C0)
        labh = torch.empty(spec.n, dtype=torch.int32, pin_memory=True)
        Ch = torch.empty(C0.shape, dtype=torch.float32, pin_memory=True)
        Xd = torch.empty_like(X)
        ke = max(1, min(args.steps, 3))

        def e2e_step():
            Xd.copy_(Xh, non_blocking=True)
            C.copy_(C0h, non_blocking=True)
            run(Xd, None)
            if not sharded:
                labh.copy_(labels, non_blocking=True)
            Ch.copy_(C, non_blocking=True)
            torch.cuda.synchronize()

        for _ in range(2):  # the second identical call captures fk_lloyd's graph
            e2e_step()
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        f0.record()
        for _ in range(ke):
            e2e_step()
        f1.record()
        torch.cuda.synchronize()
        ems = f0.elapsed_time(f1)
        if dist:
            t = torch.tensor([ems], device=dev, dtype=torch.float64)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            ems = t.item()
        out["e2e"] = {"value": spec.n * niter * ke * world / (ems / 1e3), "unit": UNIT,
                      "h2d_bytes_per_step": X.numel() * X.element_size() + C0.numel() * 4,
                      "d2h_bytes_per_step": (0 if sharded else spec.n * 4) + C0.numel() * 4
                      + niter * 8,
                      "steps": ke}
        del Xh, Xd

    if not args.no_cpu_baseline and world == 1 and rank == 0:
        S = min(spec.n, 1 << 16)
        Xs = X[:S].cpu()
        Xs = Xs.double().numpy() if spec.dtype == "bf16" else Xs.numpy()
        v, cores, sample = cpu_baseline(Xs, C0.cpu().numpy(), spec.metric,
                                        "bf16" if spec.dtype == "bf16" else "f32",
                                        args.cpu_seconds)
        out["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                               "sample": sample, "host_nproc": os.cpu_count()}
    if rank == 0:
        print(json.dumps(out), flush=True)


def streamed_arm(args, spec, rank, world, dist):
    """X in pinned host memory, streamed every iteration (fk_lloyd_streamed).  One process,
    one GPU: the step is a complete k-means run; the value is points x iterations per second
    of device time, with the host-to-device rate it needed beside it."""
    import torch

    from exact_lloyd_means_b200 import fk
    from synth import gaussian_mixture, init_indices
    if world != 1:
        raise SystemExit("--streamed runs on one GPU")
    dev = torch.device("cuda", torch.cuda.current_device())
    niter = args.niter or spec.niter
    tdt = torch.bfloat16 if spec.dtype == "bf16" else torch.float32
    e_bytes = 2 if spec.dtype == "bf16" else 4
    Xh = torch.empty((spec.n, spec.d), dtype=tdt, pin_memory=True)
    # generate on the device in slices and park them in pinned host memory
    X, _, _ = gaussian_mixture(spec.n, spec.d, spec.k, centers=spec.centers, sigma=spec.sigma,
                               weights=spec.weights, zipf_s=spec.zipf_s, dtype=spec.dtype,
                               seed=spec.seed, device=dev)
    C0 = X[init_indices(spec.n, spec.k, spec.seed, device=dev)].float().contiguous()
    Xh.copy_(X)
    del X
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    # the pinned host-to-device copy rate of this machine, for context
    probe = torch.empty(1 << 28, dtype=torch.uint8, pin_memory=True)
    probe_d = torch.empty_like(probe, device=dev)
    h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    probe_d.copy_(probe, non_blocking=True)
    h0.record()
    for _ in range(4):
        probe_d.copy_(probe, non_blocking=True)
    h1.record()
    torch.cuda.synchronize()
    h2d_gbs = 4 * probe.numel() / (h0.elapsed_time(h1) / 1e3) / 1e9
    del probe, probe_d
    chunk = args.streamed
    ws = fk.streamed_workspace(chunk, spec.d, spec.k, tdt, spec.metric, device=dev)
    C = torch.empty_like(C0)

    def step():
        C.copy_(C0)
        return fk.fk_lloyd_streamed(Xh, C, niter, ws, chunk, metric=spec.metric)

    for _ in range(args.warmup):
        step()
    uuid = None
    try:
        uuid = torch.cuda.get_device_properties(dev).uuid
    except Exception:
        pass
    sampler = ClockSampler(uuid)
    sampler.start()
    time.sleep(0.4)
    torch.cuda.synchronize()
    launches0 = fk.launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        objs = step()
    e1.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = e0.elapsed_time(e1)
    value = spec.n * niter * args.steps / (ms / 1e3)
    need = spec.n * spec.d * e_bytes * niter * args.steps / (ms / 1e3) / 1e9
    print(json.dumps({
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": spec.dtype, "data": "synthetic",
        "config": {"workload": spec.name, "N": spec.n, "d": spec.d, "K": spec.k,
                   "metric": spec.metric, "niter_per_step": niter, "mode": "streamed",
                   "chunk_rows": chunk,
                   "l2": "X streamed from pinned host memory every iteration"},
        "streamed": {"h2d_gbs_used": need, "h2d_gbs_measured": h2d_gbs,
                     "frac_of_h2d": need / h2d_gbs,
                     "x_host_gb": spec.n * spec.d * e_bytes / 1e9},
        "gpu_launches": fk.launch_count() - launches0, "final_objective": objs[-1],
        "clocks": clocks}), flush=True)


SEARCH_UNIT = "queries/s"


def search_metric(nprobe, k):
    return f"queries/sec of IVF-Flat search (nprobe {nprobe}, top-{k}) on 1 B200"


def fp64_peak_tflops(peaks_path=None):
    """fp64 FMA peak of the B200 from its unit counts and clock: 148 SMs x 64 fp64 FMA lanes
    per SM per clock x 2 flops x the maximum SM clock (1965 MHz unless MEASURED_PEAKS.json
    records another)."""
    mhz = 1965.0
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            mhz = float(json.load(f).get("sm_max_mhz", mhz))
    return 148 * 64 * 2 * mhz * 1e6 / 1e12, mhz


def search_cpu_sample(spec, seconds, nq_cap, rank_seed=0):
    """The oracle's IVF-Flat search timed on this host's cores over a bounded query sample.
    The index it searches is the workload's mixture components as cells (the oracle cannot
    run the 20-iteration build of a million points in bounded time); cells of the same
    sizes make the same amount of work.  Returns (queries/s, threads, description, step)."""
    import numpy as np

    import oracle
    from synth import gaussian_mixture, mixture_queries
    X, comp, cen = gaussian_mixture(spec.n, spec.d, spec.k, centers=spec.centers,
                                    sigma=spec.sigma, weights=spec.weights,
                                    zipf_s=spec.zipf_s, dtype="f32", seed=spec.seed)
    labels = comp.numpy().astype(np.int32)
    Xd = oracle.normalize_rows(X) if spec.metric == "cosine" else oracle._f64(X)
    Cd = oracle.normalize_rows(cen) if spec.metric == "cosine" else oracle._f64(cen)
    del X
    Q = mixture_queries(nq_cap, spec.d, spec.k, centers=spec.centers, sigma=spec.sigma,
                        weights=spec.weights, zipf_s=spec.zipf_s, seed=spec.seed,
                        stream=1 + rank_seed)
    Qd = oracle.normalize_rows(Q) if spec.metric == "cosine" else oracle._f64(Q)

    def one(S, nprobe, k):
        t0 = time.perf_counter()
        oracle.ivf_search(Qd[:S], Cd, Xd, labels, nprobe, k)
        return time.perf_counter() - t0

    return Qd, one


def search_arm(args, spec, rank, world, dist):
    """IVF-Flat search over the index of the workload (LEANN guide, "性能对比": 1M x 768,
    nlist 4096, top-10, an nprobe sweep).  Each rank builds the same index (fk_lloyd, then
    fk_ivf_lists and fk_ivf_norms) and searches its own batch of queries: replicas, weak
    scaling.  A step is one fk_ivf_search call over the batch (cosine: with the query
    normalisation)."""
    import torch

    from exact_lloyd_means_b200 import fk
    from synth import gaussian_mixture, init_indices, mixture_queries

    dev = torch.device("cuda", torch.cuda.current_device())
    nprobe, k, nq = args.search, args.topk, args.queries
    X, _, _ = gaussian_mixture(spec.n, spec.d, spec.k, centers=spec.centers, sigma=spec.sigma,
                               weights=spec.weights, zipf_s=spec.zipf_s, dtype="f32",
                               seed=spec.seed, device=dev)
    C0 = X[init_indices(spec.n, spec.k, spec.seed, device=dev)].float().contiguous()
    index = fk.IvfFlatIndex.build(X, C0, args.niter or spec.niter, metric=spec.metric)
    del X
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    Q = mixture_queries(nq, spec.d, spec.k, centers=spec.centers, sigma=spec.sigma,
                        weights=spec.weights, zipf_s=spec.zipf_s, seed=spec.seed,
                        stream=1 + rank, device=dev)
    ws = fk.ivf_search_workspace(nq, spec.d, spec.k, spec.n, nprobe, k, device=dev)
    D = torch.empty((nq, k), dtype=torch.float32, device=dev)
    I = torch.empty((nq, k), dtype=torch.int32, device=dev)
    P = torch.empty((nq, nprobe), dtype=torch.int32, device=dev)

    def step(Qin, timing=None):
        index.search(Qin, k, nprobe, ws=ws, distances=D, ids=I, probes=P, timing=timing)

    for _ in range(args.warmup):
        step(Q)
    torch.cuda.synchronize()
    # work of one step: (query, point) distance evaluations of the fine pass
    sizes = (index.offsets[1:] - index.offsets[:-1]).long()
    evals = int(sizes[P.long()].sum().item())
    fine_flops = 2.0 * spec.d * evals
    coarse_flops = 2.0 * spec.d * nq * spec.k

    uuid = None
    try:
        uuid = torch.cuda.get_device_properties(dev).uuid
    except Exception:
        pass
    sampler = ClockSampler(uuid)
    sampler.start()
    time.sleep(0.4)
    acc = {}
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = fk.launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        tm = {}
        step(Q, tm)
        for key, v in tm.items():
            acc[key] = acc.get(key, 0.0) + v
    e1.record()
    torch.cuda.synchronize()
    launches = fk.launch_count() - launches0
    if dist:
        dist.barrier()
    clocks = sampler.stop()
    ms = e0.elapsed_time(e1)
    if dist:
        t = torch.tensor([ms], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = t.item()
    value = nq * args.steps * world / (ms / 1e3)
    phases = {key: v / args.steps for key, v in acc.items()}
    peak, mhz = fp64_peak_tflops()
    fine_tf = fine_flops / (phases["ms_fine"] / 1e3) / 1e12
    coarse_tf = coarse_flops / (phases["ms_coarse"] / 1e3) / 1e12
    out = {"metric": search_metric(nprobe, k), "value": value, "unit": SEARCH_UNIT,
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": f"ivf_search_{spec.n}x{spec.d}_nlist{spec.k}_nq{nq}"
                                  f"_nprobe{nprobe}_k{k}_{spec.metric}",
                      "N": spec.n, "d": spec.d, "nlist": spec.k, "queries": nq,
                      "nprobe": nprobe, "k": k, "metric": spec.metric,
                      "index": f"fk_lloyd {args.niter or spec.niter} iterations + "
                               "fk_ivf_lists + fk_ivf_norms, built before timing",
                      "l2": "cell-ordered points (N x d fp32) larger than L2; no flush"},
           "roofline": ({"bound": "tensor", "achieved": fine_tf,
                         "peak": load_peaks()["bf16"] / 3, "unit": "TFLOP/s",
                         "frac": fine_tf / (load_peaks()["bf16"] / 3), "traffic": None,
                         "kernel": "ivf_fine_scr_kernel (fine pass: three bf16 products per "
                                   "term on mma.m16n8k16, fp32 accumulation)",
                         "flops_per_launch": fine_flops, "avg_ms": phases["ms_fine"],
                         "peak_basis": "measured bf16 burst peak / 3 (a third of the tensor "
                                       "work is useful); mma.m16n8k16 bf16 measured alone "
                                       "at 550 TFLOP/s on this GPU"}
                        if phases.get("screened_fine") else
                        {"bound": "alu", "achieved": fine_tf, "peak": peak,
                         "unit": "TFLOP/s", "frac": fine_tf / peak, "traffic": None,
                         "kernel": "ivf_tile_kernel<true> (fine pass, fp64 mma.m8n8k4)",
                         "flops_per_launch": fine_flops, "avg_ms": phases["ms_fine"],
                         "peak_basis": f"148 SMs x 64 fp64 FMA/clk x 2 x {mhz:.0f} MHz"}),
           "fine_path": "tensor-core screening (three bf16 products) + fp64 re-ranking"
                        if phases.get("screened_fine") else "fp64",
           "coarse": {"path": "tensor-core screening + fp64 re-ranking"
                              if phases.get("screened_coarse") else "fp64",
                      "useful_tflops": coarse_tf, "flops": coarse_flops,
                      "avg_ms": phases["ms_coarse"],
                      "frac": coarse_tf / (load_peaks()["bf16"] if phases.get("screened_coarse")
                                           else peak),
                      "frac_of": "measured bf16 burst peak" if phases.get("screened_coarse")
                                 else "fp64 peak"},
           "distance_evals_per_query": evals / nq,
           "phase_ms_per_step": phases, "gpu_launches": launches, "clocks": clocks}

    if not args.no_e2e:
        Qh = torch.empty(Q.shape, dtype=torch.float32, pin_memory=True)
        Qh.copy_(Q)
        Dh = torch.empty(D.shape, dtype=torch.float32, pin_memory=True)
        Ih = torch.empty(I.shape, dtype=torch.int32, pin_memory=True)
        Qd = torch.empty_like(Q)
        ke = max(1, args.steps)

        def e2e_step():
            Qd.copy_(Qh, non_blocking=True)
            step(Qd)
            Dh.copy_(D, non_blocking=True)
            Ih.copy_(I, non_blocking=True)
            torch.cuda.synchronize()

        e2e_step()
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record()
        for _ in range(ke):
            e2e_step()
        f1.record()
        torch.cuda.synchronize()
        ems = f0.elapsed_time(f1)
        if dist:
            t = torch.tensor([ems], device=dev, dtype=torch.float64)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            ems = t.item()
        out["e2e"] = {"value": nq * ke * world / (ems / 1e3), "unit": SEARCH_UNIT,
                      "h2d_bytes_per_step": Q.numel() * 4,
                      "d2h_bytes_per_step": D.numel() * 4 + I.numel() * 4, "steps": ke}

    if not args.no_cpu_baseline and world == 1 and rank == 0:
        import oracle
        Qd, one = search_cpu_sample(spec, args.cpu_seconds, nq)
        S = 16
        t = one(S, nprobe, k)
        while t < 1.0 and S < nq:
            S = min(nq, S * 4)
            t = one(S, nprobe, k)
        S2 = int(min(nq, max(S, S * args.cpu_seconds / max(t, 1e-9))))
        t2 = one(S2, nprobe, k)
        out["cpu_baseline"] = {"value": S2 / t2, "unit": SEARCH_UNIT,
                               "cores": oracle.threads(), "kind": "oracle",
                               "sample": f"oracle IVF-Flat search of {S2} queries over the "
                                         "workload's mixture components as cells",
                               "host_nproc": os.cpu_count()}
    if rank == 0:
        print(json.dumps(out), flush=True)


def search_reference_arm(args, spec, rank, world):
    """The oracle's IVF-Flat search timed on the host as the reference arm: each step
    searches a bounded sample of the query batch."""
    if rank != 0:
        return
    import oracle
    _reference_threads(oracle, world)
    nprobe, k = args.search, args.topk
    Qd, one = search_cpu_sample(spec, args.cpu_seconds, args.queries)
    S = 16
    t = one(S, nprobe, k)
    while t < 0.5 and S < args.queries:
        S = min(args.queries, S * 2)
        t = one(S, nprobe, k)
    for _ in range(args.warmup):
        one(S, nprobe, k)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one(S, nprobe, k)
    dt = time.perf_counter() - t0
    value = S * args.steps / dt
    sample = (f"oracle IVF-Flat search of {S} of the {args.queries} queries per step, over "
              "the workload's mixture components as cells")
    print(json.dumps({
        "impl": "reference", "metric": search_metric(nprobe, k), "value": value,
        "unit": SEARCH_UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"ivf_search_{spec.n}x{spec.d}_nlist{spec.k}_nq{args.queries}"
                               f"_nprobe{nprobe}_k{k}_{spec.metric}",
                   "sample_queries": S},
        "cpu_baseline": {"value": value, "unit": SEARCH_UNIT, "cores": oracle.threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": SEARCH_UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0}}), flush=True)


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    from dataclasses import replace

    from synth import CONFIGS
    if args.workload is None:
        args.workload = ("ivf_1000000x768_k4096_f32_cosine" if args.search
                         else "large_100000000x128_k32768_bf16")
    spec = CONFIGS[args.workload]
    if args.n:
        spec = replace(spec, n=args.n, name=spec.name.replace(str(spec.n), str(args.n)))
    if args.k:
        spec = replace(spec, k=args.k, name=spec.name.replace(f"k{spec.k}", f"k{args.k}"))
    if args.impl == "reference":
        if args.search:
            search_reference_arm(args, spec, rank, world)
        else:
            reference_arm(args, spec, rank, world)
        return
    import torch
    dist = None
    if world > 1 or args.dp:
        import datetime

        import torch.distributed as tdist
        # NCCL prints its version banner on stdout when NCCL_DEBUG=VERSION; the bench's
        # stdout carries exactly one JSON line, so keep library banners off it
        if os.environ.get("NCCL_DEBUG", "").upper() == "VERSION":
            os.environ["NCCL_DEBUG"] = "WARN"
        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        if world == 1:  # --dp on one process: a one-rank group
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            os.environ.setdefault("MASTER_PORT", "29517")
            os.environ.setdefault("RANK", "0")
            os.environ.setdefault("WORLD_SIZE", "1")
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180))
        dist = tdist
    if args.search:
        search_arm(args, spec, rank, world, dist)
    elif args.streamed:
        streamed_arm(args, spec, rank, world, dist)
    else:
        fk_arm(args, spec, rank, world, dist)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
