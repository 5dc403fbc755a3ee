"""Benchmark: exact batched Lloyd's K-Means on B200 through libfk.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fk|reference]

Workload (the API shape of the flash-kmeans functional example): B=32
independent problems, N=75600 points, d=128, K=1000 centroids, fp16 points
~ N(0, 1) i.i.d., initial centroids = a seeded index set of points, up to 20
Lloyd iterations with tol = 1e-4 on the max centroid shift.

One step = one fk_lloyd call (the whole hot path: FlashAssign, counting sort,
segment reduce, finalize, tol check) on device-resident points.  value = Lloyd
iterations per second over all ranks (each rank runs its own B=32 problem:
weak scaling, no data-path collective).  The points (619 MB) exceed the 126 MB
L2, so no flush is needed between steps.

Also reported: the FlashAssign kernel's achieved TFLOP/s against the measured
tensor peak (CUDA events around every launch, on the launching stream), the
update's GB/s against measured HBM bandwidth, the end-to-end rate through the
C ABI with pinned host buffers (host->device copy of the points and
device->host copy of ids and centroids inside every step), SM clocks sampled
during the timed region, and the fp64 CPU checker timed on a bounded sample.

--impl reference times that checker as the reference arm (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "api"
# a timed region at least this long is compared with the sustained tensor
# peak (measured over a seconds-long loop), a shorter one with the burst peak
SUSTAINED_REGION_MS = 2000.0
METRIC = "Lloyd iter/s at B32·N75600·K1000·d128 fp16; assign TFLOP/s; update GB/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def env_int(name, default):
    try:
        return int(os.environ.get(name, default))
    except ValueError:
        return default


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash():
    """Hash of the FlashAssign kernel's own sources (the kernel file, the sm_100
    PTX layer, the norm-row arithmetic) and of the constants it takes from the
    internal header, so host-side declarations there do not count as a change."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "clustering_flashassign_b200", "csrc")
    for name in ["fk_assign_tc.cu", "fk_assign_common.cuh", "fk_sm100.cuh", "fk_norms.cuh"]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    with open(os.path.join(csrc, "fk_internal.h")) as f:
        consts = [ln for ln in f if re.match(r"\s*(constexpr|enum|inline)\b", ln)]
    h.update("".join(consts).encode())
    return h.hexdigest()[:16]


def recorded_traffic():
    """DRAM bytes per FlashAssign launch from the committed ncu summary, if it
    was taken on the current kernel source (its hash is recorded there)."""
    p = os.path.join(ROOT, "profiles", "flash_assign_api.md")
    if not os.path.exists(p):
        return None
    txt = open(p).read()
    m_hash = re.search(r"kernel source hash:\s*([0-9a-f]{16})", txt)
    m_bytes = re.search(r"dram bytes per full launch:\s*([0-9.eE+]+)", txt)
    if not m_hash or not m_bytes or m_hash.group(1) != kernel_source_hash():
        return None
    return float(m_bytes.group(1))


class ClockSampler:
    """SM clock and throttle-reason samples (NVML, every 20 ms) during the timed
    region; the nvidia-smi query loop is the fallback when NVML is missing."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
            "hw_thermal_slowdown": 0x40}

    def __init__(self, gpu_index, period_s=0.02):
        self.idx = gpu_index
        self.period = period_s
        self.rows = []
        self.nvml = None
        self.thread = None
        self.stop = False
        self.proc = None
        self.path = None

    def _loop(self, h):
        import pynvml
        while not self.stop:
            try:
                sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
                rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.rows.append((float(sm), float(mx), int(rs)))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        try:
            import threading

            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.idx)
            self.nvml = pynvml
            self.thread = threading.Thread(target=self._loop, args=(h,), daemon=True)
            self.thread.start()
            return self
        except Exception:
            self.nvml = None
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.thread is not None:
            self.stop = True
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def _smi_rows(self):
        rows = []
        if not self.path or not os.path.exists(self.path):
            return rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                bits = 0
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        bits |= self.BITS[n]
                rows.append((float(parts[1]), float(parts[2]), bits))
            except ValueError:
                continue
        os.unlink(self.path)
        return rows

    def summary(self):
        rows = self.rows if self.nvml is not None else self._smi_rows()
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        loaded = [r for r in rows if r[0] > 0.5 * r[1]] or rows
        reasons = sorted({n for r in rows for n, bit in self.BITS.items() if r[2] & bit})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows),
                "source": "nvml" if self.nvml is not None else "nvidia-smi"}


def metric_for(w):
    if w.name == WORKLOAD:
        return METRIC
    return f"Lloyd iter/s at B{w.B}·N{w.N}·K{w.K}·d{w.d} {w.dtype}; assign TFLOP/s; update GB/s"


def rank_workload(rank, name=WORKLOAD, **overrides):
    """The workload of one rank: the same shape on every rank, its own seeds
    (weak scaling over independent problems: ranks share no data)."""
    import synthdata
    w = synthdata.WORKLOADS[name]
    return synthdata.scaled(w, seed=w.seed + 7919 * rank, init_seed=w.init_seed + 100 * rank, **overrides)


def make_inputs(rank, name=WORKLOAD):
    import synthdata
    w = rank_workload(rank, name)
    x, idx, init = synthdata.make(w)
    return w, x, init


def reduce_over_ranks(dist, device, to_max, to_sum):
    """(element-wise max of to_max, element-wise sum of to_sum) over all ranks;
    the identity without a process group.  Every rank must call it."""
    if dist is None:
        return [float(v) for v in to_max], [float(v) for v in to_sum]
    import torch
    tmax = torch.tensor([float(v) for v in to_max], dtype=torch.float64, device=device)
    tsum = torch.tensor([float(v) for v in to_sum], dtype=torch.float64, device=device)
    dist.all_reduce(tmax, op=dist.ReduceOp.MAX)
    dist.all_reduce(tsum, op=dist.ReduceOp.SUM)
    return [float(v) for v in tmax.tolist()], [float(v) for v in tsum.tolist()]


# distance terms (points x centroids x d) the CPU sample may cover: about
# 2-3 s of the fp64 checker on 16 cores; the one-thread sample about 2 s
CPU_SAMPLE_TERMS = 4e10
CPU_SAMPLE_TERMS_1T = 2e9


def host_info():
    """The host the CPU baseline ran on: logical CPUs, the ones this process
    may use, and the CPU model."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        usable = len(os.sched_getaffinity(0))
    except AttributeError:
        usable = os.cpu_count()
    return {"nproc": usable, "logical_cpus": os.cpu_count(), "cpu_model": model}


def cpu_sample_points(w, batches):
    """Points per batch of the CPU sample: all of them, or a prefix when the
    sample would exceed CPU_SAMPLE_TERMS."""
    terms = batches * w.N * w.K * w.d
    if terms <= CPU_SAMPLE_TERMS:
        return w.N
    return max(min(w.N, 1024), int(w.N * CPU_SAMPLE_TERMS / terms))


def cpu_oracle_sample(x, init, w, batches, threads=0, points=None):
    """One Lloyd iteration of the fp64 checker on `batches` of the workload
    (the first `points` points of each, all by default)."""
    import numpy as np

    import oracle
    import synthdata
    xs = np.ascontiguousarray(x[:batches, :points] if points else x[:batches])
    c = synthdata.to_f64(init[:batches], w.dtype)
    t0 = time.perf_counter()
    chat = oracle.round_to(c, w.dtype)
    ids, _, _ = oracle.assign(xs, w.dtype, chat, nthreads=threads)
    oracle.update(xs, w.dtype, ids, c)
    return time.perf_counter() - t0


def run_reference(args, rank):
    """Reference arm: the fp64 CPU checker on a bounded sample (rank 0 only)."""
    if rank != 0:
        return
    import oracle
    w, x, init = make_inputs(0)
    batches = 1
    for _ in range(args.warmup):
        cpu_oracle_sample(x, init, w, batches)
    times = [cpu_oracle_sample(x, init, w, batches) for _ in range(args.steps)]
    t = sum(times) / len(times)
    value = 1.0 / (t * w.B / batches)
    cores = oracle.max_threads()
    sample = (f"one Lloyd iteration (assign + update) of {batches} of the {w.B} batches per step, "
              f"extrapolated linearly to all {w.B}")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "iter/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{WORKLOAD}: B={w.B} N={w.N} K={w.K} d={w.d} {w.dtype}",
                       "parallelism": "host threads"},
            "cpu_baseline": {"value": value, "unit": "iter/s", "cores": cores, "kind": "oracle",
                             "sample": sample, **host_info()},
            "e2e": {"value": value, "unit": "iter/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_fk(args, rank, world, local_rank, dist):
    import numpy as np
    import torch

    import clustering_flashassign_b200 as fk

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w, x, init = make_inputs(rank, args.workload)

    def as_torch(a):  # bf16 arrays are stored as uint16 bit patterns
        t = torch.from_numpy(a)
        return t.view(torch.bfloat16) if w.dtype == "bf16" else t

    xd = as_torch(x).to(dev)
    initd = as_torch(init).to(dev)
    ids = torch.empty((w.B, w.N), dtype=torch.int32, device=dev)
    centers = torch.empty((w.B, w.K, w.d), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        return fk.fk_lloyd(xd, initd, w.iters, w.tol, ids, centers)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()

    fk.fk_profile_read(reset=True)
    fk.fk_profile_enable(2)  # events around every assign and every whole update only
    launches0 = fk.fk_launch_count()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    iters_total = 0
    with ClockSampler(local_rank) as clk:
        torch.cuda.synchronize(dev)
        if dist is not None:
            dist.barrier()
        start.record(stream)
        for _ in range(args.steps):
            iters_total += step()
        stop.record(stream)
        torch.cuda.synchronize(dev)
        if dist is not None:
            dist.barrier()
    fk.fk_profile_enable(False)
    prof = fk.fk_profile_read(reset=True)
    launches = fk.fk_launch_count() - launches0
    ms = start.elapsed_time(stop)
    clocks = clk.summary()
    # the update's split into sort / reduce / finalize: one more step with an
    # event pair around every phase (outside the timed region)
    fk.fk_profile_enable(1)
    step()
    fk.fk_profile_enable(False)
    split = fk.fk_profile_read(reset=True)

    (ms_max,), (iters_all,) = reduce_over_ranks(dist, dev, [ms], [iters_total])

    # end to end through the C ABI with pinned host buffers
    xh = as_torch(x).pin_memory()
    inith = as_torch(init).pin_memory()
    idsh = torch.empty((w.B, w.N), dtype=torch.int32).pin_memory()
    cenh = torch.empty((w.B, w.K, w.d), dtype=torch.float32).pin_memory()

    def e2e_step():
        return fk.fk_lloyd(xh, inith, w.iters, w.tol, idsh, cenh, host_mode=fk.FK_HOST_RESIDENT)

    e2e_step()
    e_steps = max(1, min(args.steps, 5))
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_iters = 0
    e0.record(stream)
    for _ in range(e_steps):
        e_iters += e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e_ms = e0.elapsed_time(e1)
    (e_ms,), (e_iters,) = reduce_over_ranks(dist, dev, [e_ms], [e_iters])
    h2d = x.nbytes + init.nbytes
    d2h = w.B * w.N * 4 + w.B * w.K * w.d * 4

    if rank != 0:
        return

    peaks, src = load_peaks()
    flop = 2.0 * w.B * w.N * w.K * w.d
    a_ms = prof["assign_ms"] / max(1, prof["assign_launches"])
    achieved = flop / (a_ms * 1e-3) / 1e12
    tf32 = w.dtype == "f32" and w.d % 4 == 0 and w.K * w.d >= 16384
    peak_pair = {}
    if tf32:
        # fp32 on the tensor cores, 3xTF32: three tf32 passes per algorithmic flop;
        # the peak is a cuBLAS tf32 GEMM measured here (burst)
        peak_t = measure_tf32_tflops(dev)
        bound, kname = "tensor", "FlashAssign kind::tf32, 3 passes (k_flash_assign<float>)"
        psrc = ("measured here: cuBLAS tf32 GEMM 8192^3, best of 10 (burst); the 3xTF32 split runs 3 tensor "
                "passes per algorithmic flop, so 1/3 is the attainable fraction")
    elif w.dtype == "f32":
        # fp32 inputs take the SIMT kernel: peak from unit counts and the max clock
        mhz = float(peaks.get("sm_max_mhz", 1965.0))
        peak_t = 148 * 128 * 2 * mhz * 1e6 / 1e12
        bound, kname = "alu", "fp32 SIMT assign (k_assign_f32)"
        psrc = f"derived: 148 SMs x 128 fp32 lanes x 2 flop x {mhz:.0f} MHz"
    else:
        # fp16 runs at the bf16 rate.  The burst peak is the one for a timed
        # region shorter than the seconds-long loop the sustained figure comes
        # from; both fractions are reported.
        burst = float(peaks["bf16_tflops"])
        sustained = float(peaks.get("bf16_tflops_sustained") or burst)
        long_region = ms_max >= SUSTAINED_REGION_MS
        peak_t = sustained if long_region else burst
        bound, kname = "tensor", "FlashAssign (k_flash_assign)"
        psrc = (f"{src} bf16 dense, {'sustained' if long_region else 'burst'} (timed region "
                f"{ms_max / 1e3:.2f} s; the sustained figure applies from {SUSTAINED_REGION_MS / 1e3:.0f} s)")
        peak_pair = {"peak_burst": burst, "frac_burst": achieved / burst,
                     "peak_sustained": sustained, "frac_sustained": achieved / sustained}
    traffic = recorded_traffic() if w.name == WORKLOAD else None
    s = 2 if w.dtype != "f32" else 4
    upd_bytes = (w.B * w.N * w.d * s + 8 * w.B * w.N + 8 * w.B * w.N + 16 * w.B * w.K * w.d
                 + 2 * w.B * w.K * w.d + 12 * w.B * w.K)
    upd_ms = prof["update_ms"] / max(1, prof["update_calls"])
    upd_gbs = upd_bytes / (upd_ms * 1e-3) / 1e9
    hbm = float(peaks["hbm_gbs"])

    import oracle
    cores = oracle.max_threads()  # before the one-thread sample changes the thread count
    batches = min(4, w.B)
    pts = cpu_sample_points(w, batches)
    cpu_t = cpu_oracle_sample(x, init, w, batches, points=pts)
    cpu_value = 1.0 / (cpu_t * (w.B / batches) * (w.N / pts))
    # the same checker on one thread, on a smaller prefix of one batch
    pts1 = max(256, min(w.N, int(CPU_SAMPLE_TERMS_1T / (w.K * w.d))))
    cpu_t1 = cpu_oracle_sample(x, init, w, 1, threads=1, points=pts1)
    cpu_value_1t = 1.0 / (cpu_t1 * w.B * (w.N / pts1))

    others = None
    if w.name == WORKLOAD and not args.no_workloads:
        others = {name: time_workload(name, dev) for name in OTHER_WORKLOADS}

    baselines = None
    if w.name == WORKLOAD and not args.no_baselines:
        # the pages' two comparison kernels (materialised distances, scatter
        # atomics), timed after the bench's own region on this rank's inputs
        baselines = time_baselines(xd, initd, 5)

    line = {
        "metric": metric_for(w),
        "value": iters_all / (ms_max * 1e-3),
        "unit": "iter/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": max(args.warmup, 3),
        "ms_per_step": ms_max / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic",
        "config": {"workload": f"{w.name}: B={w.B} N={w.N} K={w.K} d={w.d} {w.dtype} "
                               + ("points ~ N(0,1), " if w.n_comp <= 1 else f"{w.n_comp}-component mixture, ")
                               + f"{w.iters} iterations max, tol={w.tol}",
                   "B": w.B, "N": w.N, "K": w.K, "d": w.d, "iterations_per_rank": iters_total,
                   "l2": (f"inputs larger than L2 (points {x.nbytes / 1e6:.0f} MB per rank)" if x.nbytes > 126e6
                          else f"points {x.nbytes / 1e6:.0f} MB per rank (fit in L2)"),
                   "parallelism": f"independent problems, {world} rank(s)"},
        "roofline": {"bound": bound, "achieved": achieved, "peak": peak_t, "unit": "TFLOP/s",
                     "frac": achieved / peak_t, "traffic": traffic,
                     "kernel": kname, "ms_per_launch": a_ms, "peak_source": psrc, **peak_pair},
        "kernels": {"assign_tflops": achieved, "assign_frac": achieved / peak_t,
                    "update_gbs": upd_gbs, "update_frac_of_hbm": upd_gbs / hbm,
                    "update_ms": upd_ms, "sort_ms": split["sort_ms"] / max(1, split["update_calls"]),
                    "reduce_ms": split["reduce_ms"] / max(1, split["update_calls"]),
                    "finalize_ms": split["finalize_ms"] / max(1, split["update_calls"]),
                    "split_from": "one extra step with an event pair around every phase",
                    "hbm_peak_gbs": hbm},
        "cpu_baseline": {"value": cpu_value, "unit": "iter/s", "cores": cores, "kind": "oracle",
                         "sample": (f"one Lloyd iteration of {batches} of {w.B} batches, extrapolated"
                                    if pts == w.N else
                                    f"one Lloyd iteration on the first {pts} of {w.N} points of {batches} "
                                    f"of {w.B} batches, extrapolated x{w.B * w.N / (batches * pts):.1f}"),
                         "one_thread": {"value": cpu_value_1t, "unit": "iter/s", "cores": 1,
                                        "sample": f"one Lloyd iteration on the first {pts1} of {w.N} points "
                                                  f"of one batch, extrapolated x{w.B * w.N / pts1:.1f}"},
                         **host_info()},
        "e2e": {"value": e_iters / (e_ms * 1e-3), "unit": "iter/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        "clocks": clocks,
    }
    if baselines is not None:
        line["baselines"] = baselines
    if others is not None:
        line["workloads"] = others
    print(json.dumps(line), flush=True)


def run_largen(args):
    """The large-N streamed workload (B=1, N=2^28, K=32768, d=128, fp16 mixture,
    64 GiB of points in pinned host memory), 3 Lloyd iterations per step.  The
    points are re-streamed every iteration in 2^24-point chunks whose copies
    overlap the compute.  Reports iterations/s, the effective and the measured
    peak pinned host-to-device bandwidth, and the ideal iteration time
    max(tensor time, copy time) against the measured one."""
    import numpy as np
    import torch

    import clustering_flashassign_b200 as fk
    import oracle
    import synthdata
    w = synthdata.WORKLOADS["largen"]
    if args.points:
        w = synthdata.scaled(w, N=args.points)
    t0 = time.perf_counter()
    xt = torch.empty((w.B, w.N, w.d), dtype=torch.float16, pin_memory=True)
    _, _, init = synthdata.make(w, out=xt.numpy())
    gen_s = time.perf_counter() - t0
    dev = torch.device("cuda", 0)
    initd = torch.from_numpy(init).to(dev)
    ids = torch.empty((w.B, w.N), dtype=torch.int32, device=dev)
    cen = torch.empty((w.B, w.K, w.d), dtype=torch.float32, device=dev)

    # pinned host -> device copy peak (one 2^24-point chunk, best of 3)
    chunk = min(w.N, 1 << 24)
    dst = torch.empty((chunk, w.d), dtype=torch.float16, device=dev)
    src = xt[0, :chunk]
    best = 1e30
    for _ in range(3):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        dst.copy_(src, non_blocking=True)
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    h2d_peak = chunk * w.d * 2 / (best * 1e-3) / 1e9
    del dst

    fk.fk_lloyd(xt, initd, 1, 0.0, ids, cen, host_mode=fk.FK_HOST_STREAM)  # warm-up (workspace)
    torch.cuda.synchronize()
    fk.fk_profile_read(reset=True)
    fk.fk_profile_enable(True)
    launches0 = fk.fk_launch_count()
    iters = 0
    with ClockSampler(0) as clk:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            iters += fk.fk_lloyd(xt, initd, w.iters, 0.0, ids, cen, host_mode=fk.FK_HOST_STREAM)
        e1.record()
        torch.cuda.synchronize()
    fk.fk_profile_enable(False)
    prof = fk.fk_profile_read(reset=True)
    ms = e0.elapsed_time(e1)
    # one more iteration with the per-chunk timeline (outside the timed region):
    # each chunk's copy must end before its compute begins (the stream waits
    # on it), and the copy of chunk j + 1 should run while chunk j computes
    fk.fk_profile_enable(3)
    fk.fk_lloyd(xt, initd, 1, 0.0, ids, cen, host_mode=fk.FK_HOST_STREAM)
    torch.cuda.synchronize()
    fk.fk_profile_enable(False)
    fk.fk_profile_read(reset=True)
    tl = fk.fk_profile_timeline()
    timeline = timeline_summary(tl)
    peaks, src_name = load_peaks()
    peak_t = float(peaks.get("bf16_tflops_sustained") or peaks["bf16_tflops"])
    flop_iter = 2.0 * w.B * w.N * w.K * w.d
    bytes_iter = w.B * w.N * w.d * 2
    iter_ms = ms / iters
    ideal_ms = max(flop_iter / (peak_t * 1e12), bytes_iter / (h2d_peak * 1e9)) * 1e3
    a_ms = prof["assign_ms"] / iters
    # checker: one iteration on the first 2^14 points with all K, extrapolated
    ns = 1 << 14
    xs = np.ascontiguousarray(xt.numpy()[:, :ns])
    c0 = synthdata.to_f64(init, w.dtype)
    tc = time.perf_counter()
    cid, _, _ = oracle.assign(xs, w.dtype, c0)
    oracle.update(xs, w.dtype, cid, c0)
    cpu_iter_s = (time.perf_counter() - tc) * (w.N / ns)
    line = {
        "metric": "Lloyd iter/s, large-N streamed from pinned host memory",
        "value": iters / (ms * 1e-3), "unit": "iter/s", "n_gpus": 1, "steps": args.steps, "warmup": 1,
        "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": f"largen: B={w.B} N={w.N} K={w.K} d={w.d} {w.dtype} mixture, points in pinned "
                               f"host memory, 2^24-point chunks, {w.iters} iterations per step",
                   "host_bytes": bytes_iter, "generation_s": gen_s},
        "roofline": {"bound": "max(tensor, pcie)", "achieved_ms_per_iter": iter_ms, "ideal_ms_per_iter": ideal_ms,
                     "frac": ideal_ms / iter_ms, "h2d_peak_gbs": h2d_peak,
                     "h2d_effective_gbs": bytes_iter / (iter_ms * 1e-3) / 1e9,
                     "assign_tflops": flop_iter / (a_ms * 1e-3) / 1e12 if a_ms > 0 else None,
                     "tensor_peak_tflops": peak_t, "peak_source": src_name},
        "cpu_baseline": {"value": 1.0 / cpu_iter_s, "unit": "iter/s", "cores": oracle.max_threads(),
                         "kind": "oracle",
                         "sample": f"one iteration on the first {ns} points with all K, extrapolated x{w.N // ns}"},
        "gpu_launches": fk.fk_launch_count() - launches0,
        "clocks": clk.summary(),
        "timeline": timeline,
    }
    print(json.dumps(line), flush=True)


# The other workloads of the parity suite, each timed briefly after the main
# measurement (not part of its timed region): CUDA events around fk_lloyd calls
# on device-resident points, FlashAssign and update times from the light
# event profile.
OTHER_WORKLOADS = ["zipf", "splitd", "tiny", "f32large"]


def measure_tf32_tflops(dev, n=8192, reps=10):
    """Dense tf32 tensor-core throughput of this GPU (cuBLAS fp32 GEMM with tf32
    allowed, n^3, best of reps): the denominator of the fp32 tensor-core path."""
    import torch
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = True
    try:
        a = torch.randn(n, n, device=dev)
        b = torch.randn(n, n, device=dev)
        for _ in range(3):
            torch.mm(a, b)
        best = 1e30
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch.mm(a, b)
            e1.record()
            torch.cuda.synchronize(dev)
            best = min(best, e0.elapsed_time(e1))
        return 2.0 * n ** 3 / (best * 1e-3) / 1e12
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev


def time_workload(name, dev, steps=3, warmup=2):
    import torch

    import clustering_flashassign_b200 as fk
    import synthdata
    w = synthdata.WORKLOADS[name]
    x, _, init = synthdata.make(w)

    def as_torch(a):
        t = torch.from_numpy(a)
        return t.view(torch.bfloat16) if w.dtype == "bf16" else t

    xd, initd = as_torch(x).to(dev), as_torch(init).to(dev)
    ids = torch.empty((w.B, w.N), dtype=torch.int32, device=dev)
    cen = torch.empty((w.B, w.K, w.d), dtype=torch.float32, device=dev)
    for _ in range(warmup):
        fk.fk_lloyd(xd, initd, w.iters, w.tol, ids, cen)
    torch.cuda.synchronize(dev)
    fk.fk_profile_read(reset=True)
    fk.fk_profile_enable(2)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    iters = 0
    e0.record()
    for _ in range(steps):
        iters += fk.fk_lloyd(xd, initd, w.iters, w.tol, ids, cen)
    e1.record()
    torch.cuda.synchronize(dev)
    fk.fk_profile_enable(False)
    prof = fk.fk_profile_read(reset=True)
    ms = e0.elapsed_time(e1)
    a_ms = prof["assign_ms"] / max(1, prof["assign_launches"])
    flop = 2.0 * w.B * w.N * w.K * w.d
    out = {"shape": f"B={w.B} N={w.N} K={w.K} d={w.d} {w.dtype}", "iter_per_s": iters / (ms * 1e-3),
           "assign_ms": a_ms, "assign_tflops": flop / (a_ms * 1e-3) / 1e12,
           "update_ms": prof["update_ms"] / max(1, prof["update_calls"]), "iterations": iters}
    if w.dtype == "f32" and w.d % 4 == 0 and w.K * w.d >= 16384:
        # 3xTF32: three tf32 passes per algorithmic flop, against a measured tf32 GEMM
        peak = measure_tf32_tflops(dev)
        out.update({"tf32_gemm_tflops": peak, "tf32_work_frac": 3 * out["assign_tflops"] / peak})
    return out


def timeline_summary(tl):
    """Per-chunk copy / compute events of one streamed iteration, summarised:
    how long copies and computes take, whether every copy ended before its
    compute began, and how much of each copy ran under the previous chunk's
    compute."""
    if not tl:
        return None
    copy = [c["copy_end"] - c["copy_begin"] for c in tl]
    comp = [c["compute_end"] - c["compute_begin"] for c in tl]
    before = sum(1 for c in tl if c["copy_end"] <= c["compute_begin"] + 1e-6)
    hidden = []
    for prev, cur in zip(tl, tl[1:]):
        # the part of this chunk's copy that ran while the previous chunk computed
        lo, hi = max(cur["copy_begin"], prev["compute_begin"]), min(cur["copy_end"], prev["compute_end"])
        span = cur["copy_end"] - cur["copy_begin"]
        hidden.append(max(0.0, hi - lo) / span if span > 0 else 1.0)
    gaps = [cur["compute_begin"] - prev["compute_end"] for prev, cur in zip(tl, tl[1:])]
    return {"chunks": len(tl), "copy_ms_mean": statistics.mean(copy), "compute_ms_mean": statistics.mean(comp),
            "copies_ended_before_their_compute": before,
            "copy_hidden_under_previous_compute_mean": statistics.mean(hidden) if hidden else None,
            "compute_gap_ms_max": max(gaps) if gaps else 0.0,
            "span_ms": tl[-1]["compute_end"] - tl[0]["copy_begin"],
            "first_chunks": [{k: round(v, 3) if isinstance(v, float) else v for k, v in c.items()} for c in tl[:4]]}


def baseline_assign_materialised(xd, cd):
    """The pages' first baseline: the distance matrix written to HBM and read
    back.  One cuBLAS batched GEMM (16-bit inputs, fp32 output) writes
    G = X (-2C)^T (B, N, K), ||c||^2 is added in place, argmin reads it.
    Returns the ids (B, N) int64."""
    import torch
    cn = (cd.float() ** 2).sum(-1).unsqueeze(1)             # (B, 1, K) fp32
    dmat = torch.bmm(xd, (-2.0 * cd).transpose(1, 2), out_dtype=torch.float32)
    dmat.add_(cn)
    return torch.argmin(dmat, dim=2)


def baseline_update_scatter(xd, ids, old):
    """The pages' second baseline: scatter atomics, one fp32 atomic add per
    point and dimension (index_add_), a bincount, a division; an empty
    cluster keeps its previous centroid.  Returns (centers (B, K, d) fp32,
    counts (B, K) int64)."""
    import torch
    B, N, d = xd.shape
    K = old.shape[1]
    flat = (ids.long() + torch.arange(B, device=xd.device).unsqueeze(1) * K).view(-1)
    sums = torch.zeros((B * K, d), dtype=torch.float32, device=xd.device)
    sums.index_add_(0, flat, xd.reshape(B * N, d).float())
    cnt = torch.bincount(flat, minlength=B * K)
    new = torch.where(cnt.unsqueeze(1) > 0, sums / cnt.clamp_min(1).unsqueeze(1), old.reshape(B * K, d))
    return new.view(B, K, d), cnt.view(B, K)


def time_baselines(xd, cd, reps):
    """CUDA-event times (ms per call) of the two baselines and of fk_assign and
    fk_update on the same inputs, with the speed-ups."""
    import torch

    import clustering_flashassign_b200 as fk
    B, N, d = xd.shape
    K = cd.shape[1]

    def timed(fn):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    ids = torch.empty((B, N), dtype=torch.int32, device=xd.device)
    t_fa = timed(lambda: fk.fk_assign(xd, cd, ids))
    t_matd = timed(lambda: baseline_assign_materialised(xd, cd))
    agree = float((baseline_assign_materialised(xd, cd) == ids.long()).float().mean())
    centers = cd.float()
    counts = torch.empty((B, K), dtype=torch.int32, device=xd.device)
    t_scat = timed(lambda: baseline_update_scatter(xd, ids, centers))
    work = centers.clone()
    t_upd = timed(lambda: fk.fk_update(xd, ids, work, counts))
    return {"assign_materialised_d_ms": t_matd, "assign_flashassign_ms": t_fa,
            "assign_speedup": t_matd / t_fa, "assign_ids_agree": agree,
            "materialised_d_bytes": B * N * K * 4,
            "update_scatter_atomic_ms": t_scat, "update_sort_inverse_ms": t_upd,
            "update_speedup": t_scat / t_upd,
            "scatter_atomic_gbs": B * N * d * 4 / (t_scat * 1e-3) / 1e9,
            "reps": reps}


def run_baselines(args):
    """The pages' comparison points, rebuilt on B200 at the api shape (context
    for the kernels' speedups; library code, not the product path): the
    distance matrix materialised and argmin'd, and the scatter-atomic update,
    each timed with CUDA events next to fk_assign and fk_update on the same
    inputs."""
    import torch
    w, x, init = make_inputs(0)
    dev = torch.device("cuda", 0)
    xd = torch.from_numpy(x).to(dev)
    cd = torch.from_numpy(init).to(dev)
    line = {"metric": "baselines at the api shape (ms per call; speedup = baseline / libfk)",
            "workload": f"api: B={w.B} N={w.N} K={w.K} d={w.d} {w.dtype}"}
    line.update(time_baselines(xd, cd, max(1, args.steps)))
    line["flashassign_tflops"] = 2.0 * w.B * w.N * w.K * w.d / (line["assign_flashassign_ms"] * 1e-3) / 1e12
    print(json.dumps(line), flush=True)


def run_kernel_case(args):
    """Launch only one step kind on the bench workload (for profiler captures):
    assign = fk_assign, update = fk_update, lloyd = fk_lloyd with two
    iterations, each warmup + steps times.  In an fk_lloyd call the first
    assign sums the point norms from its shared tiles and stores them, the
    second reads them; both fill the sort's tile histogram, as in the bench
    (after the one fk_assign below, odd-numbered assign launches are first
    assigns)."""
    import torch

    import clustering_flashassign_b200 as fk
    import synthdata
    w = rank_workload(0, args.workload, **({"N": args.points} if args.points else {}))
    x, _, init = synthdata.make(w)
    xd = torch.from_numpy(x).cuda()
    cd = torch.from_numpy(init).cuda()
    ids = torch.empty((w.B, w.N), dtype=torch.int32, device="cuda")
    fk.fk_assign(xd, cd, ids)
    centers = cd.float()
    counts = torch.empty((w.B, w.K), dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    for _ in range(args.warmup + args.steps):
        if args.kernel_case == "assign":
            fk.fk_assign(xd, cd, ids)
        elif args.kernel_case == "lloyd":
            fk.fk_lloyd(xd, cd, 2, 0.0, ids, centers)
        else:
            fk.fk_update(xd, ids, centers, counts)
    torch.cuda.synchronize()
    print(json.dumps({"kernel_case": args.kernel_case, "B": w.B, "N": w.N, "K": w.K, "d": w.d,
                      "launches": fk.fk_launch_count(), "device_error": fk.fk_device_error()}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="fk", choices=["fk", "reference"])
    ap.add_argument("--kernel-case", default=None, choices=["assign", "update", "lloyd"],
                    help="launch only this step (profiler captures); prints no bench line")
    ap.add_argument("--points", type=int, default=0, help="with --kernel-case / --workload: points per batch")
    ap.add_argument("--baselines", action="store_true",
                    help="time the materialised-distance assign and the scatter-atomic update next to libfk")
    ap.add_argument("--no-baselines", action="store_true",
                    help="leave the two baseline timings out of the bench line")
    ap.add_argument("--no-workloads", action="store_true",
                    help="leave the timings of the other workloads out of the bench line")
    ap.add_argument("--workload", default="api", choices=["api", "tiny", "zipf", "splitd", "largen", "f32large"],
                    help="api is the benchmark; the others print their own line (largen: the 64 GiB "
                         "streamed workload)")
    args = ap.parse_args()
    world = env_int("WORLD_SIZE", 1)
    rank = env_int("RANK", 0)
    local_rank = env_int("LOCAL_RANK", 0)
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if args.kernel_case:
        run_kernel_case(args)
        return
    if args.baselines:
        run_baselines(args)
        return
    if args.workload == "largen":
        run_largen(args)
        return
    dist = None
    if world > 1:
        import datetime

        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(local_rank)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        dist = tdist
    try:
        run_fk(args, rank, world, local_rank, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
