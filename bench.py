#!/usr/bin/env python
"""Throughput of the batched Dion optimizer step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one dion_step_batched call over every weight matrix of the workload
(default: 7B-like transformer, 32 layers, hidden 4096, MLP 11008, rank 256 = 1/16,
bf16-input GEMMs, fp32 state; 224 matrices, 6.476e9 parameters).  Inputs are
synthetic and already resident in HBM when the timed region starts; they are far
larger than L2 (126 MB), so no L2 flush is needed between steps.

Prints one JSON line (rank 0).  Under torchrun every rank updates its own full set of
matrices (weak scaling, no collective on the data path); the step time is the max over
ranks of the device-timed region.

``--impl reference`` times the fp64 CPU oracle instead, on a bounded sample of the same
workload (one matrix per shape bucket per step), extrapolated to the whole workload.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "params updated/s (Dion steps/s) at 7B shapes; % of roofline"
UNIT = "params/s"


# ------------------------------------------------------------ distributed plumbing
def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def dist_setup(backend: str):
    import torch.distributed as dist
    rank, world, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return rank, world


def max_over_ranks(value: float, device=None) -> float:
    """Max of a float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and str(device).startswith("cuda"):
            dist.barrier(device_ids=[int(str(device).split(":")[1])])
        else:
            dist.barrier()


def whole_job_rate(units_per_rank: float, world: int, seconds_max: float) -> float:
    """Units processed by all ranks divided by the slowest rank's time."""
    return units_per_rank * world / seconds_max


# ------------------------------------------------------------------ clocks sampler
_REASON_BITS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
                ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4))


class Clocks:
    """SM clock, power and clock-event reasons sampled DURING the timed region.

    NVML is read from a background thread every 10 ms (read-only queries: nothing about
    the GPU's settings is changed), so even a sub-second timed region gives dozens of
    samples; without NVML, ``nvidia-smi -lms 200`` is polled instead."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_S = 0.01

    def __init__(self, gpu_index: int, pci_bus_id: str | None = None):
        self.gpu = gpu_index
        self.pci = pci_bus_id
        self.rows = []          # (sm_mhz, sm_max_mhz, power_w, reasons_bitmask)
        self.proc = None
        self.path = None
        self.thread = None
        self.stop = None
        self.source = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        if self.pci:
            try:
                return pynvml.nvmlDeviceGetHandleByPciBusId(self.pci)
            except Exception:
                pass
        return pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def _sample_nvml(self, h):
        import pynvml
        smax = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        while not self.stop.is_set():
            try:
                self.rows.append((pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM), smax,
                                  pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0,
                                  pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)))
            except Exception:
                break
            self.stop.wait(self.PERIOD_S)

    def __enter__(self):
        import threading
        try:
            h = self._nvml_handle()
            self.stop = threading.Event()
            self.thread = threading.Thread(target=self._sample_nvml, args=(h,), daemon=True)
            self.thread.start()
            self.source = "nvml, 10 ms"
            time.sleep(0.05)
            return self
        except Exception:
            self.thread = None
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            self.source = "nvidia-smi, 200 ms"
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def _smi_rows(self):
        rows = []
        try:
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                    bits = sum(b for i, (_, b) in enumerate(_REASON_BITS)
                               if parts[5 + i].lower() == "active")
                    rows.append((float(parts[1]), float(parts[2]), float(parts[3]), bits))
        except Exception:
            pass
        finally:
            if self.path and os.path.exists(self.path):
                os.unlink(self.path)
        return rows

    def summary(self):
        rows = self.rows if self.thread is not None else self._smi_rows()
        return summarize_clocks(rows, self.source)


def summarize_clocks(rows, source=None):
    """Median SM clock under load, the max clock and the throttle reasons seen, from
    (sm_mhz, sm_max_mhz, power_w, reasons_bitmask) samples."""
    if not rows:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clocks not sampled"]}
    sm = [float(r[0]) for r in rows]
    smax = max(float(r[1]) for r in rows)
    loaded = [s for s, r in zip(sm, rows) if float(r[2]) > 200.0] or sm
    reasons = sorted({name for r in rows for name, bit in _REASON_BITS if int(r[3]) & bit})
    return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": smax, "reasons": reasons,
            "samples": len(rows), "power_w_max": max(float(r[2]) for r in rows),
            "source": source}


# ------------------------------------------------------------------ roofline figures
def algorithmic(wl: W.Workload):
    """Per step: flops of the four rank-r contractions + Cholesky-QR, and the bytes the
    method must move (32 B per weight element: three dependent sweeps over B, plus the
    r-sized factors); and the bytes of the fused update alone (20 B per element)."""
    flops = sum(b.count * (8 * b.m * b.n * b.r + 3 * b.m * b.r ** 2 + b.r ** 3 / 3)
                for b in wl.buckets)
    bytes_ = sum(b.count * (32 * b.m * b.n + 4 * (3 * b.m * b.r + 6 * b.n * b.r))
                 for b in wl.buckets)
    update_bytes = sum(b.count * 20 * b.m * b.n for b in wl.buckets)
    return flops, bytes_, update_bytes


def split_ceiling(wl: W.Workload, peaks):
    """The ceiling of fp32 mode on the tensor path, whose contractions run as bf16
    products of three-way splits: six for B Q, B^T P, the Gram and the apply, three for
    the update (its two leading parts); B kept as its split, written once and read by
    both sweeps (40 B per weight element with B = M + G fused into B Q).  The time of
    those bf16 products at the measured bf16 peak, or of those bytes at the measured copy
    bandwidth, whichever is longer."""
    flops = sum(b.count * (36 * b.m * b.n * b.r + 18 * b.m * b.r ** 2 + b.r ** 3 / 3)
                for b in wl.buckets)
    bytes_ = sum(b.count * (40 * b.m * b.n + 4 * (3 * b.m * b.r + 6 * b.n * b.r))
                 for b in wl.buckets)
    t = max(flops / (peaks["bf16_tflops"] * 1e12), bytes_ / (peaks["hbm_gbs"] * 1e9))
    return flops, bytes_, t


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "k_tc_update_traffic_r256_shapes.json")


def update_traffic():
    """DRAM bytes per weight element of the fused update by matrix shape ("MxN"), from the
    committed ncu captures, and the hash of the kernel source they were taken on."""
    if os.path.exists(TRAFFIC_FILE):
        d = json.load(open(TRAFFIC_FILE))
        return d.get("dram_bytes_per_element"), d.get("kernel_source_hash")
    return None, None


def update_traffic_per_launch(wl: W.Workload, launches: float):
    """The update's DRAM bytes per launch on this workload from the per-shape captures
    (bytes per element of each bucket's shape times its elements, over the launches);
    None when a bucket's shape was not captured or the kernel changed since."""
    per, h = update_traffic()
    if not per or h != update_kernel_hash() or launches <= 0:
        return None
    total = 0.0
    for b in wl.buckets:
        key = f"{b.m}x{b.n}"
        if key not in per:
            return None
        total += per[key] * b.params
    return total / launches


def update_kernel_hash():
    """Hash of the fused-update kernel's source (its section of k_tc.cu and the PTX
    helpers): a captured traffic figure is only reported while this is unchanged."""
    import hashlib
    csrc = os.path.join(ROOT, "rank_orthonormalized_optimizer_b200", "csrc")
    src = open(os.path.join(csrc, "k_tc.cu")).read()
    marker = "// ------------------------------------------------------------------ fused update"
    upd = src[src.index(marker):] if marker in src else src
    return hashlib.sha256((upd + open(os.path.join(csrc, "tc_ptx.cuh")).read()).encode()).hexdigest()[:16]


# ------------------------------------------------------------------ oracle timing
def oracle_sample(wl: W.Workload, steps: int, budget_s: float = 20.0):
    """Time the fp64 oracle on one matrix per bucket; returns (params/s, seconds, cores,
    note).  The seconds are the whole workload's step extrapolated from the sample by
    the bucket counts."""
    import oracle
    blas = "unknown"
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        cores = max((i.get("num_threads", 0) for i in info), default=os.cpu_count())
        blas = ", ".join(sorted({f"{i.get('internal_api')} {i.get('version')}" for i in info
                                 if i.get("user_api") == "blas"})) or "unknown"
    except Exception:
        cores = os.cpu_count()
    per_bucket = []
    spent = 0.0
    for bi, b in enumerate(wl.buckets):
        X = W.weights(wl, bi, "cpu", slots=[0])[0].double().numpy()
        M = W.momentum(wl, bi, "cpu", slots=[0])[0].double().numpy()
        Q = W.right_factor(wl, bi, "cpu", slots=[0])[0].double().numpy()
        G = W.gradient(wl, bi, 0, "cpu", slots=[0])[0].double().numpy()
        times = []
        for _ in range(max(1, steps)):
            t0 = time.perf_counter()
            X, M, Q, _, _ = oracle.dion_step(X, M, G, Q, wl.mu, wl.lr)
            times.append(time.perf_counter() - t0)
            spent += times[-1]
            if spent > budget_s:
                break
        per_bucket.append(statistics.median(times))
    step_s = sum(b.count * t for b, t in zip(wl.buckets, per_bucket))
    note = (f"fp64 NumPy oracle (BLAS: {blas}; host has {os.cpu_count()} logical cores), one matrix per bucket "
            f"({', '.join(f'{b.m}x{b.n}' for b in wl.buckets)}), median of up to {steps} steps each, "
            f"scaled by bucket counts ({', '.join(str(b.count) for b in wl.buckets)}) to the full "
            f"{wl.params:.4g}-parameter step ({step_s:.1f} s extrapolated)")
    return wl.params / step_s, step_s, cores, note


def l2_note(wl: W.Workload, world: int = 1) -> str:
    """How the timed steps stand against the 126 MB L2: the fp32 X, M and G a step streams
    (per rank) either dwarf it, and no flush is needed, or they do not."""
    state = 12 * wl.params / world
    if state > 4 * L2_BYTES:
        return f"inputs ({state / 1e9:.3g} GB of fp32 X, M, G per rank) far larger than L2; no flush"
    if state > L2_BYTES:
        return (f"inputs ({state / 1e6:.3g} MB of fp32 X, M, G) larger than L2 but partly "
                f"resident between steps; no flush: a latency-bound case, quoted as a time")
    return (f"inputs ({state / 1e6:.3g} MB of fp32 X, M, G) resident in L2: a launch-bound "
            f"case, quoted as a time, not against the roofline")


# ------------------------------------------------------------------ the GPU arm
def _pci_bus_id(dev):
    import torch
    try:
        p = torch.cuda.get_device_properties(dev)
        return f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
    except Exception:
        return None


def run_ours(args):
    import numpy as np
    import torch

    rank, world = dist_setup("nccl")
    _, _, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from rank_orthonormalized_optimizer_b200 import DionB200

    wl = W.WORKLOADS[args.workload]
    opt = DionB200([(b.count, b.m, b.n, b.r) for b in wl.buckets], mu=wl.mu,
                   precision=wl.precision, kernel_path=args.kernel_path,
                   stack_orth=args.stack_orth)
    nb = len(wl.buckets)
    X = [W.weights(wl, i, dev) for i in range(nb)]
    M = [W.momentum(wl, i, dev) for i in range(nb)]
    Q = [W.right_factor(wl, i, dev) for i in range(nb)]
    G = [W.gradient(wl, i, 0, dev) for i in range(nb)]
    ws = opt.alloc_workspace(dev)
    status = opt.alloc_status(dev)
    stream = torch.cuda.current_stream(dev)

    for _ in range(args.warmup):
        opt.step(X, M, G, Q, wl.lr, ws, status, stream)
    torch.cuda.synchronize(dev)

    # timed region: K steps, barrier + sync on both sides, device events
    opt.profile_enable(True)
    launches = 0
    with Clocks(local, _pci_bus_id(dev)) as clk:
        barrier(dev)
        torch.cuda.synchronize(dev)
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(args.steps):
            opt.step(X, M, G, Q, wl.lr, ws, status, stream)
            launches += opt.last_launch_count
        t1.record(stream)
        torch.cuda.synchronize(dev)
        barrier(dev)
    clocks = clk.summary()
    ms_local = t0.elapsed_time(t1) / args.steps
    prof = opt.profile_read()
    opt.profile_enable(False)
    ms = max_over_ranks(ms_local, dev)
    st = status.cpu()

    value = whole_job_rate(wl.params, world, ms / 1e3)
    flops, bytes_alg, upd_bytes = algorithmic(wl)
    peaks = measured_peaks()
    upd_ms = prof["update"][0] / args.steps
    upd_launches = prof["update"][1] / args.steps
    achieved = upd_bytes / (upd_ms / 1e3) / 1e9
    traffic = update_traffic_per_launch(wl, upd_launches)
    roof_t = max(flops / (peaks["bf16_tflops"] * 1e12), bytes_alg / (peaks["hbm_gbs"] * 1e9))
    comp_bytes = sum(b.count * (20 * b.m * b.n + 8 * b.n * b.r) for b in wl.buckets)
    comp_t = comp_bytes / (peaks["hbm_gbs"] * 1e9)

    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "steps_per_s": 1e3 / ms * 1.0,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if wl.precision == "bf16" else "f32", "data": "synthetic",
        "config": {"workload": wl.name, "matrices": sum(b.count for b in wl.buckets),
                   "params_per_gpu": wl.params,
                   "buckets": [[b.count, b.m, b.n, b.r] for b in wl.buckets],
                   "state": "fp32 X, M, G, Q", "gemm_inputs": wl.precision,
                   "kernel_path": args.kernel_path, "stack_orth": bool(args.stack_orth),
                   "parallelism": f"matrix-partitioned x{world} (each rank its own matrices)",
                   "l2": l2_note(wl)},
        "roofline": {"bound": "hbm", "kernel": "fused update (M and X)",
                     "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
                     "peak_source": peaks["source"],
                     "per_step_ms": upd_ms, "algorithmic_bytes_per_step": upd_bytes},
        "step_roofline": {"t_roofline_ms": roof_t * 1e3, "frac": roof_t * 1e3 / ms,
                          "flops": flops, "bytes": bytes_alg,
                          # the state alone (read M, G, X, Q; write M, X, Q), as if the three
                          # sweeps over B needed no more than one
                          "compulsory_bytes": comp_bytes,
                          "t_compulsory_ms": comp_t * 1e3,
                          "frac_compulsory": comp_t * 1e3 / ms},
        "kernel_ms_per_step": {k: v[0] / args.steps for k, v in prof.items()},
        "gpu_launches": launches,
        "status_bits": int(np.bitwise_or.reduce(st.numpy())) if st.numel() else 0,
        "clocks": clocks,
    }

    if wl.precision == "fp32" and args.kernel_path == "tensor":
        sf, sb, st_ = split_ceiling(wl, peaks)
        result["split_roofline"] = {"t_ms": st_ * 1e3, "frac": st_ * 1e3 / ms,
                                    "bf16_product_flops": sf, "bytes": sb}

    # end to end through the C ABI with the gradients in pinned host memory
    if not args.no_e2e:
        Gh = []
        for g in G:
            h = torch.empty(g.shape, dtype=g.dtype, pin_memory=True)
            h.copy_(g)
            Gh.append(h)
        hs = torch.zeros(opt.num_matrices, dtype=torch.int32).pin_memory()
        opt.step_from_host(X, M, G, Q, Gh, wl.lr, ws, status, hs, stream)
        barrier(dev)
        t_start = time.perf_counter()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            opt.step_from_host(X, M, G, Q, Gh, wl.lr, ws, status, hs, stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, dev)
        result["e2e"] = {"value": whole_job_rate(wl.params, world, e2e_ms / 1e3), "unit": UNIT,
                         "h2d_bytes_per_step": sum(g.numel() * 4 for g in Gh),
                         "d2h_bytes_per_step": hs.numel() * 4, "ms_per_step": e2e_ms,
                         "steps": args.e2e_steps,
                         "note": "gradients uploaded from pinned host memory and the per-matrix "
                                 "status read back every step (dion_step_batched_from_host)"}
        del Gh
        _ = time.perf_counter() - t_start

    if not args.no_vector:
        del ws
        torch.cuda.empty_cache()
        result["vector_step"] = measure_vector_step(dev, stream, peaks)

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, step_s, cores, note = oracle_sample(wl, steps=2)
        result["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                                  "sample": note}
    if rank == 0:
        print(json.dumps(result), flush=True)
    opt.close()
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()


# ------------------------------------------------------------ row-sharded step
def run_rowshard(args):
    """The workload's matrices split by rows over the ranks (dion_init_sharded): every
    rank holds rows of every matrix, and each step all-reduces the Grams and R over NCCL
    (strong scaling: the total work is fixed).  At one rank nothing is exchanged; the
    line then measures what the sharded protocol itself costs (its host round trip)."""
    import numpy as np
    import torch

    rank, world = dist_setup("nccl")
    _, _, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from rank_orthonormalized_optimizer_b200 import DionB200RowSharded

    wl = W.WORKLOADS[args.workload]
    opt = DionB200RowSharded([(b.count, b.m, b.n, b.r) for b in wl.buckets], rank, world,
                             mu=wl.mu, precision=wl.precision)
    nb = len(wl.buckets)

    def rows(t, i):
        r0, mk = opt.row_ranges[i]
        return t[:, r0:r0 + mk].contiguous()

    X, G = [], []
    for i in range(nb):
        X.append(rows(W.weights(wl, i, dev), i))
        G.append(rows(W.gradient(wl, i, 0, dev), i))
        torch.cuda.empty_cache()
    M = [torch.zeros_like(x) for x in X]
    Q = [W.right_factor(wl, i, dev) for i in range(nb)]
    ws = opt.alloc_workspace(dev)
    status = opt.alloc_status(dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        xchg = opt.step(X, M, G, Q, wl.lr, ws, status, stream)
    torch.cuda.synchronize(dev)
    launches = 0
    with Clocks(local, _pci_bus_id(dev)) as clk:
        barrier(dev)
        torch.cuda.synchronize(dev)
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(args.steps):
            xchg = opt.step(X, M, G, Q, wl.lr, ws, status, stream)
            launches += opt.last_launch_count
        t1.record(stream)
        torch.cuda.synchronize(dev)
        barrier(dev)
    ms = max_over_ranks(t0.elapsed_time(t1) / args.steps, dev)
    st = status.cpu()
    flops, bytes_alg, _ = algorithmic(wl)
    peaks = measured_peaks()
    roof_t = max(flops / (peaks["bf16_tflops"] * 1e12),
                 bytes_alg / (peaks["hbm_gbs"] * 1e9)) / world
    result = {
        "metric": METRIC, "value": wl.params / (ms / 1e3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
        "dtype": "bf16" if wl.precision == "bf16" else "f32", "data": "synthetic",
        "config": {"workload": wl.name, "params": wl.params,
                   "buckets": [[b.count, b.m, b.n, b.r] for b in wl.buckets],
                   "parallelism": f"row-sharded x{world} (every matrix split by rows)",
                   "l2": l2_note(wl, world)},
        "exchanges_per_step": [k for k, _ in xchg],
        "allreduce_floats_per_step": sum(c for _, c in xchg) if world > 1 else 0,
        "step_roofline": {"t_roofline_ms": roof_t * 1e3, "frac": roof_t * 1e3 / ms},
        "gpu_launches": launches,
        "status_bits": int(np.bitwise_or.reduce(st.numpy())) if st.numel() else 0,
        "clocks": clk.summary(),
    }
    if rank == 0:
        print(json.dumps(result), flush=True)
    opt.close()
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()


# ------------------------------------------------------------ vector (1-D) parameters
L2_BYTES = 126 << 20                    # B200 L2
VEC_BYTES = {"adamw": 28, "lion": 20}   # per element: AdamW reads x, g, m, v and writes
                                        # x, m, v; Lion reads x, g, m and writes x, m


def measure_vector_step(dev, stream, peaks, warmup=3, iters=10,
                        names=("vectors_64x4Mi", "norms_h4096_l32")):
    """AdamW and Lion over the vector parameters (dion_vec_step through a prepared
    VecStepPlan): a bank of 64 x 4 Mi elements (4 GiB of state, far larger than L2)
    against the copy bandwidth, and the 65 RMSNorm gains of the 7B-like decoder
    (L2-resident): per call through the C ABI, where the host's call and launch cost
    dominates, and with the calls enqueued ahead of the device, which leaves the
    device time."""
    import torch

    from rank_orthonormalized_optimizer_b200 import VecStepPlan
    out = {}
    for name in names:
        vw = W.VECTOR_WORKLOADS[name]
        n = vw.params
        big = 16 * n > L2_BYTES        # the four state arrays do not fit in L2
        reps = iters if big else 20 * iters
        flat = {k: torch.empty(n, dtype=torch.float32, device=dev) for k in "xgmv"}
        views = {k: [] for k in "xgmv"}
        off = 0
        for i, sz in enumerate(vw.sizes):
            vals = W.vector_state(vw, i, 0, dev)
            for k, t in zip("xgmv", vals):
                flat[k][off:off + sz].copy_(t)
                views[k].append(flat[k][off:off + sz])
            off += sz
        rec = {"elements": n, "tensors": len(vw.sizes)}
        for rule in ("adamw", "lion"):
            plan = VecStepPlan(views["x"], views["g"], views["m"],
                               views["v"] if rule == "adamw" else None, rule=rule)
            for t in range(warmup):
                plan.step(t + 1, stream)
            barrier(dev)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            launches = 0
            for t in range(reps):
                launches += plan.step(warmup + t + 1, stream)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            ms = max_over_ranks(e0.elapsed_time(e1) / reps, dev)
            gbs = VEC_BYTES[rule] * n / (ms * 1e-3) / 1e9
            r = {"us": ms * 1e3, "launches_per_step": launches // reps,
                 "bytes_per_element": VEC_BYTES[rule], "achieved_GBs": gbs,
                 "frac_of_copy_peak": gbs / peaks["hbm_gbs"], "peak_source": peaks["source"]}
            if not big:
                # the same calls with the host ahead of the device: a bounded spin kernel
                # (about 20 ms) holds the stream while every call is enqueued, so the
                # events bracket the launches back to back (device time per call)
                with torch.cuda.stream(stream):
                    torch.cuda._sleep(40_000_000)
                e0.record(stream)
                for t in range(reps):
                    plan.step(warmup + reps + t + 1, stream)
                e1.record(stream)
                torch.cuda.synchronize(dev)
                r["queued_us"] = max_over_ranks(e0.elapsed_time(e1) / reps, dev) * 1e3
            rec[rule] = r
        rec["l2"] = ("state (%.2f GB) larger than L2" % (16 * n / 1e9) if big
                     else "state resident in L2 (%.1f MB); launch-bound" % (16 * n / 1e6))
        out[name] = rec
        del flat, views
        torch.cuda.empty_cache()
    return out


def run_vector_only(args):
    """The vector-parameter step alone: one JSON line with its timings."""
    import torch

    rank, world = dist_setup("nccl")
    _, _, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    peaks = measured_peaks()
    rec = measure_vector_step(dev, torch.cuda.current_stream(dev), peaks, warmup=args.warmup,
                              iters=args.steps, names=(args.vector_only,))
    if rank == 0:
        print(json.dumps({"metric": "vector-parameter step (AdamW, Lion)", "n_gpus": world,
                          "steps": args.steps, "warmup": args.warmup, "data": "synthetic",
                          "peak_GBs": peaks["hbm_gbs"], "peak_source": peaks["source"],
                          "vector_step": rec}), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()


# ------------------------------------------------------------------ the oracle arm
def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    wl = W.WORKLOADS[args.workload]
    for _ in range(args.warmup):
        oracle_sample(wl, steps=1, budget_s=5.0)
    t0 = time.perf_counter()
    vals = []
    cores = note = None
    for _ in range(args.steps):
        v, step_s, cores, note = oracle_sample(wl, steps=1, budget_s=10.0)
        vals.append(step_s)
    wall = time.perf_counter() - t0
    step_s = statistics.median(vals)
    value = wl.params / step_s
    sampled = len(wl.buckets)
    total = sum(b.count for b in wl.buckets)
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": wl.name, "params": wl.params},
        # each timed step runs one matrix per shape bucket; ms_per_step is that sample
        # scaled by the bucket counts to the whole workload, not a measured step
        "extrapolated": total != sampled,
        "matrices_run_per_step": sampled, "matrices_per_workload_step": total,
        "sample_ms_per_step": wall / max(args.steps, 1) * 1e3,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": note},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": wall}), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=W.HEADLINE, choices=sorted(W.WORKLOADS))
    ap.add_argument("--kernel-path", default="tensor", choices=["tensor", "simt"])
    ap.add_argument("--stack-orth", action="store_true",
                    help="one orthonormalisation stack per (m, r) across buckets")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-vector", action="store_true",
                    help="skip the AdamW / Lion step of the vector parameters")
    ap.add_argument("--rowshard", action="store_true",
                    help="split every matrix by rows over the ranks (all-reduce of the Grams "
                         "and R over NCCL) instead of giving each rank its own matrices")
    ap.add_argument("--vector-only", default=None, choices=sorted(W.VECTOR_WORKLOADS),
                    help="time only the vector-parameter step on this workload (for profiling "
                         "its kernel with little else on the device)")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args)
    elif args.vector_only:
        run_vector_only(args)
    elif args.rowshard:
        run_rowshard(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
