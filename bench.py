#!/usr/bin/env python
"""Benchmark of the Shampoo optimizer step (statistics + inverse roots +
grafted apply) on B200, through the library's C-ABI.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cuda|reference]
                  [--config transformer_layer_b512]

A step is update_stats, compute_roots on every root_interval-th step
(counted from the first timed step, so K = root_interval times the root
step exactly once per interval) and apply, on one fixed seeded gradient set
per step.  Inputs are resident in HBM before timing; each step is timed with
CUDA events on the optimizer's stream and L2 is flushed (a 256 MiB write)
between steps, outside the events.  With N > 1 (torchrun) every rank runs its
own copy of the parameter set: the blocks are independent, so there is no
data-path collective (weak scaling); the job time is the max over ranks.
Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from shampoo_second_order_b200 import workloads as wl  # noqa: E402

METRIC = "Shampoo optimizer step ms and TFLOP/s (stats+roots+apply) vs B200 peak, 1 GPU"
UNIT = "TFLOP/s"

# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from an
# ncu capture of the named kernel on the named workload (float64 Newton
# products, both factors, the default --steps/--warmup); None for any other
# workload, mode or kernel until measured there.
TRAFFIC_PER_LAUNCH = {
    # the 9 launches of the timed root step of the Transformer-layer run (the
    # first, whose X product is a scaled copy: 0.80 GB; 4 more with every
    # matrix iterating: ~1.01 GB each; 3 with a few: 17 MB; 1 with none),
    # averaged like `achieved`
    ("transformer_layer_b512", "newton_step_a"): 542061340,
}


# ---------------------------------------------------------------------------
# Work model: algorithmic flops and bytes of the workload
# ---------------------------------------------------------------------------
def blocks_of(cfg):
    b = cfg["block_size"]
    blks, segs = [], []
    for s in cfg["shapes"]:
        if len(s) == 2:
            for r0 in range(0, s[0], b):
                for c0 in range(0, s[1], b):
                    blks.append((min(b, s[0] - r0), min(b, s[1] - c0)))
        else:
            for s0 in range(0, s[0], b):
                segs.append(min(b, s[0] - s0))
    return blks, segs


def block_sides(cfg):
    """Per block, library order: 0 both factors, 2 R only (one-sided weights
    listed in cfg["right_only"] by parameter index)."""
    ro = set(cfg.get("right_only", ()))
    out = []
    b = cfg["block_size"]
    for i, s in enumerate(cfg["shapes"]):
        if len(s) == 2:
            out += [2 if i in ro else 0] * (-(-s[0] // b) * -(-s[1] // b))
    return out


def matrix_sizes(cfg):
    """(valid side, products per Newton step) per statistic, library order;
    a factor rooted at p/2 = 2 takes 3 products (X T, T T, T^2 M)."""
    blks, segs = blocks_of(cfg)
    out = []
    for (m, n), sd in zip(blks, block_sides(cfg)):
        pl = 4 if cfg["p"] == 4 and sd == 0 else 3
        out += [(m, pl), (n, pl)]   # a dropped factor runs no iterations
    out += [(ln, 3 if cfg["p"] == 4 else 3) for ln in segs]   # p/2 = 2: X T, T T, T^2 M
    return out


def stats_flops(cfg):
    """SYRK triangles: m(m+1) n for L and n(n+1) m for R (R only for a
    one-sided block); len(len+1) per segment."""
    blks, segs = blocks_of(cfg)
    return (sum((0 if sd else m * (m + 1) * n) + n * (n + 1) * m for (m, n), sd in zip(blks, block_sides(cfg)))
            + sum(l * (l + 1) for l in segs))


def apply_flops(cfg):
    """Two chained GEMMs per block, 2mn(m+n) (G R only, 2mn^2, for a one-sided
    block); a matvec 2 len^2 per segment."""
    blks, segs = blocks_of(cfg)
    return (sum((2 * m * n * n if sd else 2 * m * n * (m + n)) for (m, n), sd in zip(blks, block_sides(cfg)))
            + sum(2 * l * l for l in segs))


def newton_flops(cfg, iters, per_kernel=False):
    """Symmetric products: n^2 (n+1) flops each (the upper triangle), times
    products per step, times the iterations each matrix ran; the first step's
    X0 T0 is a scaled copy (X0 = c^{-1} I), not a product."""
    sizes = matrix_sizes(cfg)
    a = b = c = 0
    for (n, prods), k in zip(sizes, iters):
        k = k if k >= 0 else -1 - k
        f = n * n * (n + 1)
        a += (2 * k - (1 if k > 0 else 0)) * f
        b += (k * f) if prods == 4 else 0
        c += k * f
    return (a, b, c) if per_kernel else a + b + c


def ozaki_ops(cfg, iters, slices, per_kernel=False):
    """int8 tensor-core operations the emulated Newton products execute: per
    product, every 128 x 64 tile of the upper triangle of the b x b slot runs
    slices (slices + 1) / 2 digit products over the padded K = b."""
    S = -(-cfg["block_size"] // 64) * 64
    tc, tr = S // 64, -(-S // 128)
    ntri = sum(max(0, tc - 2 * ti) for ti in range(tr))
    nk = -(-S // 128)
    per = ntri * nk * 128 * 2 * 128 * 64 * slices * (slices + 1) // 2
    a = b = c = 0
    for (n, prods), k in zip(matrix_sizes(cfg), iters):
        k = k if k >= 0 else -1 - k
        a += 2 * k * per
        b += (k * per) if prods == 4 else 0
        c += k * per
    return (a, b, c) if per_kernel else a + b + c


def numel(cfg):
    return wl.count_params(cfg["shapes"])


def max_over_ranks(ms, dist, device):
    """The job time: the largest per-rank device time (one all-reduce)."""
    import torch
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(ms)
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flops_per_rank, world, job_ms):
    """Whole-job throughput: the work of all ranks over the slowest rank's time."""
    return world * flops_per_rank / (job_ms * 1e-3) / 1e12


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """SM clock and throttle reasons of one GPU, polled through NVML every
    2 ms on a background thread while the timed region runs (nvidia-smi's
    fastest loop is too slow for a region of tens of milliseconds)."""
    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, uuid=None, index=0):
        import threading
        self.samples, self.reasons, self.max_mhz, self.err = [], set(), None, None
        self.stop_flag = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            h = None
            if uuid:
                try:
                    h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
                except Exception:
                    h = None
            self.h = h or pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:   # no NVML: report why
            self.nv, self.err = None, str(e)
            return
        self.t = threading.Thread(target=self._run, daemon=True)
        self.t.start()

    def _run(self):
        nv = self.nv
        while not self.stop_flag.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                get = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    nv.nvmlDeviceGetCurrentClocksThrottleReasons
                r = get(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception as e:
                self.err = str(e)
                return
            time.sleep(0.002)

    def stop(self):
        if self.nv is None:
            return {"error": self.err}
        self.stop_flag.set()
        self.t.join(timeout=2)
        if not self.samples:
            return {"error": self.err or "no samples"}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "NVML, 2 ms"}


def gpu_uuid(torch, dev):
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return None


def fp64_peak_tflops(torch, dev):
    """cuBLAS DGEMM throughput (torch.matmul, float64, 4096^3, best of 5)."""
    n = 4096
    a = torch.randn(n, n, dtype=torch.float64, device=dev)
    b = torch.randn(n, n, dtype=torch.float64, device=dev)
    torch.matmul(a, b)
    best = 1e9
    for _ in range(5):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        torch.matmul(a, b)
        e.record()
        e.synchronize()
        best = min(best, s.elapsed_time(e))
    del a, b
    return 2 * n ** 3 / (best * 1e-3) / 1e12


def tc_work(cfg, kernel):
    """Algorithmic (flops, bytes) of one launch of a tensor-core kernel over
    the whole parameter set: flops as bf16 MMA work (products kept x the
    exact flop count), bytes as the minimum HBM traffic (each operand read once,
    each output written once; statistics read and written on their
    upper-triangle 128-tiles)."""
    b = cfg["block_size"]
    blks, _ = blocks_of(cfg)
    f32 = cfg["grad_dtype"] == "f32"
    planes = 3 if f32 else 1
    T = (b + 127) // 128
    tri = T * (T + 1) // 2 * 128 * 128 * 4          # bytes of one statistic's upper tiles
    if kernel == "stats_tc":
        passes = 6 if f32 else 1
        fl = sum((0 if sd else m * (m + 1) * n) + n * (n + 1) * m
                 for (m, n), sd in zip(blks, block_sides(cfg))) * passes
        by = sum(2 * planes * m * n for m, n in blks) + len(blks) * 2 * 2 * tri
    elif kernel == "apply_y_tc":
        passes = 3 if f32 else 2
        fl = sum(2 * m * n * n for m, n in blks) * passes
        by = sum(2 * min(planes, 2) * m * n + 2 * 2 * n * n + 2 * 2 * m * n for m, n in blks)
    else:   # apply_p_tc
        fl = sum(2 * m * m * n for m, n in blks) * 3
        by = sum(2 * 2 * m * m + 2 * 2 * m * n + 4 * m * n for m, n in blks)
    return fl, by


def roofline(cfg, prof, iters_sum, steps, n_root_steps, peaks, fp64_peak, slices=6, traffic_key=None):
    """Achieved vs peak for the kernel with the largest share of device time."""
    names = {k: v for k, v in prof.items() if v[1] > 0}
    if not names:
        return None, None
    top = max(names, key=lambda k: names[k][1])
    launches, ms = names[top]
    sec = ms * 1e-3
    hbm = peaks["hbm_gbs"]
    bf16 = peaks["bf16_tflops"]
    blks, segs = blocks_of(cfg)
    el = numel(cfg)
    gbytes = 2 if cfg["grad_dtype"] == "bf16" else 4
    work = None
    if top.startswith("newton_step"):
        a, b, c = newton_flops(cfg, iters_sum, per_kernel=True)
        fl = {"newton_step_a": a, "newton_step_b": b, "newton_step_c": c}[top]
        work = ("tensor", fl / 1e12 / sec, fp64_peak, "TFLOP/s", fl / max(launches, 1),
                "cuBLAS DGEMM (fp64) measured in this run")
    elif top.startswith("ozaki_step"):
        a, b, c = ozaki_ops(cfg, iters_sum, slices, per_kernel=True)
        ops = {"ozaki_step_a": a, "ozaki_step_b": b, "ozaki_step_c": c}[top]
        work = ("tensor", ops / 1e12 / sec, 2 * bf16, "TOP/s", ops / max(launches, 1),
                "MEASURED_PEAKS.json bf16_tflops (burst) x 2, the int8 : bf16 dense ratio")
    elif top in ("stats_tc", "apply_y_tc", "apply_p_tc"):
        fl, by = tc_work(cfg, top)
        fl, by = fl * launches, by * launches
        ft, fh = fl / 1e12 / sec / bf16, by / 1e9 / sec / hbm
        if ft >= fh:
            work = ("tensor", fl / 1e12 / sec, bf16, "TFLOP/s", fl / launches,
                    "MEASURED_PEAKS.json bf16_tflops (burst)")
        else:
            work = ("hbm", by / 1e9 / sec, hbm, "GB/s", by / launches, "MEASURED_PEAKS.json hbm_gbs")
    elif top == "ozaki_split":
        S = -(-cfg["block_size"] // 64) * 64
        sets = 0
        for (n, prods), k in zip(matrix_sizes(cfg), iters_sum):
            k = k if k >= 0 else -1 - k
            sets += 3 * n_root_steps + k * (5 if prods == 4 else 4)   # X T M at the start; X T2 (T4) M T per step
        by = sets * S * S * (8 + slices)                              # read float64, write the slices
        work = ("hbm", by / 1e9 / sec, hbm, "GB/s", by / max(launches, 1), "MEASURED_PEAKS.json hbm_gbs")
    elif top == "newton_lanczos":
        by = sum(12 * 4 * n * n for n, _ in matrix_sizes(cfg)) * n_root_steps   # 12 matvecs, fp32 operator
        work = ("hbm", by / 1e9 / sec, hbm, "GB/s", by / max(launches, 1), "MEASURED_PEAKS.json hbm_gbs")
    elif top == "update":
        by = el * (4 + 8 + (8 if cfg["momentum"] else 0)) * steps
        work = ("hbm", by / 1e9 / sec, hbm, "GB/s", by / max(launches, 1), "MEASURED_PEAKS.json hbm_gbs")
    elif top in ("dnorm", "diag_update", "check_finite", "gather"):
        per = {"dnorm": gbytes + 4, "diag_update": gbytes + 8, "check_finite": gbytes,
               "gather": gbytes + (6 if gbytes == 4 else 2)}[top]
        by = el * per * steps
        work = ("hbm", by / 1e9 / sec, hbm, "GB/s", by / max(launches, 1), "MEASURED_PEAKS.json hbm_gbs")
    if work is None:
        return top, None
    bound, ach, peak, unit, per_launch, src = work
    tr = TRAFFIC_PER_LAUNCH.get((traffic_key, top)) if traffic_key else None
    return top, {"kernel": top, "bound": bound, "achieved": round(ach, 3), "peak": round(peak, 2),
                 "unit": unit, "frac": round(ach / peak, 4), "traffic": tr,
                 "algorithmic_per_launch": per_launch, "launches": launches,
                 "avg_launch_ms": round(ms / launches, 5), "peak_source": src}


# ---------------------------------------------------------------------------
# CPU legs (oracle): the baseline line and the reference arm
# ---------------------------------------------------------------------------
def oracle_sample(cfg, n_steps):
    """Time the fp64 oracle on the full workload: n_steps of stats + apply and
    one root step; returns (seconds per step amortised over the root
    interval, description)."""
    from oracle import ShampooOracle
    o = ShampooOracle(cfg["shapes"], cfg["block_size"], cfg["beta2"], cfg["eps"], cfg["p"],
                      cfg["graft"], cfg["momentum"])
    W = [w.astype(np.float64) for w in wl.make_params(cfg["shapes"], cfg["seed"])]
    g = wl.make_grads(cfg["shapes"], cfg["seed"], 0, cfg["grad_std"], cfg["grad_dtype"])
    o.update_stats(g)
    t0 = time.perf_counter()
    o.compute_roots()
    t_root = time.perf_counter() - t0
    t0 = time.perf_counter()
    for t in range(n_steps):
        o.update_stats(g)
        W = o.apply(W, g, cfg["lr"])
    t_sa = (time.perf_counter() - t0) / n_steps
    return t_sa + t_root / cfg["root_interval"], t_root, t_sa


def pages_design_root_ms(cfg, n_sample=4):
    """The pages' root route on host cores: fp64 coupled Newton (the
    oracle's CPU copy) on the first n_sample statistics after 2 steps,
    extrapolated to every statistic of the set by n^3."""
    from oracle import ShampooOracle, coupled_newton_inverse_root
    o = ShampooOracle(cfg["shapes"], cfg["block_size"], cfg["beta2"], cfg["eps"], cfg["p"],
                      cfg["graft"], cfg["momentum"])
    for t in range(2):
        o.update_stats(wl.make_grads(cfg["shapes"], cfg["seed"], t, cfg["grad_std"], cfg["grad_dtype"]))
    mats = o.matrices()
    t0 = time.perf_counter()
    done = 0.0
    for A, p in mats[:n_sample]:
        coupled_newton_inverse_root(A, cfg["eps"], p)
        done += A.shape[0] ** 3
    el = time.perf_counter() - t0
    total = sum(A.shape[0] ** 3 for A, _ in mats)
    return el * total / done * 1e3


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def reference_arm(args, cfg, rank, world):
    if rank != 0:
        return 0
    sizes = matrix_sizes(cfg)
    from oracle import ShampooOracle
    o = ShampooOracle(cfg["shapes"], cfg["block_size"], cfg["beta2"], cfg["eps"], cfg["p"],
                      cfg["graft"], cfg["momentum"])
    W = [w.astype(np.float64) for w in wl.make_params(cfg["shapes"], cfg["seed"])]
    grads = [wl.make_grads(cfg["shapes"], cfg["seed"], t, cfg["grad_std"], cfg["grad_dtype"])
             for t in range(2)]
    for t in range(args.warmup):
        W = o.step(W, grads[t % 2], cfg["lr"], t == 0)
    t0 = time.perf_counter()
    n_root = 0
    for j in range(args.steps):
        r = j % cfg["root_interval"] == 0
        n_root += r
        W = o.step(W, grads[j % 2], cfg["lr"], r)
    el = time.perf_counter() - t0
    # The flops credited are the CUDA arm's: stats + apply per step and, per
    # root step, the Newton products at the iteration count the CPU coupled
    # Newton needs, here the mean over the first four statistics.
    from oracle import coupled_newton_inverse_root
    ks = [coupled_newton_inverse_root(A, cfg["eps"], p)[1] for A, p in o.matrices()[:4]]
    k = int(round(sum(ks) / len(ks)))
    fl = args.steps * (stats_flops(cfg) + apply_flops(cfg)) + n_root * newton_flops(cfg, [k] * len(sizes))
    val = fl / el / 1e12
    cores = blas_threads()
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": args.config, "params": numel(cfg),
                                            "block_size": cfg["block_size"]},
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"{args.steps} full oracle steps ({n_root} with roots by eigh)"},
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# the batched inverse-root kernel on its own (256 SPD 512 x 512, p = 4 and 2)
# ---------------------------------------------------------------------------
def roots_bench(args):
    import torch
    from shampoo_second_order_b200 import batched_inverse_root
    c = wl.ROOTS_CONFIG
    batch = args.batch or c["batch"]
    A, lam = wl.spd_batch(batch, c["n"], c["seed"], c["log10_kappa"])
    dev = torch.device("cuda", 0)
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        dA = torch.from_numpy(A.astype(np.float32)).to(dev)
        flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)
        fp64_peak = fp64_peak_tflops(torch, dev)
    n = c["n"]
    flops = 0
    ev = []
    for j in range(args.warmup + args.steps):
        timed = j >= args.warmup
        with torch.cuda.stream(stream):
            flush.zero_()
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record(stream)
            its = []
            for p in c["ps"]:
                X, it = batched_inverse_root(dA, p, c["eps"], c["tol"], stream=stream, method=args.roots,
                                             slices=args.slices)
                its.append((p, it))
            e.record(stream)
        stream.synchronize()
        if timed:
            ev.append((s, e))
            for p, it in its:
                k = it.cpu().numpy()
                k = np.where(k >= 0, k, -1 - k)
                # the first step's X0 T0 is a scaled copy, not a product
                flops += (int(k.sum()) * (4 if p == 4 else 3) - int((k > 0).sum())) * n * n * (n + 1)
    ms = sum(s.elapsed_time(e) for s, e in ev)
    val = flops / (ms * 1e-3) / 1e12
    line = {"metric": METRIC, "value": val, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "batched_roots_512", "batch": batch, "n": n, "p": list(c["ps"]),
                       "tol": c["tol"], "l2": "flushed between steps (256 MiB write)",
                       "newton_products": (args.roots if args.roots == "fp64"
                                           else f"int8-emulated fp64, {args.slices} slices")},
            "roofline": {"kernel": "newton (all launches of one call)", "bound": "tensor",
                         "achieved": round(val, 3), "peak": round(fp64_peak, 2), "unit": "TFLOP/s",
                         "frac": round(val / fp64_peak, 4), "traffic": None,
                         "peak_source": "cuBLAS DGEMM measured in this run"}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# the CUDA arm
# ---------------------------------------------------------------------------
def shard_bench(args, cfg, rank, world, local):
    """Block-sharded data parallelism: one parameter set, each rank owning a
    share of the parameters (shampoo_plan_shards), gradients reduce-scattered
    to their owners and updated weights all-gathered, every step inside the
    timed region.  value = the whole set's work / the slowest rank's time."""
    import torch
    import torch.distributed as dist
    from shampoo_second_order_b200.sharded import ShardedShampoo
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300))
    stream = torch.cuda.Stream(device=dev, priority=-1)
    shapes = cfg["shapes"]
    gdt = torch.bfloat16 if cfg["grad_dtype"] == "bf16" else torch.float32
    interval = cfg["root_interval"]
    W0 = wl.make_params(shapes, cfg["seed"])
    NG = 2
    with torch.cuda.stream(stream):
        W = [torch.from_numpy(w).to(dev) for w in W0]
        G = [[torch.from_numpy(g).to(dev).to(gdt)
              for g in wl.make_grads(shapes, cfg["seed"] + 17 * rank, t, cfg["grad_std"], cfg["grad_dtype"])]
             for t in range(NG)]
        flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)
    stream.synchronize()
    opt = ShardedShampoo(shapes, cfg["block_size"], cfg["beta2"], cfg["eps"], cfg["p"], cfg["graft"],
                         cfg["momentum"], cfg["grad_dtype"], interval, stream=stream)
    with torch.cuda.stream(stream):
        for t in range(args.warmup):
            opt.step(W, G[t % NG], cfg["lr"], t == 0)
    stream.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    iters = None
    with torch.cuda.stream(stream):
        for j in range(args.steps):
            flush.zero_()
            ev[j][0].record(stream)
            roots = j % interval == 0
            opt.step(W, G[j % NG], cfg["lr"], roots)
            ev[j][1].record(stream)
            if roots and opt.local is not None:
                its = opt.local.root_iterations()
                iters = its if iters is None else [a + b for a, b in zip(iters, its)]
    stream.synchronize()
    ms = max_over_ranks(sum(s.elapsed_time(e) for s, e in ev), dist if world > 1 else None, dev)
    sub = dict(cfg, shapes=[shapes[i] for i in opt.mine])
    newton = newton_flops(sub, iters) if iters else 0
    if world > 1:
        t = torch.tensor([float(newton)], dtype=torch.float64, device=dev)
        dist.all_reduce(t)
        newton = float(t.item())
    flops = args.steps * (stats_flops(cfg) + apply_flops(cfg)) + newton
    if rank == 0:
        line = {"metric": METRIC, "value": flops / (ms * 1e-3) / 1e12, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
                "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f32/f64",
                "data": "synthetic",
                "config": {"workload": args.config, "params": numel(cfg), "block_size": cfg["block_size"],
                           "grad_dtype": cfg["grad_dtype"], "root_interval": interval,
                           "parallelism": f"block-sharded dp{world}",
                           "collective_bytes_per_rank_step": opt.collective_bytes_per_step(),
                           "planned_cost_balance": round(min(opt.planned_cost) / max(opt.planned_cost), 4),
                           "l2": "flushed between steps (256 MiB write)"}}
        print(json.dumps(line), flush=True)
    opt.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--config", default="transformer_layer_b512",
                    choices=sorted(wl.CONFIGS) + ["batched_roots_512"])
    ap.add_argument("--batch", type=int, default=None,
                    help="batched_roots_512 only: number of matrices (default 256)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-async", action="store_true")
    ap.add_argument("--roots", default="fp64", choices=["fp64", "int8"],
                    help="Newton products in float64 or emulated on the int8 tensor cores")
    ap.add_argument("--slices", type=int, default=6)
    ap.add_argument("--shard", action="store_true",
                    help="one parameter set split over the ranks by owner (strong scaling, with the "
                         "gradient reduce-scatter and weight all-gather)")
    ap.add_argument("--one-sided-embedding", action="store_true",
                    help="keep only R for embedding-like weights (rows >= 16 x cols)")
    args = ap.parse_args()
    if args.config == "batched_roots_512":
        return roots_bench(args)
    cfg = wl.CONFIGS[args.config]
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    if args.warmup < 3:
        args.warmup = 3

    if args.impl == "reference":
        return reference_arm(args, cfg, rank, world)
    if args.shard:
        return shard_bench(args, cfg, rank, world, local)

    # CPU baseline first (rank 0, N = 1 only), before any GPU work
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        t_step, t_root, t_sa = oracle_sample(cfg, 2)
        cpu = {"t_step_s": t_step, "t_root_s": t_root, "t_stats_apply_s": t_sa,
               "pages_root_ms": pages_design_root_ms(cfg)}

    import torch
    import torch.distributed as dist
    from shampoo_second_order_b200 import Shampoo

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300))

    # the steps' stream outranks the library's root stream (lowest priority),
    # so asynchronous root work yields to the steps
    stream = torch.cuda.Stream(device=dev, priority=-1)
    peaks, peak_src = measured_peaks()
    with torch.cuda.stream(stream):
        fp64_peak = fp64_peak_tflops(torch, dev)
    stream.synchronize()

    shapes = cfg["shapes"]
    gdt = torch.bfloat16 if cfg["grad_dtype"] == "bf16" else torch.float32
    W0 = wl.make_params(shapes, cfg["seed"] + 17 * rank)
    NG = 4
    host_grads = [wl.make_grads(shapes, cfg["seed"] + 17 * rank, t, cfg["grad_std"], cfg["grad_dtype"])
                  for t in range(NG)]
    with torch.cuda.stream(stream):
        W = [torch.from_numpy(w).to(dev) for w in W0]
        G = [[torch.from_numpy(g).to(dev).to(gdt) for g in gs] for gs in host_grads]
        flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)
    stream.synchronize()

    opt = Shampoo(shapes, cfg["block_size"], cfg["beta2"], cfg["eps"], cfg["p"], cfg["graft"],
                  cfg["momentum"], cfg["grad_dtype"], stream=stream)
    opt.set_root_method(args.roots, args.slices)
    one_sided = []
    if args.one_sided_embedding:
        for i, s_ in enumerate(shapes):
            if len(s_) == 2 and s_[0] >= 16 * s_[1]:
                opt.set_one_sided(i, "right")
                one_sided.append(i)
        cfg = dict(cfg, right_only=one_sided)   # the work model counts what is computed
    lr = cfg["lr"]
    interval = cfg["root_interval"]

    def step(gs, roots):
        opt.update_stats(gs)
        if roots:
            opt.compute_roots()
        opt.apply(W, gs, lr)

    for t in range(args.warmup):
        step(G[t % NG], t == 0)
    stream.synchronize()

    # ---- timed region: device-resident inputs ----
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    uuid = gpu_uuid(torch, dev)
    clocks = ClockSampler(uuid, local)
    opt.profile_enable(True)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    iters_sum = [0] * opt.num_matrices()
    n_root = 0
    with torch.cuda.stream(stream):
        for j in range(args.steps):
            flush.zero_()
            roots = j % interval == 0
            ev[j][0].record(stream)
            step(G[j % NG], roots)
            ev[j][1].record(stream)
            if roots:
                n_root += 1
                its = opt.root_iterations()
                iters_sum = [a + (b if b >= 0 else -1 - b) for a, b in zip(iters_sum, its)]
    stream.synchronize()
    torch.cuda.synchronize()
    clk = clocks.stop()
    prof = opt.profile_read()
    opt.profile_enable(False)
    total_ms = max_over_ranks(sum(s.elapsed_time(e) for s, e in ev), dist if world > 1 else None, dev)
    launches = sum(v[0] for v in prof.values())

    flops_rank = args.steps * (stats_flops(cfg) + apply_flops(cfg)) + newton_flops(cfg, iters_sum)
    value = job_tflops(flops_rank, world, total_ms)

    # ---- e2e: host buffers through the public API, copies pipelined ----
    # Each step's gradients come in from pinned host memory and its updated
    # weights go back out.  Uploads run on one copy stream, downloads on another
    # (PCIe is full duplex): step j+1's gradients upload while step j computes,
    # and step j's weights are snapshotted on the device (D2D) and downloaded
    # while step j+1 computes.  The whole K-step loop is timed, from before the
    # first upload to the end of the last download.  The per-step working set
    # (statistics, roots, weights, accumulator) is several times L2, so this
    # loop does not flush L2.
    e2e = None
    if not args.no_e2e:
        pin_g = [[torch.from_numpy(g).to(gdt).pin_memory() for g in gs] for gs in host_grads]
        pin_w = [[torch.empty(w.shape, dtype=torch.float32).pin_memory() for w in W0] for _ in range(2)]
        dG = [[torch.empty_like(g) for g in G[0]] for _ in range(2)]
        snap = [[torch.empty_like(w) for w in W] for _ in range(2)]
        h2d = sum(g.numel() * g.element_size() for g in pin_g[0])
        d2h = sum(w.numel() * 4 for w in pin_w[0])
        up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        K = args.steps
        up_done = [torch.cuda.Event() for _ in range(K)]
        used = [torch.cuda.Event() for _ in range(K)]      # compute finished reading dG[j % 2]
        snapped = [torch.cuda.Event() for _ in range(K)]
        down_done = [torch.cuda.Event() for _ in range(K)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        stream.synchronize()
        t0.record(stream)

        def upload(j):
            up.wait_event(t0)
            if j >= 2:
                up.wait_event(used[j - 2])
            with torch.cuda.stream(up):
                for d, h in zip(dG[j % 2], pin_g[j % NG]):
                    d.copy_(h, non_blocking=True)
            up_done[j].record(up)

        upload(0)
        for j in range(K):
            if j + 1 < K:
                upload(j + 1)
            stream.wait_event(up_done[j])
            with torch.cuda.stream(stream):
                step(dG[j % 2], j % interval == 0)
                used[j].record(stream)
                if j >= 2:
                    stream.wait_event(down_done[j - 2])
                for d, w in zip(snap[j % 2], W):
                    d.copy_(w, non_blocking=True)
                snapped[j].record(stream)
            down.wait_event(snapped[j])
            with torch.cuda.stream(down):
                for h, d in zip(pin_w[j % 2], snap[j % 2]):
                    h.copy_(d, non_blocking=True)
            down_done[j].record(down)
        stream.wait_event(down_done[K - 1])
        t1.record(stream)
        stream.synchronize()
        e2e_ms = max_over_ranks(t0.elapsed_time(t1), dist if world > 1 else None, dev)
        e2e = {"value": job_tflops(flops_rank, world, e2e_ms), "unit": UNIT,
               "ms_per_step": e2e_ms / args.steps, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "copies": "pinned host; uploads and downloads on two copy streams, overlapped with compute"}

    # ---- asynchronous roots: the same K steps with the root job queued on the
    # library's low-priority stream after step 0's statistics and installed by
    # a later apply; the region ends when the job has been installed ----
    async_line = None
    if not args.no_async:
        K = args.steps
        sev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        stream.synchronize()
        if world > 1:
            dist.barrier()
        gen0 = opt.roots_generation()
        installed_at = None
        n_jobs = 0
        with torch.cuda.stream(stream):
            a0.record(stream)
            for j in range(K):
                flush.zero_()
                sev[j][0].record(stream)
                opt.update_stats(G[j % NG])
                if j % interval == 0:
                    n_jobs += int(opt.compute_roots_async())
                opt.apply(W, G[j % NG], lr)
                sev[j][1].record(stream)
                if installed_at is None and opt.roots_generation() > gen0:
                    installed_at = j
            if opt.install_roots(wait=True) and installed_at is None:
                installed_at = K
            a1.record(stream)
        stream.synchronize()
        async_ms = max_over_ranks(a0.elapsed_time(a1), dist if world > 1 else None, dev)
        its = opt.root_iterations()
        fl = K * (stats_flops(cfg) + apply_flops(cfg)) + n_jobs * newton_flops(
            cfg, [b if b >= 0 else -1 - b for b in its])
        st_ms = sorted(s_.elapsed_time(e_) for s_, e_ in sev)
        async_line = {"value": job_tflops(fl, world, async_ms), "unit": UNIT, "ms_per_step": async_ms / K,
                      "root_jobs": n_jobs, "installed_at_step": installed_at,
                      "step_ms_median": st_ms[len(st_ms) // 2], "step_ms_max": st_ms[-1],
                      "sync_step_ms_max": max(s_.elapsed_time(e_) for s_, e_ in ev),
                      "streams": "steps at high priority; roots on the library's lowest-priority stream"}

    # the committed DRAM traffic holds only for the workload and mode it was captured on
    tkey = args.config if (args.roots == "fp64" and not args.one_sided_embedding) else None
    top, roof = roofline(cfg, prof, iters_sum, args.steps, n_root, peaks, fp64_peak, args.slices, tkey)

    if rank == 0:
        phase = {}
        for k, (n, ms) in sorted(prof.items(), key=lambda kv: -kv[1][1]):
            phase[k] = {"launches": n, "ms": round(ms, 4), "share": round(ms / max(total_ms, 1e-9), 4)}
        cpu_line = None
        if cpu is not None:
            fl_amort = stats_flops(cfg) + apply_flops(cfg) + newton_flops(cfg, iters_sum) / max(args.steps, 1)
            cpu_line = {"value": fl_amort / cpu["t_step_s"] / 1e12, "unit": UNIT, "cores": blas_threads(),
                        "kind": "oracle",
                        "sample": ("fp64 numpy oracle on the full workload: 2 steps of stats+apply and 1 "
                                   "root step (eigh), amortised over the root interval"),
                        "ms_per_step": cpu["t_step_s"] * 1e3,
                        "root_step_ms_eigh": cpu["t_root_s"] * 1e3,
                        "root_step_ms_pages_design": round(cpu["pages_root_ms"], 1),
                        "pages_design": ("fp64 coupled Newton on host cores for every statistic "
                                         "(timed on 4, extrapolated by n^3)")}
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32/f64", "data": "synthetic",
            "config": {"workload": args.config, "params": numel(cfg), "block_size": cfg["block_size"],
                       "grad_dtype": cfg["grad_dtype"], "root_interval": interval,
                       "newton_products": (args.roots if args.roots == "fp64"
                                           else f"int8-emulated fp64, {args.slices} slices"),
                       "one_sided_right": [list(shapes[i]) for i in one_sided],
                       "one_sided_right": [list(shapes[i]) for i in one_sided],
                       "root_steps_timed": n_root, "l2": "flushed between steps (256 MiB write)",
                       "parallelism": f"replicas x{world}"},
            "roofline": roof, "cpu_baseline": cpu_line, "e2e": e2e, "async_roots": async_line,
            "gpu_launches": launches,
            "clocks": clk, "kernels": phase, "fp64_gemm_peak_tflops": round(fp64_peak, 2),
            "peaks_source": peak_src,
            "flops_per_step": {"stats": stats_flops(cfg), "apply": apply_flops(cfg),
                               "roots_per_root_step": newton_flops(cfg, iters_sum) / max(n_root, 1)},
        }
        print(json.dumps(line), flush=True)
    opt.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
