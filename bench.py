#!/usr/bin/env python
"""Benchmark of the Shampoo optimizer step (statistics + inverse roots +
grafted apply) on B200, through the library's C-ABI.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cuda|reference]
                  [--config transformer_big_b1024]

The default workload is the largest single-GPU parameter set,
Transformer-big-shaped (285.2M parameters, b = 1024, fp32 gradients,
momentum 0.9, roots every 100 steps).  A step is update_stats, compute_roots
on root steps, and apply, on one fixed seeded gradient set per step.  The
timed region runs K steps with the root computation on the first (one root
step per K <= root_interval), every call bracketed by CUDA events on the
optimizer's stream, L2 flushed (a 256 MiB write) between steps outside the
events, inputs resident in HBM.  The reported step is the amortised one:

    ms_per_step = t_stats + t_apply + t_roots / root_interval

with t_stats and t_apply the mean per-step times of the two calls and t_roots
the time of the root computation (the pages recompute roots only every few
hundred steps, at a cost up to ~100 training steps).  `value` is the
credited work of one amortised step over ms_per_step.

With N > 1 (torchrun) the default is the block-sharded data-parallel step:
one parameter set, each rank owning whole parameters, gradients
reduce-scattered (float32) to their owners and updated weights all-gathered,
every collective inside the timed region (strong scaling); --replicas runs
an independent copy per rank instead.  Job times are the max over ranks.
Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
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
    # the statistics GEMM (single-CTA 128x128 tiles, 2-term split with four
    # products, two-level accumulation over four TMEM accumulators, both
    # gradient planes of a panel per TMA box): 231.5 MB for the 20 blocks of
    # Transformer-big layer 0 (ncu, one launch, `python -m
    # shampoo_second_order_b200.run_steps`, kernel of d53cb9c; the later edits
    # of k_tc.cu left this path's loads and stores unchanged), scaled by the
    # block count to the 272 identical 1024 x 1024 blocks of a full launch
    ("transformer_big_b1024", "stats_tc"): 231501056 * 272 // 20,
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


# Credited coupled-Newton steps per statistic and root step.  Both arms (the
# CUDA path and the oracle reference, whose roots come from an
# eigendecomposition) credit a root step with the same work -- this many
# Newton steps of every statistic -- so that the ratio of their values is
# the ratio of their step times.  Each count is the mean number of steps per
# statistic the device's scaled iteration ran on the workload's first root
# step, rounded; the work the device executed is reported beside the value.
NEWTON_STEPS_CREDIT = {"single_64x32": 6, "transformer_layer_b512": 5, "transformer_big_b1024": 5,
                       "resnet50_b128": 5}


def credit_iters(cfg, k):
    """k steps for every statistic that is iterated (0 for a dropped factor of
    a one-sided block), in library order."""
    out = []
    for sd in block_sides(cfg):
        out += [0 if sd == 2 else k, k]
    blks, segs = blocks_of(cfg)
    return out + [k] * len(segs)


def credited_step_flops(cfg, name):
    """Work credited to one amortised step: statistics and apply, plus the
    credited root work over the root interval."""
    roots = newton_flops(cfg, credit_iters(cfg, NEWTON_STEPS_CREDIT.get(name, 5)))
    return stats_flops(cfg) + apply_flops(cfg) + roots / cfg["root_interval"]


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
def flat_views(flat, shapes):
    """Contiguous per-parameter views of a flat 1-D tensor that holds the
    parameters back to back, row-major, in the order of `shapes`."""
    out, o = [], 0
    for sh in shapes:
        n = int(np.prod(sh))
        out.append(flat[o:o + n].view(*sh))
        o += n
    if o != flat.numel():
        raise ValueError(f"flat buffer holds {flat.numel()} elements, the shapes {o}")
    return out


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    # no measured file: an earlier copy/cuBLAS measurement on B200s of this kind
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "fallback": True}, "fallback"


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
    planes = 2 if f32 else 1
    T = (b + 127) // 128
    tri = T * (T + 1) // 2 * 128 * 128 * 4          # bytes of one statistic's upper tiles
    if kernel == "stats_tc":
        passes = 4 if f32 else 1
        fl = sum((0 if sd else m * (m + 1) * n) + n * (n + 1) * m
                 for (m, n), sd in zip(blks, block_sides(cfg))) * passes
        by = sum(2 * planes * m * n for m, n in blks) + len(blks) * 2 * 2 * tri
    elif kernel == "apply_y_tc":
        passes = 3 if f32 else 2
        fl = sum(2 * m * n * n for m, n in blks) * passes
        by = sum(2 * planes * m * n + 2 * 2 * n * n + 2 * 2 * m * n for m, n in blks)
    else:   # apply_p_tc
        fl = sum(2 * m * m * n for m, n in blks) * 3
        by = sum(2 * 2 * m * m + 2 * 2 * m * n + 4 * m * n for m, n in blks)
    return fl, by


ROOT_KERNELS = ("newton_", "ozaki_", "split_roots")
# kernels the library runs on its second stream, beside the tensor-core GEMMs
# of the same call: their event spans include waiting for SMs the GEMMs hold,
# so they are not exclusive time and never the dominant kernel
SIDE_STREAM_KERNELS = ("check_finite", "diag_update", "stats_segments", "precond_seg")


def is_root_kernel(name):
    return name.startswith(ROOT_KERNELS)


def kernel_roof(cfg, name, launches, ms, iters_sum, steps, n_root_steps, peaks, fp64_peak, slices=6,
                traffic_key=None):
    """Achieved vs peak of one kernel over its launches in the timed region:
    algorithmic work (the work model above) over its CUDA-event time, against
    the roof that binds it.  None for kernels without a work model."""
    if launches <= 0 or ms <= 0:
        return None
    sec = ms * 1e-3
    hbm = peaks["hbm_gbs"]
    bf16 = peaks["bf16_tflops"]
    el = numel(cfg)
    gbytes = 2 if cfg["grad_dtype"] == "bf16" else 4
    work = None
    if name.startswith("newton_step"):
        a, b, c = newton_flops(cfg, iters_sum, per_kernel=True)
        fl = {"newton_step_a": a, "newton_step_b": b, "newton_step_c": c}[name]
        work = ("tensor", fl / 1e12 / sec, fp64_peak, "TFLOP/s", fl / launches,
                "cuBLAS DGEMM (fp64) measured in this run")
    elif name.startswith("ozaki_step"):
        a, b, c = ozaki_ops(cfg, iters_sum, slices, per_kernel=True)
        ops = {"ozaki_step_a": a, "ozaki_step_b": b, "ozaki_step_c": c}[name]
        work = ("tensor", ops / 1e12 / sec, 2 * bf16, "TOP/s", ops / launches,
                "MEASURED_PEAKS.json bf16_tflops (burst) x 2, the int8 : bf16 dense ratio")
    elif name in ("stats_tc", "apply_y_tc", "apply_p_tc"):
        fl, by = tc_work(cfg, name)
        fl, by = fl * launches, by * launches
        ft, fh = fl / 1e12 / sec / bf16, by / 1e9 / sec / hbm
        if ft >= fh:
            work = ("tensor", fl / 1e12 / sec, bf16, "TFLOP/s", fl / launches,
                    "MEASURED_PEAKS.json bf16_tflops (burst)")
        else:
            work = ("hbm", by / 1e9 / sec, hbm, "GB/s", by / launches, "MEASURED_PEAKS.json hbm_gbs")
    elif name == "ozaki_split":
        S = -(-cfg["block_size"] // 64) * 64
        sets = 0
        for (n, prods), k in zip(matrix_sizes(cfg), iters_sum):
            k = k if k >= 0 else -1 - k
            sets += 3 * n_root_steps + k * (5 if prods == 4 else 4)   # X T M at the start; X T2 (T4) M T per step
        by = sets * S * S * (8 + slices)                              # read float64, write the slices
        work = ("hbm", by / 1e9 / sec, hbm, "GB/s", by / launches, "MEASURED_PEAKS.json hbm_gbs")
    elif name == "newton_lanczos":
        by = sum(12 * 4 * n * n for n, _ in matrix_sizes(cfg)) * n_root_steps   # 12 matvecs, fp32 operator
        work = ("hbm", by / 1e9 / sec, hbm, "GB/s", by / launches, "MEASURED_PEAKS.json hbm_gbs")
    elif name == "update":
        by = el * (4 + 8 + (8 if cfg["momentum"] else 0)) * steps
        work = ("hbm", by / 1e9 / sec, hbm, "GB/s", by / launches, "MEASURED_PEAKS.json hbm_gbs")
    elif name in ("dnorm", "diag_update", "check_finite", "gather"):
        per = {"dnorm": gbytes + 4, "diag_update": gbytes + 8, "check_finite": gbytes,
               "gather": gbytes + (4 if gbytes == 4 else 2)}[name]
        by = el * per * steps
        work = ("hbm", by / 1e9 / sec, hbm, "GB/s", by / launches, "MEASURED_PEAKS.json hbm_gbs")
    if work is None:
        return None
    bound, ach, peak, unit, per_launch, src = work
    if peaks.get("fallback"):
        src = src.replace("MEASURED_PEAKS.json", "fallback peaks:")
    tr = TRAFFIC_PER_LAUNCH.get((traffic_key, name)) if traffic_key else None
    out = {"kernel": name, "bound": bound, "achieved": round(ach, 3), "peak": round(peak, 2),
           "unit": unit, "frac": round(ach / peak, 4), "traffic": tr,
           "algorithmic_per_launch": per_launch, "launches": launches,
           "avg_launch_ms": round(ms / launches, 5), "peak_source": src}
    if unit == "TFLOP/s" and "bf16" in src and "bf16_tflops_sustained" in peaks:
        out["frac_of_sustained"] = round(ach / peaks["bf16_tflops_sustained"], 4)
    return out


def amortised_ms(prof, steps, n_root_steps, interval):
    """Per kernel, its device time per amortised step: per-step kernels over
    the timed steps, root kernels over the root steps and the root interval."""
    out = {}
    for k, (n, ms) in prof.items():
        if is_root_kernel(k):
            out[k] = ms / max(n_root_steps, 1) / interval
        else:
            out[k] = ms / max(steps, 1)
    return out


def roofline(cfg, prof, iters_sum, steps, n_root_steps, peaks, fp64_peak, slices=6, traffic_key=None):
    """The roofline of the kernel with the largest share of the amortised
    step, and the same figures for every kernel with a work model."""
    names = {k: v for k, v in prof.items() if v[1] > 0}
    if not names:
        return None, None, {}
    am = amortised_ms(names, steps, n_root_steps, cfg["root_interval"])
    main = {k: v for k, v in am.items() if k not in SIDE_STREAM_KERNELS} or am
    top = max(main, key=main.get)
    every = {}
    for k, (n, ms) in names.items():
        r = kernel_roof(cfg, k, n, ms, iters_sum, steps, n_root_steps, peaks, fp64_peak, slices, traffic_key)
        if r is not None:
            every[k] = {x: r[x] for x in ("bound", "achieved", "unit", "frac", "avg_launch_ms")}
            if k in SIDE_STREAM_KERNELS:
                every[k]["note"] = "event span on the second stream, beside the GEMMs"
    return top, kernel_roof(cfg, top, *names[top], iters_sum, steps, n_root_steps, peaks, fp64_peak, slices,
                            traffic_key), every


# ---------------------------------------------------------------------------
# CPU legs (oracle): the baseline line and the reference arm
# ---------------------------------------------------------------------------
SAMPLE_PARAMS = 40_000_000   # sets larger than this are sampled on host cores


def sample_cfg(cfg):
    """(workload the oracle runs, its description, stats+apply scale, root
    scale).  A set small enough is run whole (scales 1).  A larger one is
    sampled by its first layer -- its first six weights, whose blocks have
    the shapes of every other layer's and of the blocked embedding -- and the
    oracle's times are scaled to the whole set by the work model: statistics
    and apply by their flops, the root step by the sum of n^3 over the
    statistics (an eigendecomposition's cost)."""
    if numel(cfg) <= SAMPLE_PARAMS:
        return cfg, "the whole parameter set", 1.0, 1.0
    sub = dict(cfg, shapes=cfg["shapes"][:6])
    sa = (stats_flops(cfg) + apply_flops(cfg)) / (stats_flops(sub) + apply_flops(sub))
    cube = lambda c: sum(n ** 3 for n, _ in matrix_sizes(c))
    return sub, (f"layer 0 ({len(sub['shapes'])} weights, {len(blocks_of(sub)[0])} blocks, "
                 f"{len(matrix_sizes(sub))} statistics), scaled to the whole set by the work model "
                 f"(x{sa:.2f} for statistics + apply, x{cube(cfg) / cube(sub):.2f} for roots)"), \
        sa, cube(cfg) / cube(sub)


def oracle_sample(cfg, n_steps=2):
    """Time the fp64 oracle on a bounded sample of the workload: one root
    step (eigh) and n_steps of statistics + apply.  Returns (ms per amortised
    step of the whole workload, root ms, stats+apply ms, description)."""
    from oracle import ShampooOracle
    sub, what, sa, rs = sample_cfg(cfg)
    o = ShampooOracle(sub["shapes"], sub["block_size"], sub["beta2"], sub["eps"], sub["p"],
                      sub["graft"], sub["momentum"])
    W = [w.astype(np.float64) for w in wl.make_params(sub["shapes"], sub["seed"])]
    g = wl.make_grads(sub["shapes"], sub["seed"], 0, sub["grad_std"], sub["grad_dtype"])
    o.update_stats(g)
    t0 = time.perf_counter()
    o.compute_roots()
    t_root = (time.perf_counter() - t0) * rs
    t0 = time.perf_counter()
    for t in range(n_steps):
        o.update_stats(g)
        W = o.apply(W, g, cfg["lr"])
    t_sa = (time.perf_counter() - t0) / n_steps * sa
    desc = (f"fp64 numpy oracle on {what}: {n_steps} steps of statistics + apply and 1 root step "
            f"(eigh), amortised over the root interval of {cfg['root_interval']}")
    return (t_sa + t_root / cfg["root_interval"]) * 1e3, t_root * 1e3, t_sa * 1e3, desc


def pages_design_root_ms(cfg, n_sample=4):
    """The pages' root route on host cores: fp64 coupled Newton (the
    oracle's CPU copy) on the first n_sample statistics after 2 steps,
    extrapolated to every statistic of the set by n^3."""
    from oracle import ShampooOracle, coupled_newton_inverse_root
    sub, _, _, _ = sample_cfg(cfg)
    o = ShampooOracle(sub["shapes"], sub["block_size"], sub["beta2"], sub["eps"], sub["p"],
                      sub["graft"], sub["momentum"])
    for t in range(2):
        o.update_stats(wl.make_grads(sub["shapes"], sub["seed"], t, sub["grad_std"], sub["grad_dtype"]))
    mats = o.matrices()
    t0 = time.perf_counter()
    done = 0.0
    for A, p in mats[:n_sample]:
        coupled_newton_inverse_root(A, cfg["eps"], p)
        done += A.shape[0] ** 3
    el = time.perf_counter() - t0
    total = sum(n ** 3 for n, _ in matrix_sizes(cfg))
    return el * total / done * 1e3


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def reference_arm(args, cfg, rank, world):
    """The oracle as the reference arm, on host cores, rank 0 only: W warm-up
    and K timed steps of the sampled workload (roots on the steps the CUDA
    arm roots on), each call timed, scaled to the whole workload and
    amortised exactly like the CUDA arm's step; credited the same work."""
    if rank != 0:
        return 0
    from oracle import ShampooOracle
    sub, what, sa, rs = sample_cfg(cfg)
    o = ShampooOracle(sub["shapes"], sub["block_size"], sub["beta2"], sub["eps"], sub["p"],
                      sub["graft"], sub["momentum"])
    W = [w.astype(np.float64) for w in wl.make_params(sub["shapes"], sub["seed"])]
    grads = [wl.make_grads(sub["shapes"], sub["seed"], t, sub["grad_std"], sub["grad_dtype"])
             for t in range(2)]
    for t in range(args.warmup):
        W = o.step(W, grads[t % 2], cfg["lr"], t == 0)
    t_st, t_ap, t_rt = [], [], []
    t0 = time.perf_counter()
    for j in range(args.steps):
        g = grads[j % 2]
        a = time.perf_counter()
        o.update_stats(g)
        b = time.perf_counter()
        t_st.append(b - a)
        if j % cfg["root_interval"] == 0:
            o.compute_roots()
            c = time.perf_counter()
            t_rt.append(c - b)
            b = c
        W = o.apply(W, g, cfg["lr"])
        t_ap.append(time.perf_counter() - b)
    wall = time.perf_counter() - t0
    t_stats = statistics.mean(t_st) * sa * 1e3
    t_apply = statistics.mean(t_ap) * sa * 1e3
    t_roots = statistics.mean(t_rt) * rs * 1e3 if t_rt else 0.0
    ms = t_stats + t_apply + t_roots / cfg["root_interval"]
    val = credited_step_flops(cfg, args.config) / (ms * 1e-3) / 1e12
    cores = blas_threads()
    sample = (f"fp64 numpy oracle on {what}: {args.steps} timed steps ({len(t_rt)} with roots by eigh), "
              f"amortised like the CUDA arm; {wall:.1f} s of host time")
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": args.config, "params": numel(cfg), "block_size": cfg["block_size"],
                       "root_interval": cfg["root_interval"]},
            "t_stats_ms": t_stats, "t_apply_ms": t_apply, "t_roots_ms": t_roots,
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
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
    (float32) to their owners and updated weights all-gathered, every
    collective inside the timed region.  Steps are timed whole; the amortised
    step is t_step + (t_root_step - t_step) / root_interval on the slowest
    rank, and value = the whole set's credited work over it."""
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
    host_grads = [wl.make_grads(shapes, cfg["seed"] + 17 * rank, t, cfg["grad_std"], cfg["grad_dtype"])
                  for t in range(NG)]
    with torch.cuda.stream(stream):
        W = [torch.from_numpy(w).to(dev) for w in W0]
        G = [[torch.from_numpy(g).to(dev).to(gdt) for g in gs] for gs in host_grads]
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
    clocks = ClockSampler(gpu_uuid(torch, dev), local)
    if opt.local is not None:
        opt.local.profile_enable(True)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    iters = None
    root_steps = []
    with torch.cuda.stream(stream):
        for j in range(args.steps):
            flush.zero_()
            ev[j][0].record(stream)
            roots = j % interval == 0
            opt.step(W, G[j % NG], cfg["lr"], roots)
            ev[j][1].record(stream)
            if roots:
                root_steps.append(j)
                if opt.local is not None:
                    its = opt.local.root_iterations()
                    iters = its if iters is None else [a + b for a, b in zip(iters, its)]
    stream.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clk = clocks.stop()
    prof = opt.local.profile_read() if opt.local is not None else {}
    t = [s_.elapsed_time(e_) for s_, e_ in ev]
    plain = [x for j, x in enumerate(t) if j not in root_steps] or t
    t_n = statistics.mean(plain)
    t_r = statistics.mean([t[j] for j in root_steps]) if root_steps else t_n
    ms_rank = t_n + max(t_r - t_n, 0.0) / interval
    ms = max_over_ranks(ms_rank, dist if world > 1 else None, dev)
    total_ms = max_over_ranks(sum(t), dist if world > 1 else None, dev)
    sub = dict(cfg, shapes=[shapes[i] for i in opt.mine])
    newton = newton_flops(sub, iters) / max(len(root_steps), 1) if iters else 0.0
    launches = sum(v[0] for v in prof.values())
    if world > 1:
        x = torch.tensor([float(newton), float(launches)], dtype=torch.float64, device=dev)
        dist.all_reduce(x)
        newton, launches = float(x[0].item()), int(x[1].item())
    F = credited_step_flops(cfg, args.config)
    executed = stats_flops(cfg) + apply_flops(cfg) + newton / interval

    # end to end with host buffers, every rank alike: its gradients come in
    # from pinned host memory as one flat buffer, the sharded step runs
    # (reduce-scatter, owner step, all-gather), and the updated weights go
    # back out from a device snapshot; roots amortised as above
    e2e = None
    if not args.no_e2e:
        shapes_w = [tuple(w.shape) for w in W0]
        total = sum(int(np.prod(sh)) for sh in shapes_w)
        pin_g = []
        for gs in host_grads[:2]:
            flat = torch.empty(total, dtype=gdt).pin_memory()
            for v, g in zip(flat_views(flat, shapes_w), gs):
                v.copy_(torch.from_numpy(g).to(gdt))
            pin_g.append(flat)
        pin_w = [torch.empty(total, dtype=torch.float32).pin_memory() for _ in range(2)]
        dG_flat = [torch.empty(total, dtype=gdt, device=dev) for _ in range(2)]
        dG = [flat_views(f, shapes_w) for f in dG_flat]
        snap_flat = [torch.empty(total, dtype=torch.float32, device=dev) for _ in range(2)]
        snap = [flat_views(f, shapes_w) for f in snap_flat]
        K = args.steps
        up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        up_done = [torch.cuda.Event() for _ in range(K)]
        used = [torch.cuda.Event() for _ in range(K)]
        snapped = [torch.cuda.Event() for _ in range(K)]
        down_done = [torch.cuda.Event() for _ in range(K)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        stream.synchronize()
        if world > 1:
            dist.barrier()
        t0.record(stream)

        def upload(j):
            up.wait_event(t0)
            if j >= 2:
                up.wait_event(used[j - 2])
            with torch.cuda.stream(up):
                dG_flat[j % 2].copy_(pin_g[j % 2], non_blocking=True)
            up_done[j].record(up)

        upload(0)
        for j in range(K):
            if j + 1 < K:
                upload(j + 1)
            stream.wait_event(up_done[j])
            with torch.cuda.stream(stream):
                opt.step(W, dG[j % 2], cfg["lr"], False)
                used[j].record(stream)
                if j >= 2:
                    stream.wait_event(down_done[j - 2])
                for d, w in zip(snap[j % 2], W):
                    d.copy_(w, non_blocking=True)
                snapped[j].record(stream)
            down.wait_event(snapped[j])
            with torch.cuda.stream(down):
                pin_w[j % 2].copy_(snap_flat[j % 2], non_blocking=True)
            down_done[j].record(down)
        stream.wait_event(down_done[K - 1])
        t1.record(stream)
        stream.synchronize()
        e2e_rank = t0.elapsed_time(t1) / K + max(t_r - t_n, 0.0) / interval
        e2e_ms = max_over_ranks(e2e_rank, dist if world > 1 else None, dev)
        h2d = pin_g[0].numel() * pin_g[0].element_size()
        e2e = {"value": F / (e2e_ms * 1e-3) / 1e12, "unit": UNIT, "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": h2d * world, "d2h_bytes_per_step": total * 4 * world,
               "copies": "every rank: pinned host, its gradients up as one flat buffer and the full "
                         "updated weights down from a device snapshot, per step, on two copy streams",
               "amortisation": "K-step loop with host copies, plus (t_root_step - t_step) / root_interval"}
        del pin_g, pin_w, dG, dG_flat, snap, snap_flat

    # the roofline of rank 0's owned share (its own kernels and work model)
    roof, every = None, {}
    if rank == 0 and opt.local is not None:
        try:
            peaks, _ = measured_peaks()
            fp64_peak = fp64_peak_tflops(torch, dev)
            _, roof, every = roofline(sub, prof, iters, args.steps, len(root_steps), peaks, fp64_peak,
                                      args.slices, None)
            if roof is not None:
                roof["scope"] = "rank 0's owned parameters"
        except Exception as exc:   # a figure for the line, not a reason to stop the ranks
            roof = {"error": repr(exc)[:200]}
    if rank == 0:
        line = {"metric": METRIC, "value": F / (ms * 1e-3) / 1e12, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f32/f64",
                "data": "synthetic",
                "config": {"workload": args.config, "params": numel(cfg), "block_size": cfg["block_size"],
                           "grad_dtype": cfg["grad_dtype"], "root_interval": interval,
                           "parallelism": f"block-sharded dp{world}",
                           "amortisation": "ms_per_step = t_step + (t_root_step - t_step) / root_interval, "
                                           "slowest rank",
                           "collective_bytes_per_rank_step": opt.collective_bytes_per_step(),
                           "planned_cost_balance": round(min(opt.planned_cost) / max(opt.planned_cost), 4),
                           "l2": "flushed between steps (256 MiB write)"},
                "t_step_ms": t_n, "t_root_step_ms": t_r, "timed_region_ms": total_ms,
                "executed_tflops": executed / (ms * 1e-3) / 1e12,
                "gpu_launches": launches, "clocks": clk,
                "cpu_baseline": None, "e2e": e2e, "roofline": roof, "kernel_roofs": every}
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
    ap.add_argument("--config", default="transformer_big_b1024",
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
                    help="the block-sharded step also at N = 1 (the default for N > 1)")
    ap.add_argument("--replicas", action="store_true",
                    help="N > 1: an independent copy of the set per rank, no collective (weak scaling)")
    ap.add_argument("--one-sided-embedding", action="store_true",
                    help="keep only R for embedding-like weights (rows >= 16 x cols)")
    ap.add_argument("--gemm-tiles", default="pair", choices=["pair", "single"],
                    help="GEMM tiling: 256 x 256 CTA-pair tiles where the block side allows, or "
                         "128 x 128 single-CTA tiles")
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
    if args.shard or (world > 1 and not args.replicas):
        return shard_bench(args, cfg, rank, world, local)

    # CPU baseline first (rank 0, N = 1 only), before any GPU work
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        ms, t_root, t_sa, desc = oracle_sample(cfg, 2)
        cpu = {"ms": ms, "t_root_ms": t_root, "t_sa_ms": t_sa, "desc": desc,
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
    opt.set_gemm_tiles(args.gemm_tiles == "pair")
    one_sided = []
    if args.one_sided_embedding:
        for i, s_ in enumerate(shapes):
            if len(s_) == 2 and s_[0] >= 16 * s_[1]:
                opt.set_one_sided(i, "right")
                one_sided.append(i)
        cfg = dict(cfg, right_only=one_sided)   # the work model counts what is computed
    lr = cfg["lr"]
    interval = cfg["root_interval"]

    for t in range(args.warmup):
        opt.update_stats(G[t % NG])
        if t == 0:
            opt.compute_roots()
        opt.apply(W, G[t % NG], lr)
    stream.synchronize()

    # ---- timed region: device-resident inputs, every call between events ----
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(gpu_uuid(torch, dev), local)
    opt.profile_enable(True)
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    iters_sum = [0] * opt.num_matrices()
    root_steps = []
    with torch.cuda.stream(stream):
        for j in range(K):
            flush.zero_()
            e = ev[j]
            g = G[j % NG]
            e[0].record(stream)
            opt.update_stats(g)
            e[1].record(stream)
            if j % interval == 0:
                opt.compute_roots()
                root_steps.append(j)
            e[2].record(stream)
            opt.apply(W, g, lr)
            e[3].record(stream)
            if j in root_steps:
                its = opt.root_iterations()
                iters_sum = [a + (b if b >= 0 else -1 - b) for a, b in zip(iters_sum, its)]
    stream.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clk = clocks.stop()
    prof = opt.profile_read()
    opt.profile_enable(False)
    n_root = len(root_steps)
    t_stats = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    t_apply = statistics.mean(e[2].elapsed_time(e[3]) for e in ev)
    t_roots = statistics.mean(ev[j][1].elapsed_time(ev[j][2]) for j in root_steps) if root_steps else 0.0
    ms_rank = t_stats + t_apply + t_roots / interval
    ms = max_over_ranks(ms_rank, dist if world > 1 else None, dev)
    region_ms = max_over_ranks(sum(e[0].elapsed_time(e[3]) for e in ev), dist if world > 1 else None, dev)
    launches = sum(v[0] for v in prof.values())

    F = credited_step_flops(cfg, args.config)
    newton_exec = newton_flops(cfg, iters_sum) / max(n_root, 1)
    executed = stats_flops(cfg) + apply_flops(cfg) + newton_exec / interval
    value = job_tflops(F, world, ms)

    # ---- e2e: host buffers through the public API, copies pipelined ----
    # Each step's gradients come in from pinned host memory and its updated
    # weights go back out.  Uploads run on one copy stream, downloads on another
    # (PCIe is full duplex): step j+1's gradients upload while step j computes,
    # and step j's weights are snapshotted on the device (D2D) and downloaded
    # while step j+1 computes.  Gradients travel as one flat buffer per step
    # (the optimizer gets per-parameter views of it) and the weight snapshot
    # as another: two large copies run the link closer to its rate than one
    # copy per parameter (1.14 GB each way: 23 vs 27.5 ms on this GPU's
    # link).  The K-step loop of statistics + apply is timed from before the
    # first upload to the end of the last download; the root step moves no
    # host data, so its device time enters amortised exactly as in the
    # device-resident number.
    e2e = None
    if not args.no_e2e:
        shapes_w = [tuple(w.shape) for w in W0]
        total = sum(int(np.prod(sh)) for sh in shapes_w)
        pin_g = []
        for gs in host_grads[:2]:
            flat = torch.empty(total, dtype=gdt).pin_memory()
            for v, g in zip(flat_views(flat, shapes_w), gs):
                v.copy_(torch.from_numpy(g).to(gdt))
            pin_g.append(flat)
        pin_w = [torch.empty(total, dtype=torch.float32).pin_memory() for _ in range(2)]
        dG_flat = [torch.empty(total, dtype=gdt, device=dev) for _ in range(2)]
        dG = [flat_views(f, shapes_w) for f in dG_flat]
        snap_flat = [torch.empty(total, dtype=torch.float32, device=dev) for _ in range(2)]
        snap = [flat_views(f, shapes_w) for f in snap_flat]
        h2d = pin_g[0].numel() * pin_g[0].element_size()
        d2h = pin_w[0].numel() * 4
        up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
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
                dG_flat[j % 2].copy_(pin_g[j % 2], non_blocking=True)
            up_done[j].record(up)

        upload(0)
        for j in range(K):
            if j + 1 < K:
                upload(j + 1)
            stream.wait_event(up_done[j])
            with torch.cuda.stream(stream):
                opt.update_stats(dG[j % 2])
                opt.apply(W, dG[j % 2], lr)
                used[j].record(stream)
                if j >= 2:
                    stream.wait_event(down_done[j - 2])
                for d, w in zip(snap[j % 2], W):
                    d.copy_(w, non_blocking=True)
                snapped[j].record(stream)
            down.wait_event(snapped[j])
            with torch.cuda.stream(down):
                pin_w[j % 2].copy_(snap_flat[j % 2], non_blocking=True)
            down_done[j].record(down)
        stream.wait_event(down_done[K - 1])
        t1.record(stream)
        stream.synchronize()
        loop_ms = t0.elapsed_time(t1)
        e2e_ms = max_over_ranks(loop_ms / K + t_roots / interval, dist if world > 1 else None, dev)
        e2e = {"value": job_tflops(F, world, e2e_ms), "unit": UNIT, "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "copies": "pinned host, one flat gradient buffer up and one flat weight snapshot down per step, "
                         "on two copy streams, overlapped with compute",
               "amortisation": "K-step statistics + apply loop with host copies, plus t_roots / root_interval"}
        del pin_g, pin_w, dG, dG_flat, snap, snap_flat

    # ---- asynchronous roots: the same K steps with the root job queued on the
    # library's low-priority stream after step 0's statistics and installed by
    # a later apply; the region ends when the job has been installed ----
    async_line = None
    if not args.no_async:
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
        st_ms = sorted(s_.elapsed_time(e_) for s_, e_ in sev)
        async_line = {"ms_region": async_ms, "steps": K, "root_jobs": n_jobs, "installed_at_step": installed_at,
                      "step_ms_median": st_ms[len(st_ms) // 2], "step_ms_max": st_ms[-1],
                      "sync_step_ms_max": max(e[0].elapsed_time(e[3]) for e in ev),
                      "streams": "steps at high priority; roots on the library's lowest-priority stream"}

    # the committed DRAM traffic holds only for the workload and mode it was captured on
    tkey = (args.config if (args.roots == "fp64" and not args.one_sided_embedding and args.gemm_tiles == "pair")
            else None)
    top, roof, every = roofline(cfg, prof, iters_sum, K, n_root, peaks, fp64_peak, args.slices, tkey)

    if rank == 0:
        am = amortised_ms(prof, K, n_root, interval)
        phase = {}
        for k, (n, kms) in sorted(prof.items(), key=lambda kv: -am[kv[0]]):
            phase[k] = {"launches": n, "ms": round(kms, 4), "ms_per_amortised_step": round(am[k], 5),
                        "share": round(am[k] / max(ms_rank, 1e-9), 4)}
        cpu_line = None
        if cpu is not None:
            cpu_line = {"value": F / (cpu["ms"] * 1e-3) / 1e12, "unit": UNIT, "cores": blas_threads(),
                        "kind": "oracle", "sample": cpu["desc"], "ms_per_step": cpu["ms"],
                        "root_step_ms_eigh": cpu["t_root_ms"], "stats_apply_ms": cpu["t_sa_ms"],
                        "root_step_ms_pages_design": round(cpu["pages_root_ms"], 1),
                        "pages_design": ("fp64 coupled Newton on host cores for every statistic "
                                         "(timed on 4, extrapolated by n^3)")}
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32/f64", "data": "synthetic",
            "config": {"workload": args.config, "params": numel(cfg), "block_size": cfg["block_size"],
                       "grad_dtype": cfg["grad_dtype"], "root_interval": interval,
                       "newton_products": (args.roots if args.roots == "fp64"
                                           else f"int8-emulated fp64, {args.slices} slices"),
                       "one_sided_right": [list(shapes[i]) for i in one_sided],
                       "gemm_tiles": args.gemm_tiles,
                       "root_steps_timed": n_root,
                       "amortisation": "ms_per_step = t_stats + t_apply + t_roots / root_interval",
                       "credited_newton_steps_per_statistic": NEWTON_STEPS_CREDIT.get(args.config, 5),
                       "l2": "flushed between steps (256 MiB write)",
                       "parallelism": "single GPU" if world == 1 else f"replicas x{world}"},
            "t_stats_ms": t_stats, "t_apply_ms": t_apply, "t_roots_ms": t_roots,
            "timed_region_ms": region_ms,
            "executed_tflops": executed / (ms * 1e-3) / 1e12,
            "newton_steps_per_statistic": round(sum(iters_sum) / max(len(iters_sum), 1) / max(n_root, 1), 3),
            "roofline": roof, "kernel_roofs": every, "cpu_baseline": cpu_line, "e2e": e2e,
            "async_roots": async_line, "gpu_launches": launches,
            "clocks": clk, "kernels": phase, "fp64_gemm_peak_tflops": round(fp64_peak, 2),
            "peaks_source": peak_src,
            "flops_per_step": {"stats": stats_flops(cfg), "apply": apply_flops(cfg),
                               "roots_per_root_step_executed": newton_exec,
                               "credited_per_amortised_step": F},
        }
        print(json.dumps(line), flush=True)
    opt.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
