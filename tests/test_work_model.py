"""The algorithmic-work model that bench.py divides by the measured times.

Each count is checked against a closed form worked out by hand from the
workload's shapes (block grid, SYRK triangles, chained GEMMs, symmetric
Newton products), so that a wrong factor in the reported TFLOP/s or roofline
fraction fails here, on the CPU.
"""
import bench
from shampoo_second_order_b200 import workloads as wl


def test_transformer_layer_block_grid_and_counts():
    c = wl.CONFIGS["transformer_layer_b512"]
    blks, segs = bench.blocks_of(c)
    # 4 x 1024^2 (4 blocks each) + 1024 x 4096 and 4096 x 1024 (16 each)
    assert len(blks) == 48 and all(b == (512, 512) for b in blks)
    assert segs == [512, 512, 512, 512]   # two 1024-long vectors
    assert bench.numel(c) == 4 * 1024 * 1024 + 2 * 1024 * 4096 + 2 * 1024
    # statistics: L and R triangles m(m+1)n per block, l(l+1) per segment
    tri = 512 * 513 * 512
    assert bench.stats_flops(c) == 48 * 2 * tri + 4 * 512 * 513
    # apply: G R (2 m n^2) then L Y (2 m^2 n) per block; a matvec per segment
    assert bench.apply_flops(c) == 48 * 4 * 512 ** 3 + 4 * 2 * 512 ** 2
    # 96 factors at p = 4 and 4 segments at p/2 = 2, all 512 wide
    sizes = bench.matrix_sizes(c)
    assert sizes.count((512, 4)) == 96 and sizes.count((512, 3)) == 4


def test_newton_products_per_step():
    """p = 4: X T, T T, T^2 T^2, T^4 M per step; p/2 = 2: X T, T T, T^2 M.
    The first step's X0 T0 is a scaled copy (X0 = c^{-1} I)."""
    c = wl.CONFIGS["transformer_layer_b512"]
    n = len(bench.matrix_sizes(c))
    f = 512 * 512 * 513   # the upper triangle of one 512 x 512 product
    k = 7
    a, b, cc = bench.newton_flops(c, [k] * n, per_kernel=True)
    assert a == n * (2 * k - 1) * f
    assert b == 96 * k * f   # only the p = 4 factors form T^4
    assert cc == n * k * f
    assert bench.newton_flops(c, [k] * n) == a + b + cc
    # a matrix that gave up after k steps is reported as -1-k and counted the same
    assert bench.newton_flops(c, [-1 - k] * n) == a + b + cc
    assert bench.newton_flops(c, [0] * n) == 0


def test_other_configurations_match_their_shapes():
    big = wl.CONFIGS["transformer_big_b1024"]
    blks, segs = bench.blocks_of(big)
    # 12 x (4 x 1 + 8 + 8) blocks of 1024^2 plus the 32 x 1 embedding blocks
    assert len(blks) == 12 * 20 + 32 and not segs
    assert bench.numel(big) == 12 * (4 * 1024 ** 2 + 2 * 1024 * 8192) + 32768 * 1024
    assert bench.stats_flops(big) == len(blks) * 2 * 1024 * 1025 * 1024
    assert bench.apply_flops(big) == len(blks) * 4 * 1024 ** 3

    rn = wl.CONFIGS["resnet50_b128"]
    blks, segs = bench.blocks_of(rn)
    assert (len(blks), len(segs)) == (1576, 430)
    assert all(1 <= m <= 128 and 1 <= n <= 128 for m, n in blks)

    one = wl.CONFIGS["single_64x32"]
    assert bench.blocks_of(one) == ([(64, 32)], [])
    assert bench.stats_flops(one) == 64 * 65 * 32 + 32 * 33 * 64
    assert bench.apply_flops(one) == 2 * 64 * 32 * (64 + 32)


def test_one_sided_blocks_drop_a_factor():
    """A block kept on the right only accumulates and applies R alone."""
    c = dict(wl.CONFIGS["single_64x32"], right_only=[0])
    assert bench.block_sides(c) == [2]
    assert bench.stats_flops(c) == 32 * 33 * 64
    assert bench.apply_flops(c) == 2 * 64 * 32 * 32
    assert bench.matrix_sizes(c) == [(64, 3), (32, 3)]


def test_job_throughput_is_total_work_over_the_slowest_rank():
    # 1e12 flops per rank on 4 ranks in 2 ms: 2000 TFLOP/s for the job
    assert abs(bench.job_tflops(1e12, 4, 2.0) - 2000.0) < 1e-9


def test_committed_dram_traffic_is_reported_only_for_its_workload(monkeypatch):
    """The ncu traffic per launch was captured on one workload; the roofline
    block carries it there and null everywhere else."""
    monkeypatch.setitem(bench.TRAFFIC_PER_LAUNCH, ("transformer_layer_b512", "newton_step_a"), 123)
    peaks = {"hbm_gbs": 6500.0, "bf16_tflops": 1600.0}
    for name, key, expect in [("transformer_layer_b512", "transformer_layer_b512", True),
                              ("transformer_big_b1024", "transformer_big_b1024", False),
                              ("transformer_layer_b512", None, False)]:
        c = wl.CONFIGS[name]
        n = len(bench.matrix_sizes(c))
        prof = {"newton_step_a": (9, 50.0), "stats_tc": (20, 1.0)}
        top, roof, every = bench.roofline(c, prof, [7] * n, 20, 1, peaks, 35.0, 6, key)
        assert top == "newton_step_a" and roof["bound"] == "tensor"
        assert (roof["traffic"] is not None) == expect
        assert set(every) == {"newton_step_a", "stats_tc"}
        # achieved = the launches' credited products over their event time
        a = bench.newton_flops(c, [7] * n, per_kernel=True)[0]
        assert abs(roof["achieved"] - a / 50e-3 / 1e12) < 1e-3 * roof["achieved"]


def test_the_dominant_kernel_is_taken_on_the_amortised_step():
    """Root kernels count once per root interval: 5 ms of Newton in one root
    step of a 100-step interval weighs 0.05 ms per step, less than a 0.5 ms
    statistics GEMM that runs every step."""
    c = wl.CONFIGS["transformer_big_b1024"]
    n = len(bench.matrix_sizes(c))
    prof = {"newton_step_a": (9, 5.0), "stats_tc": (20, 10.0)}
    am = bench.amortised_ms(prof, 20, 1, c["root_interval"])
    assert abs(am["newton_step_a"] - 0.05) < 1e-12 and abs(am["stats_tc"] - 0.5) < 1e-12
    top, roof, _ = bench.roofline(c, prof, [5] * n, 20, 1, {"hbm_gbs": 6500.0, "bf16_tflops": 1600.0}, 35.0)
    assert top == "stats_tc"


def test_both_arms_credit_the_same_step_work():
    """The credited work of an amortised step: statistics + apply + the
    credited Newton steps of every iterated statistic over the interval (a
    dropped one-sided factor is not iterated)."""
    c = wl.CONFIGS["transformer_big_b1024"]
    k = bench.NEWTON_STEPS_CREDIT["transformer_big_b1024"]
    f = 1024 * 1024 * 1025
    # 544 statistics of side 1024, p = 4: per step X T (less the first), T T, T2 T2, T4 M
    roots = 544 * (4 * k - 1) * f
    assert bench.credited_step_flops(c, "transformer_big_b1024") == (
        bench.stats_flops(c) + bench.apply_flops(c) + roots / 100)
    one = dict(wl.CONFIGS["single_64x32"], right_only=[0])
    assert bench.credit_iters(one, 6) == [0, 6]


def test_end_to_end_buffers_are_the_parameters_back_to_back():
    """The end-to-end loop uploads each step's gradients as one flat buffer and
    hands the optimizer per-parameter views of it: the views must be
    contiguous, shaped like the parameters, cover the buffer exactly in order,
    and the bytes per step must be the parameters' bytes."""
    import numpy as np
    import torch
    shapes = [s if len(s) == 2 else (s[0],) for s in wl.CONFIGS["resnet50_b128"]["shapes"][:12]]
    total = sum(int(np.prod(s)) for s in shapes)
    flat = torch.arange(total, dtype=torch.float32)
    vs = bench.flat_views(flat, shapes)
    assert [tuple(v.shape) for v in vs] == [tuple(s) for s in shapes]
    assert all(v.is_contiguous() for v in vs)
    o = 0
    for v in vs:   # element k of view i is element offs[i] + k of the buffer
        assert float(v.reshape(-1)[0]) == o and float(v.reshape(-1)[-1]) == o + v.numel() - 1
        o += v.numel()
    assert o == total == flat.numel()
    assert flat.numel() * 4 == sum(int(np.prod(s)) * 4 for s in shapes)
    import pytest
    with pytest.raises(ValueError):
        bench.flat_views(torch.zeros(total + 1), shapes)
