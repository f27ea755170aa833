"""Parity of the CUDA path with the fp64 oracle, through the C-ABI.

Tolerances (relative Frobenius error per object):
  statistics L, R, S              <= 1e-5
  roots, condition number <= 1e6  <= 1e-3
  per block: W_new and the step dW = W_new - W_old   <= 1e-3
The condition number is that of the oracle's statistic plus eps I.  Beyond
1e6 the root is not compared: a float32 statistic only resolves eigenvalues
down to about 2^-24 of its largest, so the root's near-null part is set by
rounding there; the parameters, which those directions do not reach, are
still compared.
Both sides take the same seeded inputs from the workloads module; the oracle
never sees a value the CUDA path produced except where a test compares.
"""
import numpy as np
import pytest

from oracle import ShampooOracle, block_partition, inverse_root, vector_segments
from shampoo_second_order_b200 import workloads as wl

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

STATS_TOL = 1e-5
ROOT_TOL = 1e-3
STEP_TOL = 1e-3


@pytest.fixture(scope="module", autouse=True)
def cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from shampoo_second_order_b200 import _lib
    _lib.lib()   # fails loudly if the library is missing
    yield


def rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    nb = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (nb if nb > 0 else 1.0)


def to_dev(x, dtype):
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def pieces(shape, b):
    if len(shape) == 2:
        return [(slice(r0, r0 + m), slice(c0, c0 + n)) for (r0, c0, m, n) in block_partition(*shape, b)]
    return [(slice(s0, s0 + ln),) for (s0, ln) in vector_segments(shape[0], b)]


SIDE_CODE = {"both": 0, "left": 1, "right": 2}


def run_pair(shapes, b, beta2, eps, graft, mu, lr, gdtype, steps, interval, seed, gstd,
             check_every=True, check_state=True, method="fp64", sides=None, tiles="pair"):
    """tiles: "pair" (the default: 256 x 256 CTA-pair tiles where the block
    side is a multiple of 256) or "single" (128 x 128 single-CTA tiles)."""
    from shampoo_second_order_b200 import Shampoo
    o = ShampooOracle(shapes, b, beta2, eps, 4, graft, mu,
                      sides=None if sides is None else [SIDE_CODE[x] for x in sides])
    opt = Shampoo(shapes, b, beta2, eps, 4, graft, mu, gdtype)
    opt.set_root_method(method)
    opt.set_gemm_tiles(tiles == "pair")
    for i, sd in enumerate(sides or []):
        if sd != "both":
            opt.set_one_sided(i, sd)
    W0 = wl.make_params(shapes, seed)
    Wo = [w.astype(np.float64) for w in W0]
    Wd = [torch.from_numpy(w).cuda() for w in W0]
    worst = {"stats": 0.0, "roots": 0.0, "dW": 0.0, "W": 0.0}
    for t in range(steps):
        g = wl.make_grads(shapes, seed, t, gstd, gdtype)
        gd = [to_dev(x, gdtype) for x in g]
        roots = (t % interval == 0)
        prev_d = [w.cpu().numpy().astype(np.float64) for w in Wd]
        prev_o = Wo
        Wo = o.step(Wo, g, lr, roots)
        opt.step(Wd, gd, lr, roots)
        torch.cuda.synchronize()
        if not (check_every or t == steps - 1):
            continue
        if check_state and (roots or t == steps - 1):
            mats = o.matrices()
            ro = o.root_matrices()
            for k in range(opt.num_matrices()):
                S, _ = opt.read_matrix(0, k)
                worst["stats"] = max(worst["stats"], rel(S, mats[k][0]))
                assert opt.matrix_info(k)[1] == mats[k][1]
                ev = np.linalg.eigvalsh(mats[k][0]) + eps
                if ev.max() / max(ev.min(), 1e-300) > 1e6:
                    continue
                X, _ = opt.read_matrix(1, k)
                worst["roots"] = max(worst["roots"], rel(X, ro[k]))
        for i, s in enumerate(shapes):
            wd = Wd[i].cpu().numpy().astype(np.float64)
            d_gpu, d_ref = wd - prev_d[i], Wo[i] - prev_o[i]   # the step, once per parameter
            for sl in pieces(s, b):
                worst["dW"] = max(worst["dW"], rel(d_gpu[sl], d_ref[sl]))
                worst["W"] = max(worst["W"], rel(wd[sl], Wo[i][sl]))
    opt.close()
    return worst


def assert_worst(w):
    assert w["stats"] <= STATS_TOL, w
    assert w["roots"] <= ROOT_TOL, w
    assert w["dW"] <= STEP_TOL, w
    assert w["W"] <= STEP_TOL, w


# --------------------------------------------------------------------------
# whole steps on small cases (several tiles, ragged tails, both grad dtypes)
# --------------------------------------------------------------------------
def test_single_64x32_ten_steps():
    c = wl.CONFIGS["single_64x32"]
    w = run_pair(c["shapes"], c["block_size"], c["beta2"], c["eps"], c["graft"], c["momentum"],
                 c["lr"], c["grad_dtype"], c["steps"], c["root_interval"], c["seed"], c["grad_std"])
    assert_worst(w)


@pytest.mark.parametrize("gdtype", ["f32", "bf16"])
@pytest.mark.parametrize("graft,mu", [(1, 0.0), (0, 0.0), (1, 0.9)])
def test_ragged_mixed_set(gdtype, graft, mu):
    shapes = [(200, 130), (64, 64), (19, 200), (130,), (64,), (1, 77)]
    w = run_pair(shapes, 64, 0.99, 1e-6, graft, mu, 0.1, gdtype, steps=6, interval=3, seed=7,
                 gstd=1e-2)
    assert_worst(w)


def test_block_128_many_tiles():
    shapes = [(300, 257), (128, 384), (500,)]
    w = run_pair(shapes, 128, 0.999, 1e-6, 1, 0.0, 0.1, "f32", steps=4, interval=2, seed=8, gstd=1e-3)
    assert_worst(w)


@pytest.mark.parametrize("tiles", ["pair", "single"])
@pytest.mark.parametrize("gdtype", ["f32", "bf16"])
def test_block_1024_ragged_maximum_size(gdtype, tiles):
    """The largest block side (b = 1024) with ragged last blocks in both
    directions (1100 = 1024 + 76, 1030 = 1024 + 6) and a 1-D parameter longer
    than one segment, on both GEMM tilings."""
    shapes = [(1100, 1030), (1030,)]
    w = run_pair(shapes, 1024, 0.999, 1e-6, 1, 0.0, 0.1, gdtype, steps=3, interval=2, seed=15,
                 gstd=1e-3, check_every=False, tiles=tiles)
    assert_worst(w)


@pytest.mark.parametrize("tiles", ["pair", "single"])
@pytest.mark.parametrize("gdtype,b", [("f32", 512), ("bf16", 512), ("f32", 256)])
def test_pair_tiles_ragged_sets(gdtype, b, tiles):
    """Block sides that are multiples of 256 run the GEMMs on CTA pairs
    (256 x 256 tiles; fp32 statistics too): ragged blocks whose valid part
    ends inside the first or the second 128 rows of a pair tile, a weight
    narrower than one tile, graft and momentum, against the oracle on both
    tilings."""
    shapes = [(600, 700), (130, 1100), (1300, 40), (300,)]
    w = run_pair(shapes, b, 0.99, 1e-6, 1, 0.9, 0.1, gdtype, steps=4, interval=3, seed=16,
                 gstd=1e-2, tiles=tiles)
    assert_worst(w)


def test_transformer_layer_b512_full_size():
    """The Transformer-layer set at full size in the bench's launch
    configuration: 21 steps, roots at steps 1 and 21."""
    c = wl.CONFIGS["transformer_layer_b512"]
    w = run_pair(c["shapes"], c["block_size"], c["beta2"], c["eps"], c["graft"], c["momentum"],
                 c["lr"], c["grad_dtype"], 21, c["root_interval"], c["seed"], c["grad_std"],
                 check_every=False)
    assert_worst(w)


# --------------------------------------------------------------------------
# the batched inverse-root kernel on its own
# --------------------------------------------------------------------------
@pytest.mark.parametrize("n", [64, 100, 192, 512, 1000, 1024])
@pytest.mark.parametrize("p", [2, 4])
def test_batched_root_vs_oracle(n, p):
    from shampoo_second_order_b200 import batched_inverse_root
    A, _ = wl.spd_batch(6, n, seed=n + p, log10_kappa=(2.0, 6.0))
    A32 = A.astype(np.float32)
    X, iters = batched_inverse_root(torch.from_numpy(A32).cuda(), p, 1e-6)
    X = X.cpu().numpy()
    iters = iters.cpu().numpy()
    assert (iters > 0).all(), iters
    for i in range(6):
        ref = inverse_root(A32[i].astype(np.float64), 1e-6, p)
        assert rel(X[i], ref) <= ROOT_TOL, (i, rel(X[i], ref))


def test_batched_root_kappa_sweep_full_size():
    """256 SPD 512 x 512 matrices with condition numbers 1e2..1e8: every
    matrix with kappa <= 1e6 (171 of them) within 1e-3 of the oracle's root,
    for p = 4 and p = 2; the rest finite."""
    from shampoo_second_order_b200 import batched_inverse_root
    c = wl.ROOTS_CONFIG
    A, lam = wl.spd_batch(c["batch"], c["n"], c["seed"], c["log10_kappa"])
    A32 = A.astype(np.float32)
    dA = torch.from_numpy(A32).cuda()
    for p in c["ps"]:
        X, iters = batched_inverse_root(dA, p, c["eps"], c["tol"])
        X = X.cpu().numpy()
        iters = iters.cpu().numpy()
        kappa = lam.max(1) / lam.min(1)
        compared = 0
        for i in range(c["batch"]):
            if kappa[i] > 1e6:
                assert np.isfinite(X[i]).all(), (p, i)
                continue
            ref = inverse_root(A32[i].astype(np.float64), c["eps"], p)
            assert iters[i] > 0
            assert rel(X[i], ref) <= ROOT_TOL, (p, i, kappa[i], rel(X[i], ref))
            compared += 1
        assert compared == int((kappa <= 1e6).sum()) >= 170


@pytest.mark.parametrize("n", [64, 100, 192, 512])
@pytest.mark.parametrize("p", [2, 4])
def test_batched_root_int8_emulated_vs_oracle(n, p):
    """Newton with its products emulated on the int8 tensor cores (6 slices)
    reaches the oracle's root like the float64 products do, in the same
    number of steps give or take one."""
    from shampoo_second_order_b200 import batched_inverse_root
    A, _ = wl.spd_batch(6, n, seed=n + p, log10_kappa=(2.0, 6.0))
    dA = torch.from_numpy(A.astype(np.float32)).cuda()
    X, iters = batched_inverse_root(dA, p, 1e-6, method="int8")
    _, iters64 = batched_inverse_root(dA, p, 1e-6)
    X = X.cpu().numpy()
    iters, iters64 = iters.cpu().numpy(), iters64.cpu().numpy()
    assert (iters > 0).all() and (np.abs(iters - iters64) <= 1).all(), (iters, iters64)
    for i in range(6):
        ref = inverse_root(A[i].astype(np.float32).astype(np.float64), 1e-6, p)
        assert rel(X[i], ref) <= ROOT_TOL, (i, rel(X[i], ref))


def test_batched_root_int8_emulated_kappa_sweep():
    """The 256 x 512 kappa sweep (1e2..1e8) through the emulated products,
    sampled; every matrix with kappa <= 1e6 within 1e-3 of the oracle."""
    from shampoo_second_order_b200 import batched_inverse_root
    c = wl.ROOTS_CONFIG
    A, lam = wl.spd_batch(c["batch"], c["n"], c["seed"], c["log10_kappa"])
    A32 = A.astype(np.float32)
    dA = torch.from_numpy(A32).cuda()
    kappa = lam.max(1) / lam.min(1)
    for p in c["ps"]:
        X, iters = batched_inverse_root(dA, p, c["eps"], c["tol"], method="int8")
        X = X.cpu().numpy()
        iters = iters.cpu().numpy()
        for i in list(range(0, c["batch"], 16)) + [c["batch"] - 1]:
            if kappa[i] <= 1e6:
                ref = inverse_root(A32[i].astype(np.float64), c["eps"], p)
                assert iters[i] > 0
                assert rel(X[i], ref) <= ROOT_TOL, (p, i, kappa[i], rel(X[i], ref))


def test_batched_root_int8_nan_input_fails_that_matrix_only():
    from shampoo_second_order_b200 import batched_inverse_root
    A = np.stack([np.eye(128, dtype=np.float32) * 2, np.eye(128, dtype=np.float32)])
    A[1, 3, 3] = np.nan
    X, iters = batched_inverse_root(torch.from_numpy(A).cuda(), 4, 1e-6, method="int8")
    iters = iters.cpu().numpy()
    assert iters[0] >= 0 and iters[1] < 0
    assert np.allclose(X[0].cpu().numpy(), (2 + 1e-6) ** -0.25 * np.eye(128), rtol=1e-6)


@pytest.mark.parametrize("gdtype", ["f32", "bf16"])
def test_ragged_mixed_set_int8_emulated_roots(gdtype):
    shapes = [(200, 130), (64, 64), (19, 200), (130,), (64,), (1, 77)]
    w = run_pair(shapes, 64, 0.99, 1e-6, 1, 0.9, 0.1, gdtype, steps=6, interval=3, seed=7,
                 gstd=1e-2, method="int8")
    assert_worst(w)


def test_transformer_layer_b512_int8_emulated_roots():
    c = wl.CONFIGS["transformer_layer_b512"]
    w = run_pair(c["shapes"], c["block_size"], c["beta2"], c["eps"], c["graft"], c["momentum"],
                 c["lr"], c["grad_dtype"], 21, c["root_interval"], c["seed"], c["grad_std"],
                 check_every=False, method="int8")
    assert_worst(w)


# --------------------------------------------------------------------------
# one-sided blocks (Lemma 1)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("gdtype,method", [("f32", "fp64"), ("bf16", "fp64"), ("f32", "int8")])
def test_one_sided_ragged_set(gdtype, method):
    shapes = [(200, 130), (64, 64), (19, 200), (130,), (300, 64), (1, 77)]
    sides = ["left", "both", "right", "both", "right", "left"]
    w = run_pair(shapes, 64, 0.99, 1e-6, 1, 0.9, 0.1, gdtype, steps=6, interval=3, seed=9,
                 gstd=1e-2, method=method, sides=sides)
    assert_worst(w)


def test_one_sided_embedding_block_512():
    """A tall embedding-like weight kept on its column side only (the
    vocabulary side's statistics are never formed), bf16 gradients, b = 512."""
    shapes = [(4096, 512), (512, 512)]
    w = run_pair(shapes, 512, 0.999, 1e-6, 1, 0.0, 0.1, "bf16", steps=4, interval=2, seed=10,
                 gstd=1e-3, check_every=False, sides=["right", "both"])
    assert_worst(w)


def test_one_sided_state_and_argument_errors():
    from shampoo_second_order_b200 import Shampoo, _lib
    opt = Shampoo([(64, 64), (32,)], 64, 0.9, 1e-6)
    with pytest.raises(_lib.ShampooError) as e:
        opt.set_one_sided(1, "left")                 # 1-D parameter
    assert e.value.status == _lib.EINVAL
    opt.set_one_sided(0, "left")
    assert [opt.matrix_info(k)[1] for k in range(3)] == [2, 0, 2]
    opt.set_one_sided(0, "both")
    assert [opt.matrix_info(k)[1] for k in range(3)] == [4, 4, 2]
    opt.update_stats([torch.randn(64, 64, device="cuda"), torch.randn(32, device="cuda")])
    with pytest.raises(_lib.ShampooError) as e:
        opt.set_one_sided(0, "right")                # after the first statistics
    assert e.value.status == _lib.ESTATE
    opt.close()


# --------------------------------------------------------------------------
# edge cases and error conventions
# --------------------------------------------------------------------------
def test_zero_gradient_leaves_weight():
    from shampoo_second_order_b200 import Shampoo
    shapes = [(70, 70), (33,)]
    opt = Shampoo(shapes, 64, 0.9, 1e-6)
    W = [torch.randn(s, device="cuda") for s in shapes]
    W0 = [w.clone() for w in W]
    g = [torch.zeros(s, device="cuda") for s in shapes]
    opt.step(W, g, 0.1, True)
    torch.cuda.synchronize()
    for a, b in zip(W, W0):
        assert torch.equal(a, b)
    opt.close()


def test_nonfinite_gradient_skips_parameter():
    from shampoo_second_order_b200 import Shampoo
    shapes = [(64, 40), (50, 64)]
    opt = Shampoo(shapes, 64, 0.9, 1e-6)
    W = [torch.randn(s, device="cuda") for s in shapes]
    g = [torch.randn(s, device="cuda") for s in shapes]
    opt.step(W, g, 0.1, True)
    W1 = [w.clone() for w in W]
    L_before, _ = opt.read_matrix(0, 0)
    g2 = [torch.randn(s, device="cuda") for s in shapes]
    g2[0][3, 5] = float("nan")
    opt.step(W, g2, 0.1, False)
    torch.cuda.synchronize()
    assert opt.nonfinite_status() == 1
    assert torch.equal(W[0], W1[0])
    assert not torch.equal(W[1], W1[1])
    L_after, _ = opt.read_matrix(0, 0)
    assert np.array_equal(L_before, L_after)
    opt.close()


def test_apply_before_roots_is_state_error():
    from shampoo_second_order_b200 import Shampoo, _lib
    opt = Shampoo([(64, 64)], 64, 1.0, 1e-6)
    W = [torch.zeros(64, 64, device="cuda")]
    g = [torch.randn(64, 64, device="cuda")]
    opt.update_stats(g)
    with pytest.raises(_lib.ShampooError) as e:
        opt.apply(W, g, 0.1)
    assert e.value.status == _lib.ESTATE
    opt.close()


def test_iteration_cap_reports_not_converged_and_falls_back():
    from shampoo_second_order_b200 import Shampoo
    opt = Shampoo([(64, 64)], 64, 1.0, 1e-6)    # square gradient: L and R full rank
    opt.set_root_options(1e-6, 2)
    g = [torch.randn(64, 64, device="cuda")]
    opt.update_stats(g)
    assert opt.compute_roots() is False
    nf, it = opt.root_status()
    assert nf == 2 and it == 2
    # never had a root: c^{-1} I with c^p = min(||A+eps I||_F, ||A+eps I||_inf)
    L, _ = opt.read_matrix(0, 0)
    A = (g[0].double() @ g[0].double().T).cpu().numpy() + 1e-6 * np.eye(64)
    cp = min(np.linalg.norm(A), np.abs(A).sum(1).max())
    X, _ = opt.read_matrix(1, 0)
    assert np.allclose(X, cp ** -0.25 * np.eye(64), rtol=1e-5)
    # with the cap lifted they converge and replace the fallback
    opt.set_root_options(1e-6, 100)
    assert opt.compute_roots() is True
    X2, _ = opt.read_matrix(1, 0)
    assert rel(X2, inverse_root(opt.read_matrix(0, 0)[0].astype(np.float64), 1e-6, 4)) < ROOT_TOL
    opt.close()


def test_nan_statistic_fails_root_and_keeps_previous():
    from shampoo_second_order_b200 import batched_inverse_root
    A = np.stack([np.eye(64, dtype=np.float32) * 2, np.eye(64, dtype=np.float32)])
    A[1, 3, 3] = np.nan
    X, iters = batched_inverse_root(torch.from_numpy(A).cuda(), 4, 1e-6)
    iters = iters.cpu().numpy()
    assert iters[0] >= 0 and iters[1] < 0
    assert np.allclose(X[0].cpu().numpy(), (2 + 1e-6) ** -0.25 * np.eye(64), rtol=1e-6)


def test_scaled_newton_takes_fewer_steps_than_plain():
    """The Lanczos-scaled iteration reaches the same root (checked above) in
    fewer steps than the plain coupled Newton iteration needs on the same
    matrices (the oracle's CPU copy of the pages' root route)."""
    from oracle import coupled_newton_inverse_root
    from shampoo_second_order_b200 import batched_inverse_root
    A, _ = wl.spd_batch(8, 256, seed=31, log10_kappa=(2.0, 6.0))
    A32 = A.astype(np.float32)
    X, iters = batched_inverse_root(torch.from_numpy(A32).cuda(), 4, 1e-6)
    iters = iters.cpu().numpy()
    X = X.cpu().numpy()
    for i in range(8):
        _, k_plain, ok = coupled_newton_inverse_root(A32[i].astype(np.float64), 1e-6, 4)
        assert ok and 0 < iters[i] < k_plain, (i, iters[i], k_plain)
        ref = inverse_root(A32[i].astype(np.float64), 1e-6, 4)
        assert rel(X[i], ref) <= ROOT_TOL


def run_subset(cfg, steps, interval, keep):
    """Run the CUDA path on the whole parameter set of `cfg` and the oracle
    on the parameters listed in `keep` only (parameters never interact: each
    has its own statistics and its own graft scale).  Returns the worst
    per-block relative errors of W and of the last step's dW."""
    from shampoo_second_order_b200 import Shampoo
    shapes = cfg["shapes"]
    sub = [shapes[i] for i in keep]
    o = ShampooOracle(sub, cfg["block_size"], cfg["beta2"], cfg["eps"], cfg["p"], cfg["graft"],
                      cfg["momentum"])
    opt = Shampoo(shapes, cfg["block_size"], cfg["beta2"], cfg["eps"], cfg["p"], cfg["graft"],
                  cfg["momentum"], cfg["grad_dtype"])
    W0 = wl.make_params(shapes, cfg["seed"])
    Wd = [torch.from_numpy(w).cuda() for w in W0]
    Wo = [W0[i].astype(np.float64) for i in keep]
    for t in range(steps):
        g = wl.make_grads(shapes, cfg["seed"], t, cfg["grad_std"], cfg["grad_dtype"])
        roots = t % interval == 0
        prev_d = [Wd[i].cpu().numpy().astype(np.float64) for i in keep]
        prev_o = Wo
        Wo = o.step(Wo, [g[i] for i in keep], cfg["lr"], roots)
        opt.step(Wd, [to_dev(x, cfg["grad_dtype"]) for x in g], cfg["lr"], roots)
        torch.cuda.synchronize()
        del g
    worst = {"dW": 0.0, "W": 0.0}
    for k, i in enumerate(keep):
        wd = Wd[i].cpu().numpy().astype(np.float64)
        d_gpu, d_ref = wd - prev_d[k], Wo[k] - prev_o[k]
        for sl in pieces(shapes[i], cfg["block_size"]):
            worst["dW"] = max(worst["dW"], rel(d_gpu[sl], d_ref[sl]))
            worst["W"] = max(worst["W"], rel(wd[sl], Wo[k][sl]))
    opt.close()
    return worst


def test_transformer_big_full_set_sampled_parameters():
    """The ~285M-parameter Transformer-big set (b = 1024, fp32 gradients,
    momentum 0.9) runs whole on the GPU; layer 0's query, FFN-in and FFN-out
    weights are checked against the oracle over 3 steps (roots at 1 and 3)."""
    c = wl.CONFIGS["transformer_big_b1024"]
    w = run_subset(c, steps=3, interval=2, keep=[0, 4, 5])
    assert w["dW"] <= STEP_TOL and w["W"] <= STEP_TOL, w


def test_resnet50_every_weight_51_steps():
    """The ResNet-50 set at its real structure: every weight (1576 blocks of
    <= 128 with padded ragged ones, 430 vector segments, fp32 gradients,
    beta2 = 0.99) over 51 steps with roots at steps 1 and 51 (every 50), so
    49 steps run on stale roots (podcast transcript, segment 14).  Every
    statistic (3582) and every root with kappa <= 1e6 at both root steps,
    and W and dW of every block and segment at every step."""
    c = wl.CONFIGS["resnet50_b128"]
    w = run_pair(c["shapes"], c["block_size"], c["beta2"], c["eps"], c["graft"], c["momentum"], c["lr"],
                 c["grad_dtype"], 51, c["root_interval"], c["seed"], c["grad_std"])
    assert_worst(w)


def test_transformer_big_layer0_and_embedding_101_steps():
    """The Transformer-big set at its real structure where the oracle can
    follow it: layer 0 (Q, K, V, O 1024^2, FFN 1024 x 8192 and 8192 x 1024)
    plus the 32768 x 1024 embedding -- 52 blocks of 1024^2 (segment 16,
    Lemma 2) -- with fp32 gradients N(0, 1e-3), beta2 = 0.999, grafted
    momentum 0.9, over 101 steps with roots at steps 1 and 101 (every 100:
    99 steps on stale roots, segment 14).  All 104 statistics and every root
    with kappa <= 1e6 at both root steps; W and dW of every block at every
    step.  Parameters never interact, so this subset steps exactly as it
    would inside the whole set."""
    c = wl.CONFIGS["transformer_big_b1024"]
    shapes = c["shapes"][:6] + [c["shapes"][-1]]
    w = run_pair(shapes, c["block_size"], c["beta2"], c["eps"], c["graft"], c["momentum"], c["lr"],
                 c["grad_dtype"], 101, c["root_interval"], c["seed"], c["grad_std"])
    assert_worst(w)


# --------------------------------------------------------------------------
# asynchronous roots (podcast transcript, segment 16): the steps keep using
# the roots in place while the next ones are computed, then swap them in
# --------------------------------------------------------------------------
def run_async_pair(shapes, b, beta2, eps, graft, mu, lr, gdtype, steps, submit, wait_at, seed, gstd,
                   method="fp64"):
    """Roots synchronously at step 0; an asynchronous job queued after the
    statistics of each step in `submit`; a blocking install before the apply
    of each step in `wait_at`.  The library swaps a finished job in at an
    apply of its choosing; the test reads at which one from the roots
    generation and installs, on the oracle, the roots of the statistics as
    they stood at submission before the same step's apply."""
    import copy
    from shampoo_second_order_b200 import Shampoo
    o = ShampooOracle(shapes, b, beta2, eps, 4, graft, mu)
    opt = Shampoo(shapes, b, beta2, eps, 4, graft, mu, gdtype)
    opt.set_root_method(method)
    W0 = wl.make_params(shapes, seed)
    Wo = [w.astype(np.float64) for w in W0]
    Wd = [torch.from_numpy(w).cuda() for w in W0]
    worst = {"dW": 0.0, "W": 0.0}
    pending = None
    installs = []
    for t in range(steps):
        g = wl.make_grads(shapes, seed, t, gstd, gdtype)
        gd = [to_dev(x, gdtype) for x in g]
        prev_d = [w.cpu().numpy().astype(np.float64) for w in Wd]
        prev_o = Wo
        o.update_stats(g)
        opt.update_stats(gd)
        if t == 0:
            o.compute_roots()
            opt.compute_roots()
        if t in submit:
            kept = list(o.roots)          # compute_roots replaces the entries of o.roots
            o.compute_roots()
            pending, o.roots = o.roots, kept
            assert opt.compute_roots_async()
        gen0 = opt.roots_generation()
        if t in wait_at:
            opt.install_roots(wait=True)
        opt.apply(Wd, gd, lr)
        if opt.roots_generation() > gen0:
            assert pending is not None
            o.roots, pending = copy.deepcopy(pending), None
            installs.append(t)
        Wo = o.apply(Wo, g, lr)
        torch.cuda.synchronize()
        for i, s in enumerate(shapes):
            wd = Wd[i].cpu().numpy().astype(np.float64)
            d_gpu, d_ref = wd - prev_d[i], Wo[i] - prev_o[i]   # the step, once per parameter
            for sl in pieces(s, b):
                worst["dW"] = max(worst["dW"], rel(d_gpu[sl], d_ref[sl]))
                worst["W"] = max(worst["W"], rel(wd[sl], Wo[i][sl]))
    assert pending is None
    opt.close()
    return worst, installs


@pytest.mark.parametrize("gdtype,method", [("f32", "fp64"), ("bf16", "fp64"), ("f32", "int8")])
def test_async_roots_ragged_set(gdtype, method):
    shapes = [(200, 130), (64, 64), (19, 200), (130,), (64,), (1, 77)]
    w, installs = run_async_pair(shapes, 64, 0.99, 1e-6, 1, 0.0, 0.1, gdtype, steps=9,
                                 submit=(2, 5), wait_at=(4, 8), seed=7, gstd=1e-2, method=method)
    assert w["dW"] <= STEP_TOL and w["W"] <= STEP_TOL, w
    assert len(installs) == 2 and 2 <= installs[0] <= 4 and 5 <= installs[1] <= 8, installs


def test_async_roots_transformer_layer_b512():
    """The bench's set and launch configuration: roots at step 0, an
    asynchronous job after step 20's statistics, installed by step 24."""
    c = wl.CONFIGS["transformer_layer_b512"]
    w, installs = run_async_pair(c["shapes"], c["block_size"], c["beta2"], c["eps"], c["graft"],
                                 c["momentum"], c["lr"], c["grad_dtype"], steps=25, submit=(20,),
                                 wait_at=(24,), seed=c["seed"], gstd=c["grad_std"])
    assert w["dW"] <= STEP_TOL and w["W"] <= STEP_TOL, w
    assert len(installs) == 1 and 20 <= installs[0] <= 24, installs


def test_async_roots_busy_and_sync_refused():
    """While a job runs, a second submission and a synchronous computation
    are refused with EBUSY and leave the roots in use untouched; after the
    install the new roots equal the synchronous ones of the same statistics."""
    from shampoo_second_order_b200 import Shampoo, _lib
    c = wl.CONFIGS["transformer_layer_b512"]
    shapes = c["shapes"]
    opt = Shampoo(shapes, c["block_size"], c["beta2"], c["eps"], 4, 1, 0.0, "bf16")
    g = [to_dev(x, "bf16") for x in wl.make_grads(shapes, 3, 0, 1e-3, "bf16")]
    opt.update_stats(g)
    opt.compute_roots()
    X_sync0, _ = opt.read_matrix(1, 0)
    g = [to_dev(x, "bf16") for x in wl.make_grads(shapes, 3, 1, 1e-3, "bf16")]
    opt.update_stats(g)
    gen = opt.roots_generation()
    assert opt.compute_roots_async()
    busy = not opt.compute_roots_async()          # about ten milliseconds of Newton work queued
    if busy:
        with pytest.raises(_lib.ShampooError) as e:
            opt.compute_roots()
        assert e.value.status == _lib.EBUSY
    X_now, _ = opt.read_matrix(1, 0)
    if opt.roots_generation() == gen:
        assert np.array_equal(X_now, X_sync0)
    assert opt.install_roots(wait=True) or opt.roots_generation() == gen + 1
    X_async, _ = opt.read_matrix(1, 0)
    opt.compute_roots()                           # the same statistics, synchronously
    X_sync1, _ = opt.read_matrix(1, 0)
    assert rel(X_async, X_sync1) <= 1e-6
    assert busy
    opt.close()


# --------------------------------------------------------------------------
# block-sharded data parallelism through the CUDA library (one process: the
# owner plan gives every parameter to rank 0; the packing of gradients and
# weights around the library context is what runs)
# --------------------------------------------------------------------------
def test_sharded_single_rank_matches_oracle():
    from shampoo_second_order_b200.sharded import ShardedShampoo
    shapes = [(200, 130), (64, 64), (19, 200), (130,), (1, 77)]
    b, beta2, eps, lr, gstd = 64, 0.99, 1e-6, 0.1, 1e-2
    opt = ShardedShampoo(shapes, b, beta2, eps, 4, 1, 0.5, "f32", root_interval=3)
    o = ShampooOracle(shapes, b, beta2, eps, 4, 1, 0.5)
    W0 = wl.make_params(shapes, 12)
    Wd = [torch.from_numpy(w).cuda() for w in W0]
    Wo = [w.astype(np.float64) for w in W0]
    worst = 0.0
    for t in range(6):
        g = wl.make_grads(shapes, 12, t, gstd, "f32")
        prev_d = [w.cpu().numpy().astype(np.float64) for w in Wd]
        prev_o = Wo
        opt.step(Wd, [to_dev(x, "f32") for x in g], lr, t % 3 == 0)
        Wo = o.step(Wo, g, lr, t % 3 == 0)
        torch.cuda.synchronize()
        for i, s in enumerate(shapes):
            wd = Wd[i].cpu().numpy().astype(np.float64)
            for sl in pieces(s, b):
                worst = max(worst, rel((wd - prev_d[i])[sl], (Wo[i] - prev_o[i])[sl]))
    assert opt.mine == list(range(len(shapes)))
    assert worst <= STEP_TOL, worst
    opt.close()


def test_stalled_pipeline_wait_is_reported_and_the_context_survives():
    """A bounded wait that nothing satisfies ends in about a second with the
    pipeline-timeout status (no hang), and the device keeps working."""
    import time
    from shampoo_second_order_b200 import _lib, batched_inverse_root
    t0 = time.time()
    st = _lib.lib().shampoo_selftest_stalled_wait(None)
    assert st == _lib.ECUDA
    assert "timed out" in _lib.lib().shampoo_last_error(None).decode()
    assert time.time() - t0 < 30
    A = torch.eye(64, device="cuda").mul_(4.0).unsqueeze(0).contiguous()
    X, iters = batched_inverse_root(A, 2, 1e-6)
    assert int(iters[0]) >= 0
    assert torch.allclose(X[0], torch.eye(64, device="cuda") * (4.0 + 1e-6) ** -0.5)


@pytest.mark.parametrize("gdtype,b", [("f32", 128), ("bf16", 128), ("f32", 256)])
def test_statistics_gemm_timeout_is_reported_by_the_step_calls(gdtype, b):
    """The statistics GEMM of one update_stats is made to stall (its MMA
    issuer waits once on a barrier phase nothing completes): the launch runs
    out its bounded wait, aborts and sets the error word.  compute_roots, the
    next synchronising call, returns SHAMPOO_ECUDA, and so do the later calls
    on that context; a fresh context on the same device then matches the
    oracle (the abort faulted nothing).  bf16 gradients also exercise the
    statistics tile staged through shared memory by TMA."""
    import time
    from shampoo_second_order_b200 import Shampoo, _lib
    shapes = [(300, 200), (64,)]
    opt = Shampoo(shapes, b, 0.99, 1e-6, 4, 1, 0.0, gdtype)
    g = [to_dev(x, gdtype) for x in wl.make_grads(shapes, 31, 0, 1e-2, gdtype)]
    W = [torch.from_numpy(w).cuda() for w in wl.make_params(shapes, 31)]
    opt.update_stats(g)
    opt.compute_roots()
    opt.apply(W, g, 0.1)
    _lib.shampoo_selftest_stall_next_stats(opt.ctx)
    t0 = time.time()
    opt.update_stats(g)                      # asynchronous: returns before the kernel ends
    with pytest.raises(_lib.ShampooError) as e:
        opt.compute_roots()
    assert e.value.status == _lib.ECUDA and "timed out" in str(e.value)
    assert time.time() - t0 < 60
    with pytest.raises(_lib.ShampooError) as e:
        opt.root_status()
    assert e.value.status == _lib.ECUDA
    for call in (lambda: opt.update_stats(g), lambda: opt.apply(W, g, 0.1)):
        with pytest.raises(_lib.ShampooError) as e:
            call()
        assert e.value.status == _lib.ECUDA
    opt.close()
    w = run_pair(shapes, b, 0.99, 1e-6, 1, 0.0, 0.1, gdtype, steps=3, interval=2, seed=31, gstd=1e-2)
    assert_worst(w)


@pytest.mark.parametrize("b", [128, 256])
def test_apply_gemm_timeout_is_reported_by_the_step_calls(b):
    """The same failure path in the apply GEMM Y = G R^{-1/p}: at b = 256 on
    CTA pairs, whose two CTAs abort together (the even CTA's MMA issuer gives
    up, the odd CTA sees the abort flag), at b = 128 on single CTAs.  The
    next synchronising call returns SHAMPOO_ECUDA, later step calls refuse,
    and a fresh context then matches the oracle."""
    from shampoo_second_order_b200 import Shampoo, _lib
    shapes = [(300, 260), (64,)]
    opt = Shampoo(shapes, b, 0.99, 1e-6, 4, 1, 0.0, "f32")
    g = [to_dev(x, "f32") for x in wl.make_grads(shapes, 32, 0, 1e-3, "f32")]
    W = [torch.from_numpy(w).cuda() for w in wl.make_params(shapes, 32)]
    opt.update_stats(g)
    opt.compute_roots()
    _lib.shampoo_selftest_stall_next_apply(opt.ctx)
    opt.apply(W, g, 0.1)                     # asynchronous: returns before the kernel ends
    with pytest.raises(_lib.ShampooError) as e:
        opt.root_status()
    assert e.value.status == _lib.ECUDA and "timed out" in str(e.value)
    for call in (lambda: opt.update_stats(g), lambda: opt.apply(W, g, 0.1), lambda: opt.compute_roots()):
        with pytest.raises(_lib.ShampooError) as e:
            call()
        assert e.value.status == _lib.ECUDA
    opt.close()
    w = run_pair(shapes, b, 0.99, 1e-6, 1, 0.0, 0.1, "f32", steps=3, interval=2, seed=32, gstd=1e-3)
    assert_worst(w)
