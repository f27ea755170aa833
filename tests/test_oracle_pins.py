"""Pins of the fp64 oracle to facts other than its own code.

Each test checks the oracle against a closed form, an invariant, a brute
force recomputation or a second, independent route, chosen so that a dropped
term, a wrong sign or exponent, a swapped L/R or a transposed operand fails
at least one of them.  The pages print no worked example for the optimizer
step, so whole-step parity against the pages is unpinned; every function the
step is built from is pinned here.
"""
import json
import os

import numpy as np
import pytest

from oracle import (GRAFT_ADAGRAD, GRAFT_NONE, SIDE_LEFT, SIDE_RIGHT, ShampooOracle,
                    block_partition, coupled_newton_inverse_root, inverse_root, vector_segments)
from shampoo_second_order_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_spd(n, kappa, seed):
    rng = np.random.default_rng(seed)
    Q, _ = np.linalg.qr(rng.standard_normal((n, n)))
    lam = np.logspace(0, np.log10(kappa), n)
    return (Q * lam) @ Q.T, lam


# --------------------------------------------------------------------------
# Inverse roots
# --------------------------------------------------------------------------
@pytest.mark.parametrize("p", [2, 4, 8])
def test_root_of_diagonal_is_elementwise(p):
    d = np.array([3.0, 1e-3, 7.5, 1e4, 0.0])
    eps = 1e-6
    X = inverse_root(np.diag(d), eps, p)
    assert np.allclose(X, np.diag((d + eps) ** (-1.0 / p)), rtol=1e-13, atol=0)


def test_root_2x2_golden():
    """Hand-derived 2x2 cases: [[a,b],[b,a]] has eigenvectors (1,+-1)/sqrt2
    with eigenvalues a+-b, so its root has entries (u+v)/2 and (u-v)/2."""
    with open(os.path.join(GOLDEN, "roots_2x2.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        X = inverse_root(np.array(c["A"], dtype=float), c["eps"], c["p"])
        assert np.allclose(X, np.array(c["X"]), rtol=1e-12, atol=1e-15), c


@pytest.mark.parametrize("p", [2, 4])
@pytest.mark.parametrize("kappa", [1e2, 1e4, 1e6, 1e8])
def test_root_defining_property(p, kappa):
    """X^p (A + eps I) = I, the definition of the inverse p-th root."""
    A, _ = rand_spd(24, kappa, seed=int(np.log10(kappa)) + p)
    eps = 1e-6
    X = inverse_root(A, eps, p)
    Ae = A + eps * np.eye(24)
    lhs = np.linalg.matrix_power(X, p) @ Ae
    assert np.abs(lhs - np.eye(24)).max() < 1e-15 * kappa * 100
    assert np.allclose(X, X.T, atol=1e-14 * np.abs(X).max())
    assert np.linalg.eigvalsh(X).min() > 0


def test_root_rotation_equivariant():
    A, _ = rand_spd(10, 1e3, 7)
    Q, _ = np.linalg.qr(np.random.default_rng(8).standard_normal((10, 10)))
    X1 = inverse_root(Q @ A @ Q.T, 1e-6, 4)
    X2 = Q @ inverse_root(A, 1e-6, 4) @ Q.T
    assert np.allclose(X1, X2, rtol=1e-11, atol=1e-13)


def test_root_of_padded_matrix_keeps_block():
    """A ragged block padded with identity rows/cols: the root of
    blockdiag(A, I) is blockdiag(root(A), (1+eps)^{-1/p} I), so padding never
    changes the valid region (pins the GPU's padded layout)."""
    A, _ = rand_spd(7, 1e4, 3)
    eps, p = 1e-6, 4
    Ap = np.zeros((10, 10))
    Ap[:7, :7] = A
    Ap[7:, 7:] = np.eye(3)
    Xp = inverse_root(Ap, eps, p)
    assert np.allclose(Xp[:7, :7], inverse_root(A, eps, p), rtol=1e-11, atol=1e-14)
    assert np.allclose(Xp[7:, 7:], (1 + eps) ** (-1 / p) * np.eye(3), rtol=1e-12)
    assert np.abs(Xp[:7, 7:]).max() < 1e-14


@pytest.mark.parametrize("p", [2, 4])
@pytest.mark.parametrize("kappa", [1e2, 1e4, 1e6])
def test_newton_agrees_with_eigh(p, kappa):
    """Two independent routes to the same root: coupled Newton vs eigh."""
    A, _ = rand_spd(32, kappa, seed=11 + p)
    X, it, ok = coupled_newton_inverse_root(A, 1e-6, p, tol=1e-12, max_iter=200)
    assert ok and it > 2
    ref = inverse_root(A, 1e-6, p)
    assert np.linalg.norm(X - ref) / np.linalg.norm(ref) < 1e-9


def _scalar_newton(lam, eps, p, tol=1e-6, max_iter=100):
    """The coupled iteration on a diagonal matrix is one scalar iteration per
    eigenvalue: m <- m ((p+1-m)/p)^p, x <- x (p+1-m)/p from m0 = (l+eps)/c^p,
    x0 = c^{-1}, c^p = the largest l + eps (the max row sum of a diagonal)."""
    lam = np.asarray(lam, dtype=np.float64) + eps
    cp = lam.max()
    m, x = lam / cp, np.full(lam.shape, cp ** (-1.0 / p))
    for k in range(max_iter + 1):
        if np.abs(m - 1.0).max() <= tol:
            return x, k
        t = (p + 1 - m) / p
        x, m = x * t, t ** p * m
    return x, None


@pytest.mark.parametrize("p,counts", [(4, [9, 14, 19, 25]), (2, [10, 15, 21, 27])])
def test_newton_on_a_diagonal_is_scalar_newton(p, counts):
    """Iteration count and result of the matrix iteration equal those of the
    scalar recurrence, over spectra spanning kappa = 1e2 ... 1e8 (the counts
    grow by about 5 per factor of 100 in kappa, as the scalar map predicts)."""
    for kappa, expect in zip([1e2, 1e4, 1e6, 1e8], counts):
        lam = np.array([1.0, np.sqrt(kappa), kappa])
        X, it, ok = coupled_newton_inverse_root(np.diag(lam), 1e-12, p)
        xs, ks = _scalar_newton(lam, 1e-12, p)
        assert ok and it == ks == expect, (kappa, it, ks)
        assert np.allclose(np.diag(X), xs, rtol=1e-14, atol=0)
        assert np.abs(X - np.diag(np.diag(X))).max() == 0.0


def _denman_beavers(B, iters=60):
    """Square root and inverse square root of an SPD matrix by the
    Denman-Beavers iteration (Y <- (Y + Z^{-1})/2, Z <- (Z + Y^{-1})/2 from
    Y = B, Z = I), a third route that shares nothing with eigh or Newton."""
    Y, Z = B.copy(), np.eye(B.shape[0])
    for _ in range(iters):
        Y, Z = 0.5 * (Y + np.linalg.inv(Z)), 0.5 * (Z + np.linalg.inv(Y))
    return Y, Z


@pytest.mark.parametrize("p", [2, 4])
def test_root_matches_denman_beavers(p):
    """(A + eps I)^{-1/2} is Denman-Beavers' Z; (A + eps I)^{-1/4} is the
    inverse square root of its square root Y."""
    A, _ = rand_spd(16, 1e4, seed=21 + p)
    B = A + 1e-6 * np.eye(16)
    Y, Z = _denman_beavers(B)
    ref = Z if p == 2 else _denman_beavers(Y)[1]
    X = inverse_root(A, 1e-6, p)
    assert np.linalg.norm(X - ref) / np.linalg.norm(ref) < 1e-10


def test_newton_tolerance_1e6_is_enough_for_1e3():
    """At the cfg tolerance (max|M-I| <= 1e-6) Newton is far inside 1e-3."""
    A, _ = rand_spd(48, 1e8, 21)
    X, it, ok = coupled_newton_inverse_root(A, 1e-6, 4)
    ref = inverse_root(A, 1e-6, 4)
    assert ok
    assert np.linalg.norm(X - ref) / np.linalg.norm(ref) < 1e-5


def test_newton_diverges_flagged_on_nan():
    A = np.eye(4)
    A[1, 1] = np.nan
    _, _, ok = coupled_newton_inverse_root(A, 1e-6, 4)
    assert not ok


# --------------------------------------------------------------------------
# Blocking
# --------------------------------------------------------------------------
def test_block_partition_covers_exactly_once():
    for rows, cols, b in [(64, 32, 64), (4096, 1024, 512), (19, 64, 128),
                          (2304, 256, 128), (5, 7, 2), (1, 1, 1)]:
        cover = np.zeros((rows, cols), dtype=int)
        for r0, c0, m, n in block_partition(rows, cols, b):
            assert 1 <= m <= b and 1 <= n <= b
            cover[r0:r0 + m, c0:c0 + n] += 1
        assert (cover == 1).all()
    segs = vector_segments(1000, 128)
    assert sum(l for _, l in segs) == 1000 and segs[-1] == (896, 104)


def test_workload_block_counts():
    """Block counts of the workloads, by enumerating their shapes."""
    def count(cfg):
        nb = ns = 0
        for s in cfg["shapes"]:
            if len(s) == 2:
                nb += len(block_partition(s[0], s[1], cfg["block_size"]))
            else:
                ns += len(vector_segments(s[0], cfg["block_size"]))
        return nb, ns
    assert count(wl.CONFIGS["single_64x32"]) == (1, 0)
    assert count(wl.CONFIGS["transformer_layer_b512"]) == (48, 4)
    assert count(wl.CONFIGS["transformer_big_b1024"]) == (272, 0)
    assert count(wl.CONFIGS["resnet50_b128"]) == (1576, 430)


# --------------------------------------------------------------------------
# Statistics
# --------------------------------------------------------------------------
@pytest.mark.parametrize("beta2", [1.0, 0.9])
def test_stats_match_bruteforce_history(beta2):
    """L_t[i,j] = sum_s beta2^(t-s) sum_k G_s[i,k] G_s[j,k], summed element by
    element in plain Python from the stored gradient history."""
    rng = np.random.default_rng(5)
    shape, b, T = (5, 3), 4, 4
    hist = [rng.standard_normal(shape) for _ in range(T)]
    o = ShampooOracle([shape, (6,)], b, beta2, 1e-6)
    vh = [rng.standard_normal(6) for _ in range(T)]
    for t in range(T):
        o.update_stats([hist[t], vh[t]])
    for k, (r0, c0, m, n) in enumerate(block_partition(5, 3, b)):
        L, R = o.stats[0][k]
        for i in range(m):
            for j in range(m):
                ref = sum(beta2 ** (T - 1 - s) * sum(hist[s][r0 + i, c0 + q] * hist[s][r0 + j, c0 + q]
                                                     for q in range(n)) for s in range(T))
                assert abs(L[i, j] - ref) < 1e-12
        for i in range(n):
            for j in range(n):
                ref = sum(beta2 ** (T - 1 - s) * sum(hist[s][r0 + q, c0 + i] * hist[s][r0 + q, c0 + j]
                                                     for q in range(m)) for s in range(T))
                assert abs(R[i, j] - ref) < 1e-12
    for k, (s0, ln) in enumerate(vector_segments(6, b)):
        S = o.stats[1][k]
        for i in range(ln):
            for j in range(ln):
                ref = sum(beta2 ** (T - 1 - s) * vh[s][s0 + i] * vh[s][s0 + j] for s in range(T))
                assert abs(S[i, j] - ref) < 1e-12
    a_ref = sum(beta2 ** (T - 1 - s) * hist[s] ** 2 for s in range(T))
    assert np.allclose(o.diag[0], a_ref, rtol=1e-14)


# --------------------------------------------------------------------------
# Whole step: closed forms
# --------------------------------------------------------------------------
@pytest.mark.parametrize("graft", [GRAFT_NONE, GRAFT_ADAGRAD])
@pytest.mark.parametrize("beta2", [1.0, 0.95])
def test_block_size_one_is_diagonal_adagrad(graft, beta2):
    """With 1x1 blocks L = R = a (a scalar per entry) and S = a for 1-D, so
    the update is exactly the diagonal-Adagrad step g / sqrt(a + eps) and the
    graft scale is 1.  Pins blocking, both exponents and eps placement."""
    rng = np.random.default_rng(9)
    shapes = [(3, 4), (5,)]
    eps, lr = 1e-3, 0.1
    o = ShampooOracle(shapes, 1, beta2, eps, p=4, graft=graft)
    W = [rng.standard_normal(s) for s in shapes]
    a = [np.zeros(s) for s in shapes]
    for t in range(4):
        g = [rng.standard_normal(s) for s in shapes]
        Wn = o.step(W, g, lr, do_roots=True)
        for i in range(2):
            a[i] = beta2 * a[i] + g[i] ** 2
            ref = W[i] - lr * g[i] / np.sqrt(a[i] + eps)
            assert np.allclose(Wn[i], ref, rtol=1e-13, atol=1e-14)
            if graft == GRAFT_ADAGRAD:
                assert abs(o.last_scale[i] - 1.0) < 1e-12
        W = Wn


@pytest.mark.parametrize("shape", [(4, 6), (6, 4), (1, 5)])
def test_rank_one_gradient_closed_form(shape):
    """One step with G = u v^T: G is an eigvector direction of both factors,
    L^{-1/4} G R^{-1/4} = G / sqrt(|u|^2 |v|^2 + eps)."""
    rng = np.random.default_rng(4)
    u, v = rng.standard_normal(shape[0]), rng.standard_normal(shape[1])
    G = np.outer(u, v)
    eps = 1e-4
    o = ShampooOracle([shape], 64, 1.0, eps, graft=GRAFT_NONE)
    W = np.zeros(shape)
    Wn = o.step([W], [G], 1.0, do_roots=True)[0]
    ref = -G / np.sqrt(np.sum(G * G) + eps)
    assert np.allclose(Wn, ref, rtol=1e-11, atol=1e-14)


def test_vector_single_step_closed_form():
    """1-D, one step: S = g g^T, and (g g^T + eps I)^{-1/2} g = g/sqrt(|g|^2+eps)
    (full-matrix Adagrad on the segment)."""
    g = np.array([0.3, -1.2, 2.0, 0.5, 0.0, 1.0])
    eps = 1e-3
    o = ShampooOracle([(6,)], 8, 1.0, eps, graft=GRAFT_NONE)
    Wn = o.step([np.zeros(6)], [g], 1.0, do_roots=True)[0]
    assert np.allclose(Wn, -g / np.sqrt(g @ g + eps), rtol=1e-12)


@pytest.mark.parametrize("beta2", [1.0, 0.8])
def test_orientation_closed_form(beta2):
    """Two steps on a 3x4 weight: G1 = al e1 f1^T, G2 = ga e2 f1^T.
    L = beta2 al^2 e1e1^T + ga^2 e2e2^T and R = (beta2 al^2 + ga^2) f1f1^T,
    so P2 = ga (ga^2+eps)^{-1/4} (beta2 al^2+ga^2+eps)^{-1/4} e2 f1^T.
    Swapping L and R, dropping beta2 or using the wrong exponent breaks it."""
    al, ga, eps = 2.0, 0.5, 1e-2
    e = np.eye(3)
    f = np.eye(4)
    G1 = al * np.outer(e[0], f[0])
    G2 = ga * np.outer(e[1], f[0])
    o = ShampooOracle([(3, 4)], 8, beta2, eps, graft=GRAFT_NONE)
    W = np.zeros((3, 4))
    W = o.step([W], [G1], 1.0, do_roots=True)[0]
    W2 = o.step([W], [G2], 1.0, do_roots=True)[0]
    P2 = W - W2
    ref = ga * (ga ** 2 + eps) ** -0.25 * (beta2 * al ** 2 + ga ** 2 + eps) ** -0.25 * np.outer(e[1], f[0])
    assert np.allclose(P2, ref, rtol=1e-12, atol=1e-15)


def test_kronecker_form():
    """P = Lr G Rr is the Kronecker-product preconditioner (Lr (x) Rr) acting
    on the row-major vectorised gradient (segment 6)."""
    rng = np.random.default_rng(12)
    o = ShampooOracle([(3, 5)], 8, 1.0, 1e-3, graft=GRAFT_NONE)
    for _ in range(3):
        o.update_stats([rng.standard_normal((3, 5))])
    o.compute_roots()
    g = rng.standard_normal((3, 5))
    P = o.precondition(0, g)
    Lr, Rr = o.roots[0][0]
    ref = (np.kron(Lr, Rr) @ g.reshape(-1)).reshape(3, 5)
    assert np.allclose(P, ref, rtol=1e-12, atol=1e-14)
    # and Lr, Rr really are the -1/4 roots of the accumulated statistics
    L, R = o.stats[0][0]
    assert np.allclose(np.linalg.matrix_power(Lr, 4) @ (L + 1e-3 * np.eye(3)), np.eye(3), atol=1e-9)
    assert np.allclose(np.linalg.matrix_power(Rr, 4) @ (R + 1e-3 * np.eye(5)), np.eye(5), atol=1e-9)


def test_blocks_are_independent():
    """Without grafting (which couples blocks through the layer norm) a
    blocked ragged parameter behaves exactly like its blocks taken as
    separate parameters."""
    rng = np.random.default_rng(13)
    b = 4
    shape = (2 * b + 1, b + 2)
    blocks = block_partition(*shape, b)
    big = ShampooOracle([shape], b, 0.9, 1e-4, graft=GRAFT_NONE)
    small = ShampooOracle([(m, n) for (_, _, m, n) in blocks], 64, 0.9, 1e-4, graft=GRAFT_NONE)
    W = rng.standard_normal(shape)
    Ws = [W[r0:r0 + m, c0:c0 + n] for (r0, c0, m, n) in blocks]
    for t in range(3):
        g = rng.standard_normal(shape)
        gs = [g[r0:r0 + m, c0:c0 + n] for (r0, c0, m, n) in blocks]
        W = big.step([W], [g], 0.1, do_roots=(t != 1))[0]
        Ws = small.step(Ws, gs, 0.1, do_roots=(t != 1))
        for (r0, c0, m, n), w in zip(blocks, Ws):
            assert np.allclose(W[r0:r0 + m, c0:c0 + n], w, rtol=1e-12, atol=1e-14)


def test_graft_scale_and_zero_gradient():
    rng = np.random.default_rng(14)
    o = ShampooOracle([(4, 4), (3,)], 8, 1.0, 1e-6, graft=GRAFT_ADAGRAD)
    W = [rng.standard_normal((4, 4)), rng.standard_normal(3)]
    g = [rng.standard_normal((4, 4)), np.zeros(3)]
    Wn = o.step(W, g, 0.1, do_roots=True)
    # zero gradient: P = 0 so s = 0 and the weight does not move
    assert np.array_equal(Wn[1], W[1]) and o.last_scale[1] == 0.0
    # nonzero: the step has the diagonal-Adagrad step's Frobenius norm
    D = g[0] / np.sqrt(g[0] ** 2 + 1e-6)
    assert abs(np.linalg.norm(W[0] - Wn[0]) / 0.1 - np.linalg.norm(D)) < 1e-12


def test_stale_roots_are_used_between_root_steps():
    """Segment 14: between root steps the last roots are applied.  With 1x1
    blocks, step 2 without a root update gives P = g2/sqrt(a1+eps) while the
    graft target uses a2."""
    eps = 1e-3
    o = ShampooOracle([(1, 1)], 1, 1.0, eps, graft=GRAFT_ADAGRAD)
    g1, g2 = np.array([[0.7]]), np.array([[-1.3]])
    W = o.step([np.zeros((1, 1))], [g1], 1.0, do_roots=True)[0]
    Wn = o.step([W], [g2], 1.0, do_roots=False)[0]
    a1, a2 = 0.49, 0.49 + 1.69
    P = g2 / np.sqrt(a1 + eps)
    D = g2 / np.sqrt(a2 + eps)
    s = abs(D[0, 0]) / abs(P[0, 0])
    assert np.allclose(W - Wn, s * P, rtol=1e-13)
    assert abs(o.last_scale[0] - np.sqrt((a1 + eps) / (a2 + eps))) < 1e-13


def test_momentum_double_sum():
    """Heavy ball on the grafted step, 1x1 blocks so U_t = D_t:
    W_T = W_0 - lr sum_t sum_{s<=t} mu^(t-s) D_s."""
    rng = np.random.default_rng(15)
    mu, lr, eps, beta2 = 0.9, 0.05, 1e-4, 0.99
    o = ShampooOracle([(2, 3)], 1, beta2, eps, graft=GRAFT_ADAGRAD, momentum=mu)
    W0 = rng.standard_normal((2, 3))
    W = W0
    Ds = []
    a = np.zeros((2, 3))
    for t in range(4):
        g = rng.standard_normal((2, 3))
        a = beta2 * a + g * g
        Ds.append(g / np.sqrt(a + eps))
        W = o.step([W], [g], lr, do_roots=True)[0]
        ref = W0 - lr * sum(sum(mu ** (tt - s) * Ds[s] for s in range(tt + 1)) for tt in range(t + 1))
        assert np.allclose(W, ref, rtol=1e-12, atol=1e-14)


def test_nonfinite_gradient_skips_parameter():
    rng = np.random.default_rng(16)
    o = ShampooOracle([(3, 3), (2, 2)], 4, 0.9, 1e-6)
    W = [rng.standard_normal((3, 3)), rng.standard_normal((2, 2))]
    W = o.step(W, [rng.standard_normal((3, 3)), rng.standard_normal((2, 2))], 0.1, True)
    L_before = o.stats[0][0][0].copy()
    bad = rng.standard_normal((3, 3))
    bad[1, 2] = np.nan
    Wn = o.step(W, [bad, rng.standard_normal((2, 2))], 0.1, False)
    assert np.array_equal(Wn[0], W[0])
    assert np.array_equal(o.stats[0][0][0], L_before)
    assert not np.array_equal(Wn[1], W[1])
    assert o.skipped == {0}


def test_apply_before_roots_raises():
    o = ShampooOracle([(2, 2)], 2, 1.0, 1e-6)
    o.update_stats([np.ones((2, 2))])
    with pytest.raises(RuntimeError):
        o.apply([np.zeros((2, 2))], [np.ones((2, 2))], 0.1)


# --------------------------------------------------------------------------
# Input generators (shared by both sides; no method arithmetic)
# --------------------------------------------------------------------------
def test_bf16_round_is_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1e-3], dtype=np.float32)
    r = wl.bf16_round(x)
    assert r[0] == 1.0 and r[1] == 1.0 and r[2] == 1.0 + 2 ** -6 and r[3] == -2.5
    assert abs(r[4] - 1e-3) / 1e-3 < 2 ** -8
    assert (wl.bf16_round(r) == r).all()


def test_spd_batch_spectrum():
    A, lam = wl.spd_batch(3, 16, seed=0, log10_kappa=(2, 6))
    for i in range(3):
        ev = np.linalg.eigvalsh(A[i])
        assert np.allclose(np.sort(ev), np.sort(lam[i]), rtol=1e-8)
    assert abs(lam[0].max() / lam[0].min() - 1e2) < 1e-6
    assert abs(lam[2].max() / lam[2].min() - 1e6) < 1e-2


# --------------------------------------------------------------------------
# One-sided preconditioning (segment 16, Lemma 1)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("side", [SIDE_LEFT, SIDE_RIGHT])
@pytest.mark.parametrize("shape", [(4, 6), (6, 4)])
def test_one_sided_rank_one_closed_form(side, shape):
    """One step with G = u v^T, one factor only: the kept factor has the
    eigenvalue |u|^2 |v|^2 along G's direction, so its -1/2 power gives
    G / sqrt(|G|^2 + eps) -- the two-sided result, while a -1/4 power or a
    root of the never-accumulated factor would not."""
    rng = np.random.default_rng(11)
    u, v = rng.standard_normal(shape[0]), rng.standard_normal(shape[1])
    G = np.outer(u, v)
    eps = 1e-4
    o = ShampooOracle([shape], 64, 1.0, eps, graft=GRAFT_NONE, sides=[side])
    Wn = o.step([np.zeros(shape)], [G], 1.0, do_roots=True)[0]
    assert np.allclose(Wn, -G / np.sqrt(np.sum(G * G) + eps), rtol=1e-11, atol=1e-14)


def test_one_sided_right_disjoint_columns_closed_form():
    """Right factor only, each step's gradient non-zero in one column c_t:
    R = sum_t beta2^(T-t) |x_t|^2 e_c e_c^T is diagonal, so the last step is
    column c_T divided by sqrt(R[c_T, c_T] + eps)."""
    rng = np.random.default_rng(12)
    m, n, beta2, eps = 5, 4, 0.9, 1e-3
    cols = [0, 2, 0, 3, 2, 0]
    xs = [rng.standard_normal(m) for _ in cols]
    o = ShampooOracle([(m, n)], 64, beta2, eps, graft=GRAFT_NONE, sides=[SIDE_RIGHT])
    W = np.zeros((m, n))
    for c, x in zip(cols, xs):
        G = np.zeros((m, n))
        G[:, c] = x
        Wn = o.step([W], [G], 1.0, do_roots=True)[0]
        W, dW = Wn, Wn - W
    T = len(cols)
    r = sum(beta2 ** (T - 1 - t) * (xs[t] @ xs[t]) for t in range(T) if cols[t] == cols[-1])
    ref = np.zeros((m, n))
    ref[:, cols[-1]] = -xs[-1] / np.sqrt(r + eps)
    assert np.allclose(dW, ref, rtol=1e-11, atol=1e-14)


def test_one_sided_left_column_is_full_matrix_adagrad_on_the_vector():
    """A 2-D m x 1 parameter with only L kept is full-matrix Adagrad on the
    column, which is what the 1-D path does: both give the same weights over
    several grafted momentum steps."""
    rng = np.random.default_rng(13)
    m = 7
    a = ShampooOracle([(m, 1)], 64, 0.95, 1e-4, momentum=0.5, sides=[SIDE_LEFT])
    b = ShampooOracle([(m,)], 64, 0.95, 1e-4, momentum=0.5)
    Wa, Wb = [rng.standard_normal((m, 1))], [None]
    Wb = [Wa[0][:, 0].copy()]
    for t in range(5):
        g = rng.standard_normal(m)
        Wa = a.step(Wa, [g.reshape(m, 1)], 0.1, do_roots=(t % 2 == 0))
        Wb = b.step(Wb, [g], 0.1, do_roots=(t % 2 == 0))
        assert np.allclose(Wa[0][:, 0], Wb[0], rtol=1e-12, atol=1e-15)


def test_one_sided_dropped_factor_stays_zero_with_identity_root():
    rng = np.random.default_rng(14)
    o = ShampooOracle([(6, 9), (9, 6)], 4, 0.9, 1e-6, sides=[SIDE_LEFT, SIDE_RIGHT])
    for _ in range(2):
        o.update_stats([rng.standard_normal((6, 9)), rng.standard_normal((9, 6))])
    o.compute_roots()
    for (L, R), (Lr, Rr) in zip(o.stats[0], o.roots[0]):
        assert not R.any() and np.array_equal(Rr, np.eye(R.shape[0]))
        assert np.allclose(Lr, inverse_root(L, 1e-6, 2.0), rtol=1e-12)
    for (L, R), (Lr, Rr) in zip(o.stats[1], o.roots[1]):
        assert not L.any() and np.array_equal(Lr, np.eye(L.shape[0]))
        assert np.allclose(Rr, inverse_root(R, 1e-6, 2.0), rtol=1e-12)
    exps = [e for _, e in o.matrices()]
    assert exps[:4] == [2.0, 0, 2.0, 0] and exps[-2:] == [0, 2.0]
