"""Plain fp64 CPU oracle of the Shampoo optimizer step.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs use it.  It shares no code with the CUDA library: it takes
numpy arrays in and gives numpy arrays back, every step in float64, written
for a reader to check by eye, with no blocking, fusion or reordering beyond
what each definition states.

What it follows (all citations are to the pages on "Scalable Second Order
Optimization for Deep Learning", Anil, Gupta, Koren, Regan, Singer):

* arXiv abstract (mlsanity.com/paper/2002.09018, "Abstract"): the method is
  a form of full-matrix Adagrad.
* podcast transcript (podcast.do-not-panic.com, segments 6-8): Shampoo keeps
  one small matrix per dimension of a weight, L for the rows and R for the
  columns, and uses their Kronecker product in place of the full
  preconditioner.
* segment 10: three extra pieces of work per step -- accumulate gradient
  outer products into L and R, take inverse fourth roots of L and R, and
  multiply the gradient by them.
* segment 12: the root is taken by a coupled Newton iteration (or an SVD) in
  double precision.
* segment 14: the roots L^{-1/4}, R^{-1/4} are recomputed only every so many
  steps; stale roots are used in between.
* segment 16: large layers are split into blocks, each preconditioned on its
  own (Lemma 2); for a layer too large even for that (a big embedding or
  softmax), only one of L and R is kept (Lemma 1).

The pages print no formula, constant or worked example.  Where they are
silent this module takes the plainest reading, listed here once:

* statistics: L <- beta2*L + G G^T, R <- beta2*R + G^T G, starting from zero,
  no (1-beta2) factor; beta2 = 1 is plain Adagrad accumulation.
* root: (A + eps*I)^{-1/p} with an absolute ridge eps, by symmetric
  eigendecomposition; eigenvalues are clamped below at eps against rounding.
* exponents: p (=4) for both factors of a 2-D block; a 1-D parameter keeps one
  statistic per segment, S <- beta2*S + g g^T, taken to the power -2/p (=-1/2:
  full-matrix Adagrad on the segment).
* blocking: row-major grid of <= b x b blocks from the top-left corner; the
  last block row / column is ragged; blocks are never padded here.
* grafting ("layer-wise", to diagonal Adagrad): a <- beta2*a + g*g,
  D = g / sqrt(a + eps), s = ||D||_F / ||P||_F over the whole parameter
  (s = 0 when ||P||_F = 0), update U = s * P.
* momentum (heavy ball, m0 = 0): m <- mu*m + U; W <- W - lr*m.
* one-sided blocks (Lemma 1): the kept factor is accumulated as above and
  taken to the power -2/p (-1/2 for p = 4: full-matrix Adagrad along that
  dimension, the exponent of the 1-D case); the dropped factor is never
  accumulated and its root is the identity, so P = L^{-2/p} G or G R^{-2/p}.
* roots are first computed after the first statistics update and then at the
  caller's interval; apply never runs without roots.
* a gradient holding a NaN or an infinity leaves its parameter untouched for
  that step: no statistics, accumulator, momentum or weight change.
"""
from __future__ import annotations

import numpy as np

GRAFT_NONE = 0
GRAFT_ADAGRAD = 1
SIDES_BOTH = 0     # L and R
SIDE_LEFT = 1      # L only (Lemma 1)
SIDE_RIGHT = 2     # R only (Lemma 1)


# ---------------------------------------------------------------------------
# Blocking (segment 16, Lemma 2)
# ---------------------------------------------------------------------------
def block_partition(rows: int, cols: int, b: int):
    """Blocks of a rows x cols parameter as (r0, c0, m, n), row-major grid.

    Each block is at most b x b; the last block row and column take what is
    left (segment 16: "block the tensor into smaller chunks and precondition
    each block separately").
    """
    out = []
    for r0 in range(0, rows, b):
        for c0 in range(0, cols, b):
            out.append((r0, c0, min(b, rows - r0), min(b, cols - c0)))
    return out


def vector_segments(n: int, b: int):
    """Segments of a length-n 1-D parameter as (s0, length), each <= b."""
    return [(s0, min(b, n - s0)) for s0 in range(0, n, b)]


# ---------------------------------------------------------------------------
# Inverse p-th root (segments 10, 12, 14)
# ---------------------------------------------------------------------------
def inverse_root(A: np.ndarray, eps: float, p: float) -> np.ndarray:
    """(A + eps*I)^{-1/p} of a symmetric PSD matrix, by eigendecomposition.

    Segment 12 names an SVD as one admissible route; for a symmetric PSD
    matrix the symmetric eigendecomposition is that SVD.  Eigenvalues are
    clamped below at eps so that rounding cannot push one under the ridge.
    """
    A = np.asarray(A, dtype=np.float64)
    n = A.shape[0]
    if n == 0:
        return np.zeros((0, 0))
    sym = 0.5 * (A + A.T)
    lam, Q = np.linalg.eigh(sym + eps * np.eye(n))
    lam = np.maximum(lam, eps)
    return (Q * lam ** (-1.0 / p)) @ Q.T


def coupled_newton_inverse_root(A: np.ndarray, eps: float, p: int,
                                tol: float = 1e-6, max_iter: int = 100):
    """(A + eps*I)^{-1/p} by the coupled Newton iteration, in float64.

    This is the root route segment 12 names, run on host cores in double
    precision as segments 12-16 describe.  It is the published coupled
    Newton iteration for the inverse p-th root (Guo & Higham 2006): with
    c^p an upper bound on the largest eigenvalue,
        X_0 = c^{-1} I,  M_0 = (A + eps I) / c^p,
        T_k = ((p+1) I - M_k) / p,  X_{k+1} = X_k T_k,  M_{k+1} = T_k^p M_k,
    so that M_k = X_k^p (A + eps I) throughout and M_k -> I, X_k -> root.
    c^p = min(||A+eps I||_F, ||A+eps I||_inf): both bound the largest
    eigenvalue of a symmetric matrix, so every eigenvalue of M_0 is in (0, 1]
    and the scalar map m -> m((p+1-m)/p)^p drives it monotonically to 1.
    Stops when max|M - I| <= tol; gives up (converged=False) on a non-finite
    residual, on 5 consecutive non-decreasing residuals, or at max_iter.

    Returns (X, iterations, converged).
    """
    A = np.asarray(A, dtype=np.float64)
    n = A.shape[0]
    I = np.eye(n)
    Ae = 0.5 * (A + A.T) + eps * I
    cp = min(np.linalg.norm(Ae, 'fro'), np.abs(Ae).sum(axis=1).max())
    X = cp ** (-1.0 / p) * I
    M = Ae / cp
    prev = np.inf
    worse = 0
    for k in range(max_iter + 1):
        res = np.abs(M - I).max()
        if not np.isfinite(res):
            return X, k, False
        if res <= tol:
            return X, k, True
        if k == max_iter:
            break
        worse = worse + 1 if res >= prev else 0
        if worse >= 5:
            return X, k, False
        prev = res
        T = ((p + 1) * I - M) / p
        X = X @ T
        M = np.linalg.matrix_power(T, p) @ M
    return X, max_iter, False


# ---------------------------------------------------------------------------
# The optimizer state and step (segment 10: stats, roots, multiply)
# ---------------------------------------------------------------------------
class ShampooOracle:
    """Blocked Shampoo with layer-wise Adagrad grafting, all in float64.

    ``shapes`` is a list of (rows, cols) for 2-D parameters and (n,) for 1-D
    ones.  ``sides`` (optional) gives per parameter SIDES_BOTH, SIDE_LEFT or
    SIDE_RIGHT (2-D parameters only).  State persists across calls; one
    optimizer step is ``update_stats(grads)``, then ``compute_roots()`` on
    root steps, then ``apply(params, grads, lr)``.
    """

    def __init__(self, shapes, block_size, beta2, eps, p=4,
                 graft=GRAFT_ADAGRAD, momentum=0.0, root_route="eigh", sides=None):
        self.shapes = [tuple(int(d) for d in s) for s in shapes]
        self.b = int(block_size)
        self.beta2 = float(beta2)
        self.eps = float(eps)
        self.p = int(p)
        self.graft = int(graft)
        self.mu = float(momentum)
        self.root_route = root_route
        self.sides = [SIDES_BOTH] * len(self.shapes) if sides is None else [int(x) for x in sides]
        self.blocks = []      # per param: list of block tuples
        self.stats = []       # per param: list of (L, R) or [S]
        self.roots = []       # per param: list of (Lr, Rr) or [Sr], or None
        self.diag = []        # per param: Adagrad accumulator a
        self.mom = []         # per param: momentum buffer m
        for s in self.shapes:
            if len(s) == 2:
                blks = block_partition(s[0], s[1], self.b)
                st = [(np.zeros((m, m)), np.zeros((n, n))) for (_, _, m, n) in blks]
            else:
                blks = vector_segments(s[0], self.b)
                st = [np.zeros((ln, ln)) for (_, ln) in blks]
            self.blocks.append(blks)
            self.stats.append(st)
            self.roots.append(None)
            self.diag.append(np.zeros(s))
            self.mom.append(np.zeros(s))
        self.steps = 0
        self.skipped = set()
        self.last_scale = [0.0] * len(self.shapes)
        self.newton_iters = []

    # -- segment 10, first piece: accumulate outer products into L and R
    def update_stats(self, grads):
        self.skipped = set()
        for i, s in enumerate(self.shapes):
            g = np.asarray(grads[i], dtype=np.float64).reshape(s)
            if not np.all(np.isfinite(g)):
                self.skipped.add(i)
                continue
            if len(s) == 2:
                side = self.sides[i]
                for k, (r0, c0, m, n) in enumerate(self.blocks[i]):
                    G = g[r0:r0 + m, c0:c0 + n]
                    L, R = self.stats[i][k]
                    if side != SIDE_RIGHT:
                        L = self.beta2 * L + G @ G.T
                    if side != SIDE_LEFT:
                        R = self.beta2 * R + G.T @ G
                    self.stats[i][k] = (L, R)
            else:
                for k, (s0, ln) in enumerate(self.blocks[i]):
                    v = g[s0:s0 + ln].reshape(ln, 1)
                    self.stats[i][k] = self.beta2 * self.stats[i][k] + v @ v.T
            self.diag[i] = self.beta2 * self.diag[i] + g * g
        self.steps += 1

    def _root(self, A, p):
        if self.root_route == "newton":
            X, it, ok = coupled_newton_inverse_root(A, self.eps, p)
            self.newton_iters.append((it, ok))
            return X
        return inverse_root(A, self.eps, p)

    # -- segment 10, second piece; segment 14: only on root steps
    def compute_roots(self):
        p2 = self.p / 2.0
        for i, s in enumerate(self.shapes):
            if len(s) == 2:
                side = self.sides[i]
                if side == SIDE_LEFT:
                    self.roots[i] = [(self._root(L, p2), np.eye(R.shape[0])) for (L, R) in self.stats[i]]
                elif side == SIDE_RIGHT:
                    self.roots[i] = [(np.eye(L.shape[0]), self._root(R, p2)) for (L, R) in self.stats[i]]
                else:
                    self.roots[i] = [(self._root(L, self.p), self._root(R, self.p))
                                     for (L, R) in self.stats[i]]
            else:
                self.roots[i] = [self._root(S, p2) for S in self.stats[i]]

    def precondition(self, i, g):
        """P = L^{-1/p} G R^{-1/p} per block (segment 10, third piece)."""
        s = self.shapes[i]
        g = np.asarray(g, dtype=np.float64).reshape(s)
        P = np.zeros(s)
        if len(s) == 2:
            for (r0, c0, m, n), (Lr, Rr) in zip(self.blocks[i], self.roots[i]):
                P[r0:r0 + m, c0:c0 + n] = Lr @ g[r0:r0 + m, c0:c0 + n] @ Rr
        else:
            for (s0, ln), Sr in zip(self.blocks[i], self.roots[i]):
                P[s0:s0 + ln] = Sr @ g[s0:s0 + ln]
        return P

    def apply(self, params, grads, lr):
        """Grafted, momentum-smoothed update; returns the new parameters."""
        if any(r is None for r in self.roots):
            raise RuntimeError("apply before compute_roots")
        out = []
        for i, s in enumerate(self.shapes):
            if i in self.skipped:
                out.append(np.asarray(params[i], dtype=np.float64).reshape(s).copy())
                continue
            g = np.asarray(grads[i], dtype=np.float64).reshape(s)
            P = self.precondition(i, g)
            if self.graft == GRAFT_ADAGRAD:
                D = g / np.sqrt(self.diag[i] + self.eps)
                nP = np.linalg.norm(P)
                scale = np.linalg.norm(D) / nP if nP > 0 else 0.0
            else:
                scale = 1.0
            self.last_scale[i] = scale
            U = scale * P
            self.mom[i] = self.mu * self.mom[i] + U
            w = np.asarray(params[i], dtype=np.float64).reshape(s)
            out.append(w - lr * self.mom[i])
        return out

    def step(self, params, grads, lr, do_roots):
        self.update_stats(grads)
        if do_roots:
            self.compute_roots()
        return self.apply(params, grads, lr)

    # -- views used by the parity tests
    def matrices(self):
        """All statistics in the library's order: per 2-D block L then R,
        then per 1-D segment S; with the exponent each is rooted at."""
        mats = []
        for i, s in enumerate(self.shapes):
            if len(s) == 2:
                side = self.sides[i]
                pl = {SIDES_BOTH: self.p, SIDE_LEFT: self.p / 2.0, SIDE_RIGHT: 0}[side]
                pr = {SIDES_BOTH: self.p, SIDE_LEFT: 0, SIDE_RIGHT: self.p / 2.0}[side]
                for (L, R) in self.stats[i]:
                    mats.append((L, pl))      # exponent 0: a dropped factor, root I
                    mats.append((R, pr))
        for i, s in enumerate(self.shapes):
            if len(s) == 1:
                for S in self.stats[i]:
                    mats.append((S, self.p / 2.0))
        return mats

    def root_matrices(self):
        out = []
        for i, s in enumerate(self.shapes):
            if len(s) == 2:
                for (Lr, Rr) in self.roots[i]:
                    out.append(Lr)
                    out.append(Rr)
        for i, s in enumerate(self.shapes):
            if len(s) == 1:
                out.extend(self.roots[i])
        return out
