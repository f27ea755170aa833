"""Seeded synthetic inputs for the Shampoo step: shapes, weights, gradients,
and SPD test matrices.

This module holds none of the optimizer's arithmetic.  It only draws random
numbers (numpy PCG64, seeded) and lays them out in the shapes of the
workloads the paper trains (a Transformer layer, Transformer-Big, ResNet-50)
and of the batched inverse-root test.  The CUDA path and the fp64 oracle both
take their inputs from here; neither imports the other.

Parameter shapes are lists of tuples: (rows, cols) for a 2-D parameter and
(n,) for a 1-D one.  "N(0, s)" means a normal with standard deviation s.
"""
from __future__ import annotations

import numpy as np

GRAFT_NONE = 0
GRAFT_ADAGRAD = 1


def transformer_layer_shapes():
    """One Transformer layer at d_model=1024, ffn=4096: Q, K, V, O projections,
    the two FFN matrices and two 1024 biases."""
    return [(1024, 1024)] * 4 + [(1024, 4096), (4096, 1024), (1024,), (1024,)]


def transformer_big_shapes(layers=12, d_model=1024, ffn=8192, vocab=32768):
    """Transformer-Big-shaped matrices: per layer 4 attention projections and
    two FFN matrices, plus a vocab x d_model embedding."""
    per = [(d_model, d_model)] * 4 + [(d_model, ffn), (ffn, d_model)]
    return per * layers + [(vocab, d_model)]


def resnet50_shapes():
    """ResNet-50 v1 weights reshaped to 2-D, with BN scale/shift and the FC
    bias as 1-D parameters.

    Conv kernels (kh, kw, Cin, Cout) become (kh*kw*Cin) x Cout.  Stem 7x7x3->64,
    four bottleneck stages of [3, 4, 6, 3] blocks with widths 64..512 and
    expansion 4, a 1x1 projection shortcut on the first block of each stage,
    FC 2048 -> 1000.
    """
    mats, vecs = [(7 * 7 * 3, 64)], [64, 64]
    cin = 64
    for w, nb in zip([64, 128, 256, 512], [3, 4, 6, 3]):
        for i in range(nb):
            for shape in ((cin, w), (9 * w, w), (w, 4 * w)):
                mats.append(shape)
                vecs += [shape[1], shape[1]]
            if i == 0:
                mats.append((cin, 4 * w))
                vecs += [4 * w, 4 * w]
            cin = 4 * w
    mats.append((2048, 1000))
    vecs.append(1000)
    return mats + [(v,) for v in vecs]


# The five workloads.  lr=0.1 and W0 ~ N(0, 0.02) are taken for all of them;
# momentum is only used by the Transformer-Big set.
CONFIGS = {
    "single_64x32": dict(
        shapes=[(64, 32)], block_size=64, beta2=1.0, eps=1e-6, p=4,
        graft=GRAFT_ADAGRAD, momentum=0.0, lr=0.1, grad_dtype="f32",
        grad_std=1.0, root_interval=1, steps=10, seed=1),
    "transformer_layer_b512": dict(
        shapes=transformer_layer_shapes(), block_size=512, beta2=0.999,
        eps=1e-6, p=4, graft=GRAFT_ADAGRAD, momentum=0.0, lr=0.1,
        grad_dtype="bf16", grad_std=1e-3, root_interval=20, steps=100, seed=2),
    "transformer_big_b1024": dict(
        shapes=transformer_big_shapes(), block_size=1024, beta2=0.999,
        eps=1e-6, p=4, graft=GRAFT_ADAGRAD, momentum=0.9, lr=0.1,
        grad_dtype="f32", grad_std=1e-3, root_interval=100, steps=100, seed=4),
    "resnet50_b128": dict(
        shapes=resnet50_shapes(), block_size=128, beta2=0.99, eps=1e-6, p=4,
        graft=GRAFT_ADAGRAD, momentum=0.0, lr=0.1, grad_dtype="f32",
        grad_std=1e-2, root_interval=50, steps=100, seed=5),
}

# The batched inverse-root workload: 256 SPD 512x512 matrices.
ROOTS_CONFIG = dict(batch=256, n=512, eps=1e-6, ps=(4, 2), tol=1e-6, seed=3,
                    log10_kappa=(2.0, 8.0))


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even) and return
    them as float32 (a storage conversion of the inputs, nothing more)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> 16) & 1) + np.uint32(0x7FFF)
    r = ((u + bias) & np.uint32(0xFFFF0000)).astype(np.uint32)
    return r.view(np.float32)


def bf16_bits(x32: np.ndarray) -> np.ndarray:
    """The upper 16 bits of float32 values that are already bf16-exact."""
    return (np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def make_params(shapes, seed, std=0.02):
    rng = np.random.Generator(np.random.PCG64(seed))
    return [(rng.standard_normal(s) * std).astype(np.float32) for s in shapes]


def make_grads(shapes, seed, step, std, dtype="f32"):
    """Gradients of one step: N(0, std) float32, rounded to bf16 if asked.
    Always returned as float32 arrays holding the exact values."""
    rng = np.random.Generator(np.random.PCG64([seed, 1000 + step]))
    out = []
    for s in shapes:
        g = (rng.standard_normal(s, dtype=np.float32) * np.float32(std)).astype(np.float32)
        if dtype == "bf16":
            g = bf16_round(g)
        out.append(g)
    return out


def spd_batch(batch, n, seed, log10_kappa=(2.0, 8.0)):
    """SPD test matrices Q diag(lam) Q^T, float64.

    Matrix i has condition number kappa_i = 10^(lo + (hi-lo) i/(batch-1));
    its eigenvalues are log-uniform on [1, kappa_i] with both ends present; Q
    is the orthogonal factor of a seeded Gaussian matrix's QR.
    Returns (A [batch, n, n], lam [batch, n]).
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    lo, hi = log10_kappa
    A = np.empty((batch, n, n))
    lams = np.empty((batch, n))
    for i in range(batch):
        k = lo + (hi - lo) * (i / max(batch - 1, 1))
        e = rng.uniform(0.0, k, size=n)
        e[0], e[-1] = 0.0, k
        lam = 10.0 ** e
        Q, Rq = np.linalg.qr(rng.standard_normal((n, n)))
        Q = Q * np.sign(np.diag(Rq))
        A[i] = (Q * lam) @ Q.T
        A[i] = 0.5 * (A[i] + A[i].T)
        lams[i] = lam
    return A, lams


def count_params(shapes):
    return int(sum(int(np.prod(s)) for s in shapes))
