"""Torch-facing handle over the C-ABI: holds one library context and passes
tensor data pointers and the current CUDA stream to it.  All arithmetic runs
in the CUDA library."""
from __future__ import annotations

import numpy as np

from . import _lib as L


class Shampoo:
    """One optimizer state for a fixed list of parameter shapes.

    shapes: (rows, cols) for 2-D parameters, (n,) for 1-D ones.  Gradients
    are float32 or bfloat16 CUDA tensors (grad_dtype "f32" / "bf16"),
    parameters float32 CUDA tensors, all contiguous.
    """

    def __init__(self, shapes, block_size, beta2, eps, p=4, graft=L.GRAFT_ADAGRAD, momentum=0.0,
                 grad_dtype="f32", stream=None):
        import torch
        self.shapes = [tuple(s) for s in shapes]
        self._numel = [int(np.prod(s)) for s in self.shapes]   # checked on every call
        self.block_size = int(block_size)
        if stream is None:
            stream = torch.cuda.current_stream()
        self.stream = stream
        handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
        dt = L.BF16 if grad_dtype == "bf16" else L.F32
        self.ctx = L.shampoo_create(self.shapes, block_size, beta2, eps, p, graft, momentum, dt, handle)

    def _check_tensors(self, ts, what):
        if len(ts) != len(self._numel):
            raise ValueError(f"expected {len(self._numel)} {what}, got {len(ts)}")
        for t, k in zip(ts, self._numel):
            if t.numel() != k or not t.is_cuda or not t.is_contiguous():
                raise ValueError(f"{what} must be contiguous CUDA tensors of the given shapes")

    def update_stats(self, grads):
        self._check_tensors(grads, "grads")
        L.shampoo_update_stats(self.ctx, grads)

    def compute_roots(self):
        """Returns True when every root converged."""
        return L.shampoo_compute_roots(self.ctx) == L.OK

    def compute_roots_async(self):
        """Queue a root job on the library's low-priority stream and return at
        once.  Returns False (nothing queued) while the previous job runs."""
        return L.shampoo_compute_roots_async(self.ctx) != L.EBUSY

    def install_roots(self, wait=False):
        """Swap in a finished job's roots (blocking for it with wait=True).
        Returns True when roots were installed."""
        return L.shampoo_install_roots(self.ctx, wait)[1] == 1

    def roots_generation(self):
        """Root sets put in use so far (sync computes and async installs)."""
        return L.shampoo_roots_generation(self.ctx)

    def apply(self, params, grads, lr):
        self._check_tensors(params, "params")
        self._check_tensors(grads, "grads")
        L.shampoo_apply(self.ctx, params, grads, lr)

    def step(self, params, grads, lr, compute_roots):
        self.update_stats(grads)
        if compute_roots:
            self.compute_roots()
        self.apply(params, grads, lr)

    def root_status(self):
        return L.shampoo_root_status(self.ctx)

    def nonfinite_status(self):
        return L.shampoo_nonfinite_status(self.ctx)

    def set_root_options(self, tol, max_iters):
        L.shampoo_set_root_options(self.ctx, tol, max_iters)

    def set_root_method(self, method="fp64", slices=6):
        """method "fp64" (float64 Newton products) or "int8" (the same products
        emulated on the int8 tensor cores with `slices` 7-bit slices)."""
        L.shampoo_set_root_method(self.ctx, _METHODS[method], slices)

    def set_gemm_tiles(self, pair=True):
        """256 x 256 CTA-pair tiles for the GEMMs where the block side allows
        (the default), or 128 x 128 single-CTA tiles everywhere."""
        L.shampoo_set_gemm_tiles(self.ctx, 1 if pair else 0)

    def set_one_sided(self, index, side):
        """Keep only one factor ("left": L, "right": R, "both": the default)
        for every block of 2-D parameter `index`; before the first step."""
        L.shampoo_set_one_sided(self.ctx, index, _SIDES[side])

    def root_iterations(self):
        return L.shampoo_root_iterations(self.ctx)

    def profile_enable(self, on=True):
        L.shampoo_profile_enable(self.ctx, on)

    def profile_read(self):
        return L.shampoo_profile_read(self.ctx)

    def num_matrices(self):
        return L.shampoo_num_matrices(self.ctx)

    def matrix_info(self, index):
        return L.shampoo_matrix_info(self.ctx, index)

    def read_matrix(self, which, index):
        """The valid corner of statistic `index` (which=0) or its root
        (which=1) as a float32 numpy array."""
        b = self.block_size
        out = np.zeros((b, b), dtype=np.float32)
        L.shampoo_read_matrix(self.ctx, which, index, out.ctypes.data)
        size, _ = self.matrix_info(index)
        return out[:size, :size].copy(), out

    def close(self):
        if self.ctx is not None:
            L.shampoo_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def batched_inverse_root(A, p, eps, tol=1e-6, max_iters=100, stream=None, method="fp64", slices=6):
    """X = (A + eps I)^{-1/p} for a float32 CUDA tensor A [batch, n, n].
    method: "fp64" (float64 products) or "int8" (float64 products emulated
    on the int8 tensor cores with `slices` 7-bit slices).
    Returns (X, iters) with iters an int32 CUDA tensor (negative = gave up)."""
    import torch
    assert A.is_cuda and A.dtype == torch.float32 and A.dim() == 3 and A.is_contiguous()
    batch, n, _ = A.shape
    X = torch.empty_like(A)
    iters = torch.empty(batch, dtype=torch.int32, device=A.device)
    if stream is None:
        stream = torch.cuda.current_stream()
    L.shampoo_batched_inverse_root_ex(A.data_ptr(), X.data_ptr(), batch, n, p, eps, tol, max_iters,
                                      iters.data_ptr(), stream.cuda_stream, _METHODS[method], slices)
    return X, iters


_METHODS = {"fp64": L.ROOTS_FP64, "int8": L.ROOTS_INT8_EMULATED}
_SIDES = {"both": L.SIDES_BOTH, "left": L.SIDE_LEFT, "right": L.SIDE_RIGHT}
