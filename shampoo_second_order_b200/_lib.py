"""ctypes binding of the C-ABI in include/shampoo.h: same names, argument
marshalling only.  Every step of the optimizer runs in the CUDA library;
this module converts Python lists to C arrays and status codes to errors.
"""
from __future__ import annotations

import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libshampoo_b200.so")

OK, EINVAL, ENOMEM, ECUDA, ENONFINITE, ENOTCONVERGED, ESTATE, EBUSY = range(8)
STATUS_NAMES = {0: "OK", 1: "EINVAL", 2: "ENOMEM", 3: "ECUDA", 4: "ENONFINITE",
                5: "ENOTCONVERGED", 6: "ESTATE", 7: "EBUSY"}
GRAFT_NONE, GRAFT_ADAGRAD = 0, 1
ROOTS_FP64, ROOTS_INT8_EMULATED = 0, 1
SIDES_BOTH, SIDE_LEFT, SIDE_RIGHT = 0, 1, 2
F32, BF16 = 0, 1

# name -> (restype, argtypes), exactly the declarations of include/shampoo.h
_P = C.c_void_p
SIGNATURES = {
    "shampoo_create": (C.c_int, [C.POINTER(_P), C.c_int, C.POINTER(C.c_int64), C.POINTER(C.c_int32),
                                 C.c_int, C.c_float, C.c_float, C.c_int, C.c_int, C.c_float, C.c_int, _P]),
    "shampoo_update_stats": (C.c_int, [_P, C.POINTER(_P)]),
    "shampoo_compute_roots": (C.c_int, [_P]),
    "shampoo_compute_roots_async": (C.c_int, [_P]),
    "shampoo_install_roots": (C.c_int, [_P, C.c_int, C.POINTER(C.c_int)]),
    "shampoo_roots_generation": (C.c_int64, [_P]),
    "shampoo_apply": (C.c_int, [_P, C.POINTER(_P), C.POINTER(_P), C.c_float]),
    "shampoo_root_status": (C.c_int, [_P, C.POINTER(C.c_int), C.POINTER(C.c_int)]),
    "shampoo_nonfinite_status": (C.c_int, [_P, C.POINTER(C.c_int)]),
    "shampoo_set_root_options": (C.c_int, [_P, C.c_double, C.c_int]),
    "shampoo_set_root_method": (C.c_int, [_P, C.c_int, C.c_int]),
    "shampoo_set_one_sided": (C.c_int, [_P, C.c_int, C.c_int]),
    "shampoo_num_matrices": (C.c_int, [_P]),
    "shampoo_matrix_info": (C.c_int, [_P, C.c_int, C.POINTER(C.c_int), C.POINTER(C.c_int)]),
    "shampoo_read_matrix": (C.c_int, [_P, C.c_int, C.c_int, _P]),
    "shampoo_root_iterations": (C.c_int, [_P, _P]),
    "shampoo_profile_enable": (C.c_int, [_P, C.c_int]),
    "shampoo_profile_count": (C.c_int, [_P]),
    "shampoo_profile_entry": (C.c_int, [_P, C.c_int, C.c_char_p, C.c_int, C.POINTER(C.c_int64),
                                        C.POINTER(C.c_double)]),
    "shampoo_last_error": (C.c_char_p, [_P]),
    "shampoo_destroy": (None, [_P]),
    "shampoo_batched_inverse_root": (C.c_int, [_P, _P, C.c_int, C.c_int, C.c_int, C.c_float,
                                               C.c_double, C.c_int, _P, _P]),
    "shampoo_batched_inverse_root_ex": (C.c_int, [_P, _P, C.c_int, C.c_int, C.c_int, C.c_float,
                                                  C.c_double, C.c_int, _P, _P, C.c_int, C.c_int]),
    "shampoo_batched_inverse_root_noalloc": (C.c_int, [_P, _P, C.c_int, C.c_int, C.c_int, C.c_float,
                                                       C.c_double, C.c_int, _P, _P]),
    "shampoo_plan_shards": (C.c_int, [C.c_int, C.POINTER(C.c_int64), C.POINTER(C.c_int32), C.c_int, C.c_int,
                                      C.c_int, C.POINTER(C.c_int32), C.POINTER(C.c_double)]),
    "shampoo_selftest_stalled_wait": (C.c_int, [_P]),
    "shampoo_selftest_stall_next_stats": (C.c_int, [_P]),
    "shampoo_set_gemm_tiles": (C.c_int, [_P, C.c_int]),
    "shampoo_selftest_stall_next_apply": (C.c_int, [_P]),
    "shampoo_version": (C.c_char_p, []),
}

_lib = None


class ShampooError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


def lib():
    """Load the compiled library (once).  Raises if it was not built: there
    is no fallback path."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing "
                               "(run python -m shampoo_second_order_b200.build)")
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(st, ctx=None, allow=()):
    if st != OK and st not in allow:
        msg = lib().shampoo_last_error(ctx)
        raise ShampooError(st, msg.decode() if msg else "")
    return st


def _ptrs(xs):
    arr = (C.c_void_p * len(xs))()
    for i, x in enumerate(xs):
        arr[i] = x if isinstance(x, int) else int(x.data_ptr())
    return arr


def shampoo_create(shapes, block_size, beta2, epsilon, p=4, graft=GRAFT_ADAGRAD, momentum=0.0,
                   grad_dtype=F32, stream=0):
    """shapes: list of (rows, cols) or (n,) tuples.  Returns the context handle."""
    n = len(shapes)
    dims = (C.c_int64 * (2 * n))()
    nd = (C.c_int32 * n)()
    for i, s in enumerate(shapes):
        if len(s) == 1:
            dims[2 * i], dims[2 * i + 1], nd[i] = 1, int(s[0]), 1
        else:
            dims[2 * i], dims[2 * i + 1], nd[i] = int(s[0]), int(s[1]), 2
    ctx = C.c_void_p()
    st = lib().shampoo_create(C.byref(ctx), n, dims, nd, int(block_size), float(beta2),
                              float(epsilon), int(p), int(graft), float(momentum), int(grad_dtype),
                              C.c_void_p(int(stream)))
    _check(st, None)
    return ctx


def shampoo_update_stats(ctx, grads):
    return _check(lib().shampoo_update_stats(ctx, _ptrs(grads)), ctx)


def shampoo_compute_roots(ctx):
    return _check(lib().shampoo_compute_roots(ctx), ctx, allow=(ENOTCONVERGED,))


def shampoo_compute_roots_async(ctx):
    """Queue a root job; returns EBUSY (no exception) while the previous one runs."""
    return _check(lib().shampoo_compute_roots_async(ctx), ctx, allow=(EBUSY, ENOTCONVERGED))


def shampoo_install_roots(ctx, wait):
    """(status, installed) of swapping in a finished job's roots."""
    inst = C.c_int()
    st = _check(lib().shampoo_install_roots(ctx, int(wait), C.byref(inst)), ctx, allow=(ENOTCONVERGED,))
    return st, inst.value


def shampoo_roots_generation(ctx):
    return lib().shampoo_roots_generation(ctx)


def shampoo_apply(ctx, params, grads, lr):
    return _check(lib().shampoo_apply(ctx, _ptrs(params), _ptrs(grads), float(lr)), ctx)


def shampoo_root_status(ctx):
    a, b = C.c_int(), C.c_int()
    _check(lib().shampoo_root_status(ctx, C.byref(a), C.byref(b)), ctx)
    return a.value, b.value


def shampoo_nonfinite_status(ctx):
    a = C.c_int()
    _check(lib().shampoo_nonfinite_status(ctx, C.byref(a)), ctx)
    return a.value


def shampoo_set_root_options(ctx, tol, max_iters):
    return _check(lib().shampoo_set_root_options(ctx, float(tol), int(max_iters)), ctx)


def shampoo_set_root_method(ctx, method, slices=6):
    return _check(lib().shampoo_set_root_method(ctx, int(method), int(slices)), ctx)


def shampoo_set_one_sided(ctx, param, side):
    return _check(lib().shampoo_set_one_sided(ctx, int(param), int(side)), ctx)


def shampoo_num_matrices(ctx):
    return lib().shampoo_num_matrices(ctx)


def shampoo_matrix_info(ctx, index):
    s, p = C.c_int(), C.c_int()
    _check(lib().shampoo_matrix_info(ctx, int(index), C.byref(s), C.byref(p)), ctx)
    return s.value, p.value


def shampoo_read_matrix(ctx, which, index, dst_ptr):
    return _check(lib().shampoo_read_matrix(ctx, int(which), int(index), C.c_void_p(int(dst_ptr))), ctx)


def shampoo_root_iterations(ctx):
    n = shampoo_num_matrices(ctx)
    out = (C.c_int32 * n)()
    _check(lib().shampoo_root_iterations(ctx, out), ctx)
    return list(out)


def shampoo_profile_enable(ctx, on):
    return _check(lib().shampoo_profile_enable(ctx, int(on)), ctx)


def shampoo_profile_read(ctx):
    """{kernel name: (launches, total ms)} since the last enable."""
    out = {}
    buf = C.create_string_buffer(64)
    for i in range(lib().shampoo_profile_count(ctx)):
        n, ms = C.c_int64(), C.c_double()
        _check(lib().shampoo_profile_entry(ctx, i, buf, 64, C.byref(n), C.byref(ms)), ctx)
        out[buf.value.decode()] = (n.value, ms.value)
    return out


def shampoo_destroy(ctx):
    lib().shampoo_destroy(ctx)


def shampoo_batched_inverse_root(A_ptr, X_ptr, batch, n, p, eps, tol, max_iters, iters_ptr=0,
                                 stream=0):
    st = lib().shampoo_batched_inverse_root(C.c_void_p(int(A_ptr)), C.c_void_p(int(X_ptr)),
                                            int(batch), int(n), int(p), float(eps), float(tol),
                                            int(max_iters), C.c_void_p(int(iters_ptr)),
                                            C.c_void_p(int(stream)))
    return _check(st, None, allow=(ENOTCONVERGED,))


def shampoo_batched_inverse_root_ex(A_ptr, X_ptr, batch, n, p, eps, tol, max_iters, iters_ptr=0,
                                    stream=0, method=ROOTS_FP64, slices=6):
    st = lib().shampoo_batched_inverse_root_ex(C.c_void_p(int(A_ptr)), C.c_void_p(int(X_ptr)),
                                               int(batch), int(n), int(p), float(eps), float(tol),
                                               int(max_iters), C.c_void_p(int(iters_ptr)),
                                               C.c_void_p(int(stream)), int(method), int(slices))
    return _check(st, None, allow=(ENOTCONVERGED,))


def shampoo_batched_inverse_root_noalloc(A_ptr, X_ptr, batch, n, p, eps, tol, max_iters, iters_ptr=0,
                                         stream=0):
    st = lib().shampoo_batched_inverse_root_noalloc(C.c_void_p(int(A_ptr)), C.c_void_p(int(X_ptr)),
                                                    int(batch), int(n), int(p), float(eps), float(tol),
                                                    int(max_iters), C.c_void_p(int(iters_ptr)),
                                                    C.c_void_p(int(stream)))
    return _check(st, None, allow=(ENOTCONVERGED,))


def shampoo_plan_shards(shapes, block_size, root_interval, nranks):
    """(owner per parameter, planned cost per rank); host only."""
    n = len(shapes)
    dims = (C.c_int64 * (2 * n))()
    nd = (C.c_int32 * n)()
    for i, s in enumerate(shapes):
        if len(s) == 1:
            dims[2 * i], dims[2 * i + 1], nd[i] = 1, int(s[0]), 1
        else:
            dims[2 * i], dims[2 * i + 1], nd[i] = int(s[0]), int(s[1]), 2
    owner = (C.c_int32 * n)()
    cost = (C.c_double * int(nranks))()
    _check(lib().shampoo_plan_shards(n, dims, nd, int(block_size), int(root_interval), int(nranks), owner, cost))
    return list(owner), list(cost)


def shampoo_set_gemm_tiles(ctx, pair):
    return _check(lib().shampoo_set_gemm_tiles(ctx, int(pair)), ctx)


def shampoo_selftest_stall_next_stats(ctx):
    return _check(lib().shampoo_selftest_stall_next_stats(ctx), ctx)


def shampoo_selftest_stall_next_apply(ctx):
    return _check(lib().shampoo_selftest_stall_next_apply(ctx), ctx)


def shampoo_version():
    return lib().shampoo_version().decode()
