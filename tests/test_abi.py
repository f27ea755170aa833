"""The C-ABI library without a GPU: it loads, exports every entry point
include/shampoo.h declares, and rejects bad arguments on the host with
SHAMPOO_EINVAL before touching the device."""
import ctypes as C
import os
import re

import pytest

from shampoo_second_order_b200 import _lib as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(shampoo_\w+)\s*\(", text)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(L.LIB_PATH):
        import __graft_entry__
        __graft_entry__.build()
    return L.lib()


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert "shampoo_create" in names and "shampoo_batched_inverse_root" in names
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) <= set(L.SIGNATURES), set(names) - set(L.SIGNATURES)


def test_version(lib):
    assert re.match(r"^\d+\.\d+\.\d+$", L.shampoo_version())


@pytest.mark.parametrize("kw,msg", [
    (dict(block_size=100), "block_size"),
    (dict(block_size=32), "block_size"),
    (dict(block_size=2048), "block_size"),
    (dict(beta2=0.0), "beta2"),
    (dict(beta2=1.5), "beta2"),
    (dict(epsilon=0.0), "epsilon"),
    (dict(p=3), "p must"),
    (dict(graft=7), "graft"),
    (dict(momentum=1.0), "momentum"),
    (dict(grad_dtype=5), "dtype"),
])
def test_create_rejects_bad_options(lib, kw, msg):
    args = dict(shapes=[(64, 32)], block_size=64, beta2=1.0, epsilon=1e-6, p=4, graft=1,
                momentum=0.0, grad_dtype=0)
    args.update(kw)
    with pytest.raises(L.ShampooError) as e:
        L.shampoo_create(args["shapes"], args["block_size"], args["beta2"], args["epsilon"],
                         args["p"], args["graft"], args["momentum"], args["grad_dtype"])
    assert e.value.status == L.EINVAL and msg in str(e.value)


def test_create_rejects_bad_shapes(lib):
    ctx = C.c_void_p()
    dims = (C.c_int64 * 2)(0, 5)
    assert lib.shampoo_create(C.byref(ctx), 1, dims, None, 64, 1.0, 1e-6, 4, 1, 0.0, 0, None) == L.EINVAL
    dims = (C.c_int64 * 2)(3, 5)
    nd = (C.c_int32 * 1)(1)          # 1-D must be given as (1, n)
    assert lib.shampoo_create(C.byref(ctx), 1, dims, nd, 64, 1.0, 1e-6, 4, 1, 0.0, 0, None) == L.EINVAL
    assert lib.shampoo_create(C.byref(ctx), 0, dims, None, 64, 1.0, 1e-6, 4, 1, 0.0, 0, None) == L.EINVAL
    assert lib.shampoo_create(None, 1, dims, None, 64, 1.0, 1e-6, 4, 1, 0.0, 0, None) == L.EINVAL
    assert not ctx.value


def test_null_context_calls(lib):
    assert lib.shampoo_update_stats(None, None) == L.EINVAL
    assert lib.shampoo_compute_roots(None) == L.EINVAL
    assert lib.shampoo_apply(None, None, None, 0.1) == L.EINVAL
    assert lib.shampoo_num_matrices(None) == 0
    assert lib.shampoo_compute_roots_async(None) == L.EINVAL
    assert lib.shampoo_install_roots(None, 0, None) == L.EINVAL
    assert lib.shampoo_roots_generation(None) == -1
    assert lib.shampoo_set_root_method(None, 1, 6) == L.EINVAL
    assert lib.shampoo_set_one_sided(None, 0, 1) == L.EINVAL
    lib.shampoo_destroy(None)


@pytest.mark.parametrize("args", [
    (0, 0, 1, 64, 4, 1e-6, 1e-6, 100),        # null pointers
    (8, 8, 0, 64, 4, 1e-6, 1e-6, 100),        # batch 0
    (8, 8, 1, 2048, 4, 1e-6, 1e-6, 100),      # n too large
    (8, 8, 1, 64, 3, 1e-6, 1e-6, 100),        # p
    (8, 8, 1, 64, 4, 0.0, 1e-6, 100),         # eps
    (8, 8, 1, 64, 4, 1e-6, 1e-6, 0),          # max_iters
])
def test_batched_root_rejects_bad_arguments(lib, args):
    a, x, batch, n, p, eps, tol, mi = args
    st = lib.shampoo_batched_inverse_root(C.c_void_p(a), C.c_void_p(x), batch, n, p, eps, tol, mi,
                                          None, None)
    assert st == L.EINVAL


@pytest.mark.parametrize("method,slices", [(2, 6), (1, 3), (1, 8), (-1, 6)])
def test_batched_root_ex_rejects_bad_method(lib, method, slices):
    st = lib.shampoo_batched_inverse_root_ex(C.c_void_p(8), C.c_void_p(8), 1, 64, 4, 1e-6, 1e-6, 100,
                                             None, None, method, slices)
    assert st == L.EINVAL


def test_package_import_does_not_load_library():
    import importlib
    import shampoo_second_order_b200 as pkg
    importlib.reload(pkg)
    from shampoo_second_order_b200 import workloads  # noqa: F401
    assert hasattr(pkg, "lib")


def _c_decls():
    """(return type, name, [parameter types]) of every declaration in include/*.h."""
    out = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        for ret, name, args in re.findall(r"([A-Za-z_][\w\s\*]*?)\b(shampoo_\w+)\s*\(([^;{]*?)\)\s*;", text,
                                          flags=re.S):
            params = [] if args.strip() in ("", "void") else [" ".join(a.split()) for a in args.split(",")]
            # drop the parameter name: the type is everything before the last identifier
            types = [re.sub(r"\s*\b\w+$", "", p).replace(" *", "*") for p in params]
            out.append((" ".join(ret.split()), name, types))
    return out


_SCALAR = {"int": C.c_int, "shampoo_graft": C.c_int, "shampoo_dtype": C.c_int, "int64_t": C.c_int64,
           "int32_t": C.c_int32, "float": C.c_float, "double": C.c_double}


def _matches(ctype, py):
    t = re.sub(r"\bconst\b", "", ctype).replace(" ", "")
    if t.endswith("*"):
        pointee = t[:-1]
        if pointee == "char":
            return py in (C.c_char_p, C.c_void_p)
        if py is C.c_void_p:   # an opaque or untyped pointer
            return True
        base = getattr(py, "_type_", None)
        return base is not None and (_SCALAR.get(pointee) is base or pointee.endswith("*"))
    return _SCALAR.get(t) is py


def test_binding_signatures_match_the_header():
    """Every ctypes signature in the binding has the header's parameter count
    and compatible types, so the binding cannot drift from the C-ABI."""
    decls = _c_decls()
    assert {n for _, n, _ in decls} == set(L.SIGNATURES)
    rets = {"shampoo_status": C.c_int, "int": C.c_int, "int64_t": C.c_int64, "const char*": C.c_char_p,
            "void": None}
    for ret, name, types in decls:
        res, args = L.SIGNATURES[name]
        assert rets[re.sub(r"\s*\*", "*", ret)] is res, (name, ret, res)
        assert len(types) == len(args), (name, types, args)
        for t, a in zip(types, args):
            assert _matches(t, a), (name, t, a)


def test_binding_checks_tensors_against_the_shapes():
    """The per-call checks of the Python binding (sizes from the shapes given
    at construction, contiguity, device) refuse a wrong list before anything
    reaches the library; built without a context, as the checks need none."""
    import torch
    from shampoo_second_order_b200.optimizer import Shampoo
    opt = object.__new__(Shampoo)
    opt.shapes = [(4, 3), (5,)]
    opt._numel = [12, 5]
    with pytest.raises(ValueError, match="expected 2"):
        opt._check_tensors([torch.zeros(4, 3)], "grads")
    with pytest.raises(ValueError, match="contiguous CUDA"):
        opt._check_tensors([torch.zeros(4, 3), torch.zeros(6)], "grads")          # wrong size
    with pytest.raises(ValueError, match="contiguous CUDA"):
        opt._check_tensors([torch.zeros(3, 4).t(), torch.zeros(5)], "grads")      # not contiguous
    with pytest.raises(ValueError, match="contiguous CUDA"):
        opt._check_tensors([torch.zeros(4, 3), torch.zeros(5)], "grads")          # host tensors
