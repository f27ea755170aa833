"""The allocation-free inverse-root entry point, against the fp64 oracle.

Some callers cannot call cudaMalloc: code whose device memory belongs to a
framework's pooling allocator, code on a path where an allocation's implicit
synchronisation is not acceptable, hosts that forbid allocation after
start-up.  shampoo_batched_inverse_root_noalloc serves them from a 64 MiB
work space compiled into the library.  Here it must

  * give roots within the root tolerance (1e-3 relative Frobenius) of the
    oracle's eigendecomposition root, for every matrix whose condition
    number is <= 1e6, on two calls in a row with different inputs;
  * do so at the largest side it accepts (n = 1024, one matrix per chunk of
    the work space) and at a ragged n = 1000 with a batch spanning several
    chunks;
  * report the same per-matrix iteration counts as the ordinary entry point,
    including the give-up codes, on a batch whose condition numbers reach
    1e8 (float32 rounding makes some of those indefinite: they diverge and
    are retried with a raised ridge) and under an iteration cap that must
    end in SHAMPOO_ENOTCONVERGED;
  * leave the device's free memory unchanged across a call;
  * refuse sizes beyond its work space on the host.

This file is collected last so that a failure here cannot hide the other
tests.
"""
import numpy as np
import pytest

from oracle import inverse_root
from shampoo_second_order_b200 import workloads as wl

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

ROOT_TOL = 1e-3
EPS = 1e-6


def rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


@pytest.fixture(scope="module", autouse=True)
def cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from shampoo_second_order_b200 import _lib
    _lib.lib()
    yield


def noalloc(dA, p, max_iters=100, fill=float("nan")):
    """(status, X, iters) of one no-alloc call on the current stream."""
    from shampoo_second_order_b200 import _lib as L
    batch, n, _ = dA.shape
    X = torch.full_like(dA, fill)
    it = torch.full((batch,), -7, dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    st = L.shampoo_batched_inverse_root_noalloc(dA.data_ptr(), X.data_ptr(), batch, n, p, EPS, 1e-6,
                                                max_iters, it.data_ptr(), s)
    torch.cuda.synchronize()
    return st, X.cpu().numpy(), it.cpu().numpy()


def ordinary(dA, p, max_iters=100):
    from shampoo_second_order_b200 import _lib as L
    batch, n, _ = dA.shape
    X = torch.empty_like(dA)
    it = torch.empty(batch, dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    st = L.shampoo_batched_inverse_root(dA.data_ptr(), X.data_ptr(), batch, n, p, EPS, 1e-6, max_iters,
                                        it.data_ptr(), s)
    torch.cuda.synchronize()
    return st, X.cpu().numpy(), it.cpu().numpy()


def check_against_oracle(A32, lam, X, iters, p, tag):
    kappa = lam.max(1) / lam.min(1)
    compared = 0
    for k in range(A32.shape[0]):
        if kappa[k] > 1e6:
            continue
        ref = inverse_root(A32[k].astype(np.float64), EPS, p)
        assert iters[k] > 0, (tag, k, iters[k])
        assert rel(X[k], ref) <= ROOT_TOL, (tag, k, kappa[k], rel(X[k], ref))
        compared += 1
    return compared


def test_noalloc_matches_oracle_on_two_calls_in_a_row():
    """n = 1024 (the maximum: one matrix per chunk) with p = 4, then a ragged
    n = 1000 batch of 3 (three chunks) with p = 2, back to back."""
    from shampoo_second_order_b200 import _lib as L
    for call, (n, batch, p, seed) in enumerate([(1024, 2, 4, 91), (1000, 3, 2, 92)]):
        A, lam = wl.spd_batch(batch, n, seed=seed, log10_kappa=(2.0, 5.0))
        A32 = A.astype(np.float32)
        st, X, it = noalloc(torch.from_numpy(A32).cuda(), p)
        assert st == L.OK, (call, st)
        assert check_against_oracle(A32, lam, X, it, p, call) == batch


def test_noalloc_small_sides_many_chunks_against_oracle():
    """n = 200 (side 256 in the work space): a batch of 40 spans three chunks."""
    from shampoo_second_order_b200 import _lib as L
    A, lam = wl.spd_batch(40, 200, seed=93, log10_kappa=(1.0, 6.0))
    A32 = A.astype(np.float32)
    st, X, it = noalloc(torch.from_numpy(A32).cuda(), 4)
    assert st == L.OK
    assert check_against_oracle(A32, lam, X, it, 4, "n200") == 40


@pytest.mark.parametrize("p", [4, 2])
def test_noalloc_ill_conditioned_batch_retries_like_the_ordinary_entry_point(p):
    """Condition numbers 1e2..1e8 at n = 512 (four matrices per chunk): the
    float32 rounding of the largest ones leaves A + eps I indefinite, their
    iteration diverges and they run again with a raised ridge on the device.
    The iteration counts (give-up codes included) equal the ordinary entry
    point's, and every matrix with kappa <= 1e6 is within the tolerance of
    the oracle."""
    A, lam = wl.spd_batch(12, 512, seed=94, log10_kappa=(2.0, 8.0))
    A32 = A.astype(np.float32)
    dA = torch.from_numpy(A32).cuda()
    st0, X0, i0 = ordinary(dA, p)
    st1, X1, i1 = noalloc(dA, p)
    assert st0 == st1
    assert np.array_equal(i0, i1), (i0, i1)
    assert np.isfinite(X1).all()
    assert check_against_oracle(A32, lam, X1, i1, p, f"p{p}") >= 8


def test_noalloc_iteration_cap_reports_not_converged():
    """max_iters = 3 cannot reach the tolerance at kappa >= 1e3: the call
    returns SHAMPOO_ENOTCONVERGED and every matrix reports -1-3 like the
    ordinary entry point (which keeps c^{-1} I as the fallback root)."""
    from shampoo_second_order_b200 import _lib as L
    A, _ = wl.spd_batch(5, 300, seed=95, log10_kappa=(3.0, 5.0))
    dA = torch.from_numpy(A.astype(np.float32)).cuda()
    st0, X0, i0 = ordinary(dA, 4, max_iters=3)
    st1, X1, i1 = noalloc(dA, 4, max_iters=3)
    assert st0 == L.ENOTCONVERGED and st1 == L.ENOTCONVERGED
    assert np.array_equal(i0, i1) and (i1 == -4).all(), (i0, i1)
    assert np.array_equal(X0, X1)


def test_noalloc_allocates_no_device_memory():
    """After a first call, a second one leaves the device's free memory as it
    was (measured by the driver, not by torch's allocator)."""
    from shampoo_second_order_b200 import _lib as L
    A, _ = wl.spd_batch(6, 256, seed=96, log10_kappa=(2.0, 4.0))
    dA = torch.from_numpy(A.astype(np.float32)).cuda()
    X = torch.empty_like(dA)
    it = torch.empty(6, dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream

    def call():
        return L.shampoo_batched_inverse_root_noalloc(dA.data_ptr(), X.data_ptr(), 6, 256, 4, EPS, 1e-6,
                                                      100, it.data_ptr(), s)
    assert call() == L.OK
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    assert call() == L.OK
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0


def test_noalloc_rejects_sizes_beyond_its_work_space():
    from shampoo_second_order_b200 import _lib as L
    A = torch.zeros(1, 1100, 1100, device="cuda")
    X = torch.zeros_like(A)
    with pytest.raises(L.ShampooError) as e:
        L.shampoo_batched_inverse_root_noalloc(A.data_ptr(), X.data_ptr(), 1, 1100, 4, 1e-6, 1e-6, 100)
    assert e.value.status == L.EINVAL and "1024" in str(e.value)
