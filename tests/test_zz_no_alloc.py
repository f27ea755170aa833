"""The allocation-free inverse-root entry point against the ordinary one.

shampoo_batched_inverse_root_noalloc serves callers that cannot call
cudaMalloc (memory owned by a framework's pool, no allocation allowed after
start-up): it keeps its work space in a 64 MiB array inside the library.  Two
calls in a row, on different inputs, must each agree with
shampoo_batched_inverse_root on the same inputs within the root tolerance;
sizes beyond the work space's maximum are refused on the host.  This file is
collected last so that a failure here cannot hide the other tests.
"""
import numpy as np
import pytest

from shampoo_second_order_b200 import workloads as wl

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

ROOT_TOL = 1e-3


def rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


@pytest.fixture(scope="module", autouse=True)
def cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from shampoo_second_order_b200 import _lib
    _lib.lib()
    yield


def both(A, p):
    from shampoo_second_order_b200 import _lib as L
    batch, n, _ = A.shape
    dA = torch.from_numpy(A).cuda()
    X0 = torch.empty_like(dA)
    X1 = torch.full_like(dA, float("nan"))
    i0 = torch.empty(batch, dtype=torch.int32, device="cuda")
    i1 = torch.full((batch,), -7, dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    L.shampoo_batched_inverse_root(dA.data_ptr(), X0.data_ptr(), batch, n, p, 1e-6, 1e-6, 100,
                                   i0.data_ptr(), s)
    L.shampoo_batched_inverse_root_noalloc(dA.data_ptr(), X1.data_ptr(), batch, n, p, 1e-6, 1e-6, 100,
                                           i1.data_ptr(), s)
    torch.cuda.synchronize()
    return X0.cpu().numpy(), X1.cpu().numpy(), i0.cpu().numpy(), i1.cpu().numpy()


def test_noalloc_matches_ordinary_entry_point_twice():
    for call, (n, batch, p) in enumerate([(200, 9, 4), (512, 6, 2)]):
        A, _ = wl.spd_batch(batch, n, seed=90 + call, log10_kappa=(2.0, 5.0))
        X0, X1, i0, i1 = both(A.astype(np.float32), p)
        assert np.array_equal(i0, i1), (call, i0, i1)
        for k in range(batch):
            assert rel(X1[k], X0[k]) <= ROOT_TOL, (call, k, rel(X1[k], X0[k]))


def test_noalloc_rejects_sizes_beyond_its_work_space():
    from shampoo_second_order_b200 import _lib as L
    A = torch.zeros(1, 1100, 1100, device="cuda")
    X = torch.zeros_like(A)
    with pytest.raises(L.ShampooError) as e:
        L.shampoo_batched_inverse_root_noalloc(A.data_ptr(), X.data_ptr(), 1, 1100, 4, 1e-6, 1e-6, 100)
    assert e.value.status == L.EINVAL and "1024" in str(e.value)
