"""ecasq_bucket_noalloc: bucketing for callers that cannot allocate device memory.

Callers such as plugins inside a framework whose caching allocator owns all
device memory, or fixed-budget real-time pipelines that forbid cudaMalloc after
start-up, cannot hand the library a workspace. This entry point keeps its
accumulators in a fixed array inside the library instead. The test calls it
through the C ABI twice in a row, with different inputs and sizes, and checks
each result against the workspace entry point ecasq_bucket: counts bit-exact,
moments to the same 1e-9 relative tolerance the other bucket tests use (both go
through the same kernels, so in practice they are identical). The second call
also shows that nothing from the first call leaks into it. It runs last in the
suite (file name) and passes on its own in a fresh process as well.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from entropy_constrained_unbiased_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def E():
    from entropy_constrained_unbiased_b200 import build, ecasq
    assert torch.cuda.is_available()
    build.build()
    ecasq.load()
    return ecasq


def _grid(X, p):
    from oracle import oracle as O
    P, st = O.grid_batch(X, p)
    assert np.all(st == 0)
    return torch.from_numpy(P).cuda()


def test_noalloc_bucket_matches_workspace_bucket_twice(E):
    cases = [W.random_case(71, 40, 3001, "student_t"), W.random_case(72, 7, 20000, "grad")]
    ps = [128, 256]
    for X, p in zip(cases, ps):  # two calls in a row on the same fixed scratch
        Xd = torch.from_numpy(X).cuda()
        P = _grid(X, p)
        c1, A1, B1, s1 = E.bucket_noalloc(Xd, P)
        c0, A0, B0, s0 = E.bucket(Xd, P)
        torch.cuda.synchronize()
        assert torch.equal(s1, s0) and int(s1.abs().sum()) == 0
        assert torch.equal(c1, c0)
        np.testing.assert_allclose(A1.cpu().numpy(), A0.cpu().numpy(), rtol=1e-9, atol=0)
        np.testing.assert_allclose(B1.cpu().numpy(), B0.cpu().numpy(), rtol=1e-9, atol=0)
        assert int(c1.sum()) == X.size


def test_noalloc_rejects_sizes_beyond_the_fixed_scratch(E):
    L = E.load()
    X = torch.zeros((1400, 8), dtype=torch.float32, device="cuda")
    P = torch.zeros((1400, 256), dtype=torch.float64, device="cuda")
    out = torch.zeros(8, dtype=torch.float64, device="cuda")
    st = torch.zeros(1400, dtype=torch.int32, device="cuda")
    rc = L.ecasq_bucket_noalloc(C.c_void_p(X.data_ptr()), C.c_void_p(P.data_ptr()), 1400, 8, 256,
                                C.c_void_p(out.data_ptr()), C.c_void_p(out.data_ptr()), C.c_void_p(out.data_ptr()),
                                C.c_void_p(st.data_ptr()), C.c_void_p(0))
    assert rc == E.ERR_WORKSPACE


def test_noalloc_capacity_boundary_at_p128(E):
    """The fixed 8 MiB scratch must hold round256(24 n (p - 1)) + round256(4 n)
    bytes: at p = 128, n = 2748 rows need 8,387,072 bytes and fit, n = 2749
    need 8,390,144 and are refused without a launch."""
    def need(n, p):
        r = lambda b: (b + 255) // 256 * 256
        return r(24 * n * (p - 1)) + r(4 * n)
    assert need(2748, 128) <= 8 << 20 < need(2749, 128)
    X = W.random_case(73, 2748, 64, "normal")
    Xd = torch.from_numpy(X).cuda()
    P = _grid(X, 128)
    c1, A1, B1, s1 = E.bucket_noalloc(Xd, P)
    c0, A0, B0, s0 = E.bucket(Xd, P)
    torch.cuda.synchronize()
    assert int(s1.abs().sum()) == 0 and torch.equal(c1, c0)
    np.testing.assert_allclose(A1.cpu().numpy(), A0.cpu().numpy(), rtol=1e-9, atol=0)
    L = E.load()
    X2 = torch.zeros((2749, 64), dtype=torch.float32, device="cuda")
    P2 = torch.zeros((2749, 128), dtype=torch.float64, device="cuda")
    out = torch.zeros(8, dtype=torch.float64, device="cuda")
    st = torch.zeros(2749, dtype=torch.int32, device="cuda")
    rc = L.ecasq_bucket_noalloc(C.c_void_p(X2.data_ptr()), C.c_void_p(P2.data_ptr()), 2749, 64, 128,
                                C.c_void_p(out.data_ptr()), C.c_void_p(out.data_ptr()), C.c_void_p(out.data_ptr()),
                                C.c_void_p(st.data_ptr()), C.c_void_p(0))
    assert rc == E.ERR_WORKSPACE
