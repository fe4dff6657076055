"""The limits of the C ABI on the GPU, against the oracle: the largest alphabet
(p = 512) for the exact solver in both memory modes, the largest code size
(s = 255) for the approximation, a 256-value code for the encoder (indices up to
255 in uint8), and zero-sized or out-of-range sizes rejected before any launch.
Tolerances as in the other parity tests.
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


def _cu(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.parametrize("hirschberg", [False, True])
def test_exact_solver_at_p512(E, O, hirschberg):
    X = W.random_case(81, 1, 5000, "normal")
    P, _ = O.grid_batch(X, 512)
    lam = np.var(X.astype(np.float64), axis=1)[:, None] * 0.02
    g = E.solve(_cu(X), _cu(P), 12, _cu(lam), hirschberg=hirschberg)
    ref = O.solve_batch(X, P, 12, lam)
    m = int(g["Q_len"][0, 0])
    q = g["Q"][0, 0, :m].cpu().numpy()
    mse, H, _ = O.eval_raw(X[0], P[0][q])
    assert mse + lam[0, 0] * H <= ref["J"][0, 0] * (1 + 1e-5)
    assert int(g["status"].abs().sum()) == 0


def test_approximation_at_s255_p512(E, O):
    X = W.random_case(82, 2, 20000, "laplace")
    P, _ = O.grid_batch(X, 512)
    lam = np.var(X.astype(np.float64), axis=1)[:, None] * np.array([[0.0, 1e-3]])
    g = E.solve_approx(_cu(X), _cu(P), 255, _cu(lam))
    ref = O.solve_approx_batch(X, P, 255, lam)
    assert int(g["status"].abs().sum()) == 0
    Q, m = g["Q"].cpu().numpy(), g["Q_len"].cpu().numpy()
    for r in range(2):
        for t in range(2):
            code = Q[r, t, : m[r, t]]
            assert m[r, t] <= 255 and np.all(Q[r, t, m[r, t]:] == -1)
            mse, _, _ = O.eval_raw(X[r], P[r][code])
            J = mse + lam[r, t] * O.eval_raw_ib(X[r], P[r][code])
            assert J <= ref["J"][r, t] * (1 + 1e-5) + 1e-300


def test_encode_with_a_256_value_code(E, O):
    X = W.random_case(83, 2, 30000, "normal")
    P, _ = O.grid_batch(X, 512)
    s = 256
    Q1 = np.stack([np.unique(np.concatenate([[0, 511], np.sort(np.random.default_rng(r).choice(
        np.arange(1, 511), 254, replace=False))])) for r in range(2)]).astype(np.int32)
    assert Q1.shape == (2, 256)
    m1 = np.full(2, 256, np.int32)
    idx, hist, st = E.encode(_cu(X), _cu(P), s, _cu(Q1), _cu(m1), 5)
    io, ho, so = O.encode_batch(X, P, Q1, m1, s, 5)
    assert int(st.abs().sum()) == 0 and np.all(so == 0)
    np.testing.assert_array_equal(idx.cpu().numpy(), io)
    np.testing.assert_array_equal(hist.cpu().numpy(), ho)
    assert io.max() == 255


def test_sizes_out_of_range_are_rejected(E):
    L = E.load()
    dummy = C.c_void_p(16)  # never dereferenced: the checks fail first
    null = C.c_void_p(0)
    # d = 0, p = 513, s = 256, n = 0
    assert L.ecasq_uniform_grid(dummy, 1, 0, 8, dummy, dummy, dummy, 64, null) == -1
    assert L.ecasq_workspace_size(1, 100, 513, 8, 1, None) == 0
    assert L.ecasq_workspace_size(1, 100, 64, 256, 1, None) == 0
    assert L.ecasq_workspace_size(0, 100, 64, 8, 1, None) == 0
    assert L.ecasq_approx_workspace_size(1, 0, 64, 8, None) == 0
    assert L.ecasq_encode(dummy, dummy, 1, 100, 64, 257, dummy, dummy, null, null, null, 1, dummy, dummy, dummy,
                          null) == -1


def test_bucket_sums_do_not_overflow_on_long_rows(E, O):
    """One row of 2^27 + 5 entries with p = 2, every entry in the one bucket
    (the worst case for the 64-bit fixed-point sums): rows of 2^27 entries or
    more keep 32 fraction bits, so the sums stay below 2^63. Counts exact and
    moments to 1e-9 against the oracle's compensated sums."""
    d = (1 << 27) + 5
    rng = np.random.default_rng(61)
    X = rng.random((1, d), dtype=np.float32)
    X[0, 0], X[0, 1] = 0.0, 1.0
    Xd = torch.from_numpy(X).cuda()
    P, cnt, A, B, st = E.grid_bucket(Xd, 2)
    assert int(st.abs().sum()) == 0 and int(cnt[0, 0]) == d
    Po, _ = O.grid_batch(X, 2)
    np.testing.assert_array_equal(P.cpu().numpy(), Po)
    co, Ao, Bo, so = O.bucket(X[0], Po[0])
    assert so == 0 and int(co[0]) == d
    assert float(A[0, 0]) == pytest.approx(Ao[0], rel=1e-9)
    assert float(B[0, 0]) == pytest.approx(Bo[0], rel=1e-9)
