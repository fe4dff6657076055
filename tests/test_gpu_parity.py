"""GPU (sm_100a) vs the fp64 oracle, element by element, through the C ABI.

Tolerances (objective J = MSE + lambda * H):
  * fp64 DP: |J_gpu - J_oracle| <= 1e-9 |J_oracle|, and the oracle's own
    evaluation of the GPU's code is within the same bound of the optimum;
  * fp32 DP: the oracle's evaluation of the GPU's code is within 1e-5 of the
    optimum (the code is re-evaluated in fp64, so mse/H of that code agree
    with the oracle's evaluation to 1e-9);
  * grid, bucket counts, encoded indices and histograms: bit-exact;
  * bucket moments, entropies: 1e-9 relative.
Ties between codes are judged by objective value.
"""
import math

import numpy as np
import pytest
import torch

from entropy_constrained_unbiased_b200 import workloads as W

pytestmark = pytest.mark.gpu

RTOL64 = 1e-9
RTOL32 = 1e-5


@pytest.fixture(scope="module")
def E():
    from entropy_constrained_unbiased_b200 import build, ecasq
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    ecasq.load()
    return ecasq


def _cu(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _np(t):
    return t.cpu().numpy()


def _case(seed, n, d, dist):
    return W.random_case(seed, n, d, dist)


def _oracle_eval(O, x, P, Q, m, lam):
    mse, H, _ = O.eval_raw(x, P[Q[:m]])
    return mse + lam * H, mse, H


# -- grid and buckets ------------------------------------------------------------

@pytest.mark.parametrize("dist,d,p", [("normal", 1024, 64), ("student_t", 4099, 128), ("grad", 70001, 256),
                                      ("lognormal", 3, 2), ("laplace", 1, 16)])
def test_grid_bit_exact(E, O, dist, d, p):
    X = _case(1, 5, d, dist)
    P, st = E.uniform_grid(_cu(X), p)
    Po, sto = O.grid_batch(X, p)
    assert np.all(_np(st) == 0) and np.all(sto == 0)
    np.testing.assert_array_equal(_np(P), Po)


def test_grid_flags_nonfinite(E, O):
    X = _case(2, 3, 257, "normal")
    X[1, 100] = np.nan
    X[2, 7] = np.inf
    _, st = E.uniform_grid(_cu(X), 16)
    assert list(_np(st)) == [0, -2, -2]


@pytest.mark.parametrize("dist,d,p,uniform", [("normal", 1024, 64, True), ("student_t", 4097, 128, True),
                                              ("grad", 100003, 256, True), ("outlier", 5000, 512, True),
                                              ("laplace", 777, 33, False)])
def test_bucket_statistics(E, O, dist, d, p, uniform):
    X = _case(3, 4, d, dist)
    if uniform:
        P, _ = O.grid_batch(X, p)
    else:
        rng = np.random.default_rng(5)
        P = np.stack([np.concatenate([[x.min()], np.sort(rng.uniform(x.min(), x.max(), p - 2)), [x.max()]])
                      for x in X.astype(np.float64)])
    cnt, A, B, st = E.bucket(_cu(X), _cu(P))
    assert np.all(_np(st) == 0)
    for r in range(X.shape[0]):
        co, Ao, Bo, so = O.bucket(X[r], P[r])
        assert so == 0
        np.testing.assert_array_equal(_np(cnt[r]), co)
        np.testing.assert_allclose(_np(A[r]), Ao, rtol=1e-9, atol=1e-12 * (P[r, -1] - P[r, 0]))
        np.testing.assert_allclose(_np(B[r]), Bo, rtol=1e-9, atol=1e-12 * (P[r, -1] - P[r, 0]) ** 2)


def test_bucket_flags_out_of_range(E, O):
    X = _case(4, 2, 300, "normal")
    P, _ = O.grid_batch(X, 16)
    X2 = X.copy()
    X2[1, 5] = P[1, -1] + 1.0
    _, _, _, st = E.bucket(_cu(X2), _cu(P))
    assert list(_np(st)) == [0, -2]


# -- grid and bucketing in one call ------------------------------------------------

GRID_BUCKET_CASES = [  # (dist, n, d, p): one-read path (aligned, d <= 16384, p <= 129), its unaligned
    ("normal", 5, 1024, 64),  # fallback (odd d), and the two-pass path (larger d or p)
    ("student_t", 7, 4096, 128),
    ("laplace", 3, 16384, 129),
    ("grad", 4, 4099, 128),
    ("outlier", 3, 777, 33),
    ("lognormal", 2, 3, 2),
    ("normal", 2, 1, 16),
    ("grad", 3, 20000, 128),
    ("mixture", 3, 5000, 256),
    ("laplace", 2, 70001, 257),   # long rows: the persistent bucketing kernel
    ("normal", 2, 9000, 1000),    # beyond 512 values: bucketing by bisection
]


def _check_grid_bucket(O, X, P, cnt, A, B, st, p):
    Po, sto = O.grid_batch(X, p)
    assert np.all(sto == 0) and np.all(_np(st) == 0)
    np.testing.assert_array_equal(_np(P), Po)
    for r in range(X.shape[0]):
        co, Ao, Bo, so = O.bucket(X[r], Po[r])
        assert so == 0
        np.testing.assert_array_equal(_np(cnt[r]), co)
        span = Po[r, -1] - Po[r, 0]
        np.testing.assert_allclose(_np(A[r]), Ao, rtol=1e-9, atol=1e-12 * span)
        np.testing.assert_allclose(_np(B[r]), Bo, rtol=1e-9, atol=1e-12 * span ** 2)


@pytest.mark.parametrize("dist,n,d,p", GRID_BUCKET_CASES)
def test_grid_bucket_matches_oracle(E, O, dist, n, d, p):
    X = _case(13, n, d, dist)
    P, cnt, A, B, st = E.grid_bucket(_cu(X), p)
    _check_grid_bucket(O, X, P, cnt, A, B, st, p)
    # the same statistics as the two separate calls
    P2, _ = E.uniform_grid(_cu(X), p)
    c2, A2, B2, _ = E.bucket(_cu(X), P2)
    assert torch.equal(P, P2) and torch.equal(cnt, c2)
    np.testing.assert_allclose(_np(A), _np(A2), rtol=1e-12, atol=1e-15 * float((P2[:, -1] - P2[:, 0]).max()))


def test_grid_bucket_unaligned_rows(E, O):
    """Rows whose start is not 16-byte aligned (d a multiple of 4, the base
    pointer 4 bytes past an aligned one): the staging falls back to plain loads."""
    X = _case(14, 6, 4096, "student_t")
    flat = torch.empty(X.size + 1, dtype=torch.float32, device="cuda")
    Xd = flat[1:].view(X.shape)
    Xd.copy_(torch.from_numpy(X))
    assert Xd.data_ptr() % 16 != 0
    P, cnt, A, B, st = E.grid_bucket(Xd, 128)
    _check_grid_bucket(O, X, P, cnt, A, B, st, 128)


def test_grid_bucket_flags_and_constant_rows(E, O):
    X = _case(15, 4, 4096, "normal")
    X[1, 100] = np.nan
    X[2, :] = 0.5
    X[3, 7] = np.inf
    P, cnt, A, B, st = E.grid_bucket(_cu(X), 64)
    assert list(_np(st)) == [0, -2, 0, -2]
    Pn = _np(P)
    assert np.all(np.isnan(Pn[1])) and np.all(np.isnan(Pn[3]))
    for r in (0, 2):
        Po, _ = O.uniform_grid(X[r], 64)
        np.testing.assert_array_equal(Pn[r], Po)
        co, Ao, Bo, _ = O.bucket(X[r], Po)
        np.testing.assert_array_equal(_np(cnt[r]), co)
        np.testing.assert_allclose(_np(A[r]), Ao, rtol=1e-9, atol=1e-12 * max(Po[-1] - Po[0], 1e-30))
    assert int(_np(cnt[2])[-1]) == 4096 and float(_np(A[2]).max()) == 0.0


# -- the DP ------------------------------------------------------------------------

SMALL = [  # (seed, n, d, p, s, dist)
    (0, 3, 400, 16, 4, "normal"),
    (1, 3, 1000, 40, 6, "laplace"),
    (2, 2, 2000, 64, 8, "student_t"),
    (3, 2, 1500, 70, 9, "lognormal"),
    (4, 2, 3000, 128, 16, "outlier"),
    (5, 2, 800, 97, 12, "grad"),
    (6, 2, 600, 24, 24, "normal"),      # s == p
    (7, 2, 600, 10, 30, "laplace"),     # s > p
    (8, 2, 500, 30, 3, "normal"),       # s = 3: layer 2 is the last
    (9, 2, 500, 30, 2, "normal"),       # s = 2: Q = {min, max}
    (10, 1, 5000, 200, 10, "normal"),   # pair tables outside shared memory
]


def _lams(X, k):
    v = float(np.var(X.astype(np.float64)))
    return np.array([[0.0, 1e-3 * v, 0.05 * v, v][: k]] * X.shape[0])


@pytest.mark.parametrize("fp64", [True, False], ids=["fp64", "fp32"])
@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"p{c[3]}s{c[4]}{c[5]}")
def test_solve_matches_oracle(E, O, case, fp64):
    seed, n, d, p, s, dist = case
    X = _case(seed, n, d, dist)
    P, _ = O.grid_batch(X, p)
    lam = _lams(X, 4)
    g = E.solve(_cu(X), _cu(P), s, _cu(lam), fp64=fp64)
    ref = O.solve_batch(X, P, s, lam)
    assert np.all(_np(g["status"]) == 0)
    Qg, mg, Jg = _np(g["Q"]), _np(g["Q_len"]), _np(g["objective"])
    msg, Hg = _np(g["mse"]), _np(g["H"])
    tol = RTOL64 if fp64 else RTOL32
    for r in range(n):
        for t in range(lam.shape[1]):
            m = mg[r, t]
            Q = Qg[r, t]
            assert 2 <= m <= min(s, p)
            assert Q[0] == 0 and Q[m - 1] == p - 1 and np.all(np.diff(Q[:m]) > 0) and np.all(Q[m:] == -1)
            Jo = ref["J"][r, t]
            Jeval, mse_e, H_e = _oracle_eval(O, X[r], P[r], Q, m, lam[r, t])
            assert Jeval <= Jo * (1 + tol) + 1e-300, (r, t, Jeval, Jo)
            assert Jeval >= Jo * (1 - 1e-12)
            # the GPU's fp64 evaluation of its own code
            assert msg[r, t] == pytest.approx(mse_e, rel=RTOL64, abs=1e-300)
            assert Hg[r, t] == pytest.approx(H_e, rel=RTOL64, abs=1e-12)
            assert Jg[r, t] == pytest.approx(Jeval, rel=RTOL64)
            if fp64:
                assert Jg[r, t] == pytest.approx(Jo, rel=RTOL64)


@pytest.mark.parametrize("fp64", [True, False], ids=["fp64", "fp32"])
def test_solve_nonuniform_alphabet(E, O, fp64):
    rng = np.random.default_rng(9)
    X = _case(11, 3, 1200, "laplace")
    p = 50
    P = np.stack([np.concatenate([[x.min()], np.sort(rng.uniform(x.min(), x.max(), p - 2)), [x.max()]])
                  for x in X.astype(np.float64)])
    lam = _lams(X, 3)
    g = E.solve(_cu(X), _cu(P), 7, _cu(lam), fp64=fp64)
    ref = O.solve_batch(X, P, 7, lam)
    tol = RTOL64 if fp64 else RTOL32
    for r in range(3):
        for t in range(3):
            m = int(_np(g["Q_len"])[r, t])
            Jeval, _, _ = _oracle_eval(O, X[r], P[r], _np(g["Q"])[r, t], m, lam[r, t])
            assert Jeval <= ref["J"][r, t] * (1 + tol)


def test_solve_degenerate_and_invalid_rows(E, O):
    X = _case(12, 3, 256, "normal")
    X[1, :] = 0.75                 # constant row
    P, _ = O.grid_batch(X, 16)
    P[2, 5] = P[2, 4]              # not strictly increasing
    g = E.solve(_cu(X), _cu(P), 5, 0.01)
    st = _np(g["status"])
    assert st[0] == 0 and st[1] == 0 and st[2] == -1
    assert _np(g["Q_len"])[1, 0] == 1 and _np(g["Q"])[1, 0, 0] == 0 and _np(g["objective"])[1, 0] == 0.0


def test_solve_stats_equals_solve(E, O):
    X = _case(13, 2, 3000, "student_t")
    P, _ = O.grid_batch(X, 64)
    Xc, Pc = _cu(X), _cu(P)
    cnt, A, B, _ = E.bucket(Xc, Pc)
    a = E.solve(Xc, Pc, 8, 0.001, fp64=True)
    b = E.solve_stats(cnt, A, B, Pc, X.shape[1], 8, 0.001, fp64=True)
    for k in ("Q", "Q_len", "objective", "mse", "H"):
        assert torch.equal(a[k], b[k]), k


# -- entropy budget ---------------------------------------------------------------

@pytest.mark.parametrize("fp64", [True, False], ids=["fp64", "fp32"])
@pytest.mark.parametrize("case", [(20, 3, 3000, 64, 10, "student_t", 2.5), (21, 2, 5000, 128, 16, "grad", 2.0),
                                  (22, 2, 2000, 48, 8, "normal", 1.2), (23, 2, 1000, 32, 6, "laplace", 9.0),
                                  (24, 2, 1000, 32, 6, "laplace", 0.05)])
def test_budget_matches_oracle(E, O, case, fp64):
    seed, n, d, p, s, dist, b = case
    X = _case(seed, n, d, dist)
    P, _ = O.grid_batch(X, p)
    g = {k: _np(v) for k, v in E.solve_budget(_cu(X), _cu(P), s, b, 30, fp64=fp64).items()}
    ref = O.solve_budget_batch(X, P, s, b, 30)
    tol = RTOL64 if fp64 else RTOL32
    for r in range(n):
        assert g["status"][r] == ref["status"][r]
        th = g["theta"][r]
        assert g["H2"][r] <= b + 1e-12 or g["status"][r] == 1
        if 0 < th < 1:
            assert g["H1"][r] > b
            assert th * g["H1"][r] + (1 - th) * g["H2"][r] == pytest.approx(b, rel=1e-12)
        # both codes are Lagrangian optima (oracle) at the GPU's lambdas
        for qk, mk, lk in (("Q1", "Q1_len", "lambda_lo"), ("Q2", "Q2_len", "lambda_hi")):
            m = g[mk][r]
            lam = g[lk][r]
            Jeval, mse_e, H_e = _oracle_eval(O, X[r], P[r], g[qk][r], m, lam)
            Jopt = O.solve_batch(X[r:r + 1], P[r:r + 1], s, np.array([[lam]]))["J"][0, 0]
            assert Jeval <= Jopt * (1 + tol) + 1e-300
        # the time-shared distortion-rate point matches the oracle's
        d_gpu = th * g["mse1"][r] + (1 - th) * g["mse2"][r]
        d_ref = ref["theta"][r] * ref["mse1"][r] + (1 - ref["theta"][r]) * ref["mse2"][r]
        assert d_gpu == pytest.approx(d_ref, rel=tol)
        if fp64:
            for k_g, k_o in (("theta", "theta"), ("H1", "H1"), ("H2", "H2"), ("mse1", "mse1"), ("mse2", "mse2"),
                             ("lambda_lo", "lam_lo"), ("lambda_hi", "lam_hi")):
                assert g[k_g][r] == pytest.approx(ref[k_o][r], rel=RTOL64, abs=1e-15), k_g


# -- encoder -------------------------------------------------------------------------

@pytest.mark.parametrize("d", [1, 3, 1024, 4099, 40000, 140003])  # 140003: three encoder chunks, ragged
def test_encode_bit_exact_single_code(E, O, d):
    X = _case(30, 3, d, "laplace")
    P, _ = O.grid_batch(X, 32)
    ref = O.solve_batch(X, P, 6, np.full((3, 1), 0.01))
    Q = np.ascontiguousarray(ref["Q"][:, 0, :])
    m = np.ascontiguousarray(ref["m"][:, 0])
    idx, hist, st = E.encode(_cu(X), _cu(P), 6, _cu(Q), _cu(m), seed=1)
    io, ho, so = O.encode_batch(X, P, Q, m, 6, 1)
    assert np.all(_np(st) == 0) and np.all(so == 0)
    np.testing.assert_array_equal(_np(idx), io)
    np.testing.assert_array_equal(_np(hist), ho)
    H = _np(E.entropy(hist))
    for r in range(3):
        assert H[r] == pytest.approx(O.entropy(ho[r], 6), rel=1e-12, abs=1e-15)


@pytest.mark.parametrize("seed,d", [(1, 20001), (2**40 + 12345, 20001), (5, 131077)])
def test_encode_bit_exact_time_shared(E, O, seed, d):
    X = _case(31, 4, d, "student_t")
    P, _ = O.grid_batch(X, 64)
    ref = O.solve_budget_batch(X, P, 10, 2.3, 30)
    args = [ref["Q1"], ref["m1"], ref["Q2"], ref["m2"], ref["theta"]]
    idx, hist, st = E.encode(_cu(X), _cu(P), 10, _cu(args[0]), _cu(args[1]), seed, _cu(args[2]), _cu(args[3]),
                             _cu(args[4]))
    io, ho, so = O.encode_batch(X, P, args[0], args[1], 10, seed, args[2], args[3], args[4])
    np.testing.assert_array_equal(_np(idx), io)
    np.testing.assert_array_equal(_np(hist), ho)
    assert np.all(_np(st) == 0)


def test_encode_flags_out_of_range(E, O):
    X = _case(32, 2, 100, "normal")
    P, _ = O.grid_batch(X, 16)
    Q = np.array([[0, 3, 15, -1], [0, 5, 12, -1]], np.int32)  # row 1 ends below max X
    m = np.array([3, 3], np.int32)
    _, _, st = E.encode(_cu(X), _cu(P), 4, _cu(Q), _cu(m), seed=3)
    assert list(_np(st)) == [0, -2]


# -- Hirschberg mode (O(p^2) DP memory, no back-pointers) ---------------------------

HIRSCH = [  # (seed, n, d, p, s, dist)
    (40, 2, 1500, 48, 9, "laplace"),
    (41, 2, 3000, 96, 12, "mixture"),
    (42, 1, 2000, 200, 16, "normal"),
    (43, 2, 800, 30, 30, "student_t"),  # s == p
    (44, 2, 600, 20, 3, "normal"),      # one value between the ends
    (45, 2, 600, 20, 4, "normal"),
    (46, 1, 4000, 300, 20, "outlier"),
]


@pytest.mark.parametrize("fp64", [True, False], ids=["fp64", "fp32"])
@pytest.mark.parametrize("case", HIRSCH, ids=lambda c: f"p{c[3]}s{c[4]}{c[5]}")
def test_hirschberg_matches_store_mode_and_oracle(E, O, case, fp64):
    seed, n, d, p, s, dist = case
    X = _case(seed, n, d, dist)
    P, _ = O.grid_batch(X, p)
    lam = _lams(X, 4)
    h = {k: _np(v) for k, v in E.solve(_cu(X), _cu(P), s, _cu(lam), fp64=fp64, hirschberg=True).items()}
    st = {k: _np(v) for k, v in E.solve(_cu(X), _cu(P), s, _cu(lam), fp64=fp64).items()}
    ref = O.solve_batch(X, P, s, lam)
    tol = RTOL64 if fp64 else RTOL32
    assert np.all(h["status"] == 0)
    for r in range(n):
        for t in range(lam.shape[1]):
            m = h["Q_len"][r, t]
            Q = h["Q"][r, t]
            assert 2 <= m <= min(s, p)
            assert Q[0] == 0 and Q[m - 1] == p - 1 and np.all(np.diff(Q[:m]) > 0) and np.all(Q[m:] == -1)
            Jeval, _, _ = _oracle_eval(O, X[r], P[r], Q, m, lam[r, t])
            assert Jeval <= ref["J"][r, t] * (1 + tol) + 1e-300, (r, t, Jeval, ref["J"][r, t])
            assert h["objective"][r, t] == pytest.approx(Jeval, rel=RTOL64)
            assert h["objective"][r, t] == pytest.approx(st["objective"][r, t], rel=tol)
            if fp64:
                assert h["objective"][r, t] == pytest.approx(ref["J"][r, t], rel=RTOL64)


def test_hirschberg_budget(E, O):
    X = _case(47, 2, 4000, "student_t")
    P, _ = O.grid_batch(X, 64)
    g = {k: _np(v) for k, v in E.solve_budget(_cu(X), _cu(P), 10, 2.5, 30, fp64=True, hirschberg=True).items()}
    ref = O.solve_budget_batch(X, P, 10, 2.5, 30)
    for r in range(2):
        for k_g, k_o in (("theta", "theta"), ("H1", "H1"), ("H2", "H2"), ("mse1", "mse1"), ("mse2", "mse2")):
            assert g[k_g][r] == pytest.approx(ref[k_o][r], rel=RTOL64, abs=1e-15), k_g
