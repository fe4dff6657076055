"""GPU (sm_100a) approximation on H(I,B) and refinement vs the fp64 oracle,
through the C ABI ("Entropy-Constrained Adaptive Stochastic Quantization
(ECASQ)", gist.science/pt/paper/2608.18147, §2.3 and §2.4).

Two set-ups:
  * from the ORACLE's bucket statistics (the *_stats entry points), fp64 layers:
    the GPU sums each interval in the same order with every operation rounded as
    written, so its pair terms equal the oracle's tables and only the last bit of
    log2 can differ. Codes must be identical (refined codes too, since the
    refinement takes every decision on those values) and objectives agree to
    1e-12 relative;
  * from X (GPU bucketing), fp32 layers (the throughput path): the oracle's
    evaluation of the GPU's code is within 1e-5 of the oracle's optimum, and the
    GPU's own fp64 figures of that code match the oracle's evaluation to 1e-9.
"""
import numpy as np
import pytest
import torch

from entropy_constrained_unbiased_b200 import workloads as W

pytestmark = pytest.mark.gpu

RTOL_EXACT = 1e-12
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


def _oracle_stats(O, X, P):
    n, p = P.shape
    cnt = np.zeros((n, p - 1), np.int64)
    A = np.zeros((n, p - 1))
    B = np.zeros((n, p - 1))
    for r in range(n):
        cnt[r], A[r], B[r], st = O.bucket(X[r], P[r])
        assert st == 0
    return _cu(cnt), _cu(A), _cu(B)


def _lams(X, k):
    v = np.var(X.astype(np.float64), axis=1)
    base = np.array([0.0, 1e-3, 1e-2, 5e-2, 0.2, 1.0])[:k]
    return v[:, None] * base[None, :]


CASES = [  # (seed, n, d, p, s, dist)
    (0, 3, 400, 16, 4, "normal"),
    (1, 3, 1000, 40, 6, "laplace"),
    (2, 2, 2000, 64, 8, "student_t"),
    (3, 2, 1500, 70, 9, "lognormal"),
    (4, 2, 3000, 128, 16, "outlier"),
    (5, 2, 800, 97, 12, "grad"),
    (6, 2, 600, 24, 24, "normal"),      # s == p
    (7, 2, 600, 10, 30, "laplace"),     # s > p
    (8, 2, 500, 30, 3, "normal"),
    (9, 2, 500, 30, 2, "normal"),       # s = 2: Q = {min, max}
    (10, 1, 6000, 300, 12, "normal"),   # p > 256: 512 threads
]


def _setup(O, seed, n, d, p, dist):
    X = W.random_case(seed, n, d, dist)
    P, st = O.grid_batch(X, p)
    assert np.all(st == 0)
    return X, P


@pytest.mark.parametrize("refine", [0, 8])
@pytest.mark.parametrize("case", CASES, ids=lambda c: f"p{c[3]}s{c[4]}{c[5]}")
def test_approx_fp64_matches_oracle_from_its_statistics(E, O, case, refine):
    seed, n, d, p, s, dist = case
    X, P = _setup(O, seed, n, d, p, dist)
    lam = _lams(X, 6)
    cnt, A, B = _oracle_stats(O, X, P)
    g = E.solve_approx_stats(cnt, A, B, _cu(P), d, s, _cu(lam), refine=refine, fp64=True)
    ref = O.solve_approx_batch(X, P, s, lam, refine=refine)
    assert int(g["status"].abs().sum()) == 0
    Q, m = g["Q"].cpu().numpy(), g["Q_len"].cpu().numpy()
    np.testing.assert_array_equal(m, ref["m"])
    np.testing.assert_array_equal(Q, ref["Q"])
    for k_g, k_o in (("objective", "J"), ("mse", "mse"), ("H", "H"), ("H_IB", "HIB")):
        np.testing.assert_allclose(g[k_g].cpu().numpy(), ref[k_o], rtol=RTOL_EXACT, atol=1e-300)


# More vectors than SMs: the launch runs one thread per column (the small cases
# above, with fewer vectors than SMs, share each column between two threads).
MANY = (21, 300, 300, 40, 6, "laplace")


@pytest.mark.parametrize("refine", [0, 8])
def test_approx_many_rows_fp64_matches_oracle_from_its_statistics(E, O, refine):
    seed, n, d, p, s, dist = MANY
    X, P = _setup(O, seed, n, d, p, dist)
    lam = _lams(X, 3)
    cnt, A, B = _oracle_stats(O, X, P)
    g = E.solve_approx_stats(cnt, A, B, _cu(P), d, s, _cu(lam), refine=refine, fp64=True)
    ref = O.solve_approx_batch(X, P, s, lam, refine=refine)
    assert int(g["status"].abs().sum()) == 0
    np.testing.assert_array_equal(g["Q_len"].cpu().numpy(), ref["m"])
    np.testing.assert_array_equal(g["Q"].cpu().numpy(), ref["Q"])
    np.testing.assert_allclose(g["objective"].cpu().numpy(), ref["J"], rtol=RTOL_EXACT, atol=1e-300)


def test_approx_many_rows_fp32_from_X_reaches_the_oracle_optimum(E, O):
    seed, n, d, p, s, dist = MANY
    X, P = _setup(O, seed, n, d, p, dist)
    lam = _lams(X, 3)
    g = E.solve_approx(_cu(X), _cu(P), s, _cu(lam))
    ref = O.solve_approx_batch(X, P, s, lam)
    assert int(g["status"].abs().sum()) == 0
    Q, m = g["Q"].cpu().numpy(), g["Q_len"].cpu().numpy()
    for r in range(n):
        for t in range(lam.shape[1]):
            q = Q[r, t, : m[r, t]]
            J = O.eval_raw(X[r], P[r][q])[0] + lam[r, t] * O.eval_raw_ib(X[r], P[r][q])
            assert J <= ref["J"][r, t] * (1 + RTOL32) + 1e-300, (r, t, J, ref["J"][r, t])


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"p{c[3]}s{c[4]}{c[5]}")
def test_approx_fp32_from_X_reaches_the_oracle_optimum(E, O, case):
    seed, n, d, p, s, dist = case
    X, P = _setup(O, seed, n, d, p, dist)
    lam = _lams(X, 6)
    g = E.solve_approx(_cu(X), _cu(P), s, _cu(lam))
    ref = O.solve_approx_batch(X, P, s, lam)
    assert int(g["status"].abs().sum()) == 0
    Q, m = g["Q"].cpu().numpy(), g["Q_len"].cpu().numpy()
    for r in range(n):
        for t in range(lam.shape[1]):
            q = Q[r, t, : m[r, t]]
            assert q[0] == 0 and q[-1] == p - 1 and np.all(np.diff(q) > 0) and 2 <= m[r, t] <= min(s, p)
            assert np.all(Q[r, t, m[r, t]:] == -1)
            mse, H, _ = O.eval_raw(X[r], P[r][q])
            hib = O.eval_raw_ib(X[r], P[r][q])
            J = mse + lam[r, t] * hib
            assert J <= ref["J"][r, t] * (1 + RTOL32) + 1e-300, (r, t, J, ref["J"][r, t])
            assert g["mse"][r, t].item() == pytest.approx(mse, rel=RTOL64, abs=1e-300)
            assert g["H"][r, t].item() == pytest.approx(H, rel=RTOL64, abs=1e-15)
            assert g["H_IB"][r, t].item() == pytest.approx(hib, rel=RTOL64, abs=1e-15)
            assert g["objective"][r, t].item() == pytest.approx(J, rel=RTOL64, abs=1e-300)


@pytest.mark.parametrize("refine", [0, 8])
@pytest.mark.parametrize("case", CASES[:6], ids=lambda c: f"p{c[3]}s{c[4]}{c[5]}")
def test_approx_refined_from_X_never_worse_than_the_approximation(E, O, case, refine):
    """From X (GPU bucketing) in fp64: the refined code has exact J no larger
    than the unrefined one's and no smaller than the exact optimum."""
    seed, n, d, p, s, dist = case
    X, P = _setup(O, seed, n, d, p, dist)
    lam = _lams(X, 6)
    a = E.solve_approx(_cu(X), _cu(P), s, _cu(lam), refine=0, fp64=True)
    r_ = E.solve_approx(_cu(X), _cu(P), s, _cu(lam), refine=8, fp64=True)
    ex = O.solve_batch(X, P, s, lam)
    for r in range(n):
        for t in range(lam.shape[1]):
            Ja = a["mse"][r, t].item() + lam[r, t] * a["H"][r, t].item()
            Jr = r_["objective"][r, t].item()
            assert Jr <= Ja * (1 + 1e-12) + 1e-300
            assert Jr >= ex["J"][r, t] * (1 - RTOL64)
            assert r_["Q_len"][r, t].item() == a["Q_len"][r, t].item()


@pytest.mark.parametrize("refine", [0, 8])
@pytest.mark.parametrize("case", [CASES[2], CASES[4], CASES[5]], ids=lambda c: f"p{c[3]}s{c[4]}{c[5]}")
def test_approx_budget_fp64_matches_oracle_from_its_statistics(E, O, case, refine):
    seed, n, d, p, s, dist = case
    X, P = _setup(O, seed, n, d, p, dist)
    cnt, A, B = _oracle_stats(O, X, P)
    for b in (1.5, 2.5):
        g = E.solve_approx_budget_stats(cnt, A, B, _cu(P), d, s, b, refine=refine, fp64=True)
        ref = O.solve_approx_budget_batch(X, P, s, b, 30, refine=refine)
        gn = {k: v.cpu().numpy() for k, v in g.items()}
        np.testing.assert_array_equal(gn["status"], ref["status"])
        np.testing.assert_array_equal(gn["Q1"], ref["Q1"])
        np.testing.assert_array_equal(gn["Q2"], ref["Q2"])
        np.testing.assert_array_equal(gn["lambda_lo"], ref["lam_lo"])
        np.testing.assert_array_equal(gn["lambda_hi"], ref["lam_hi"])
        for k_g, k_o in (("theta", "theta"), ("H1", "H1"), ("H2", "H2"), ("H_IB1", "HIB1"), ("H_IB2", "HIB2"),
                         ("mse1", "mse1"), ("mse2", "mse2")):
            np.testing.assert_allclose(gn[k_g], ref[k_o], rtol=RTOL_EXACT, atol=1e-15)


@pytest.mark.parametrize("refine", [0, 8])
def test_approx_budget_fp32_from_X(E, O, refine):
    X, P = _setup(O, 11, 4, 4000, 128, "student_t")
    b = 3.0
    g = E.solve_approx_budget(_cu(X), _cu(P), 16, b, refine=refine)
    ref = O.solve_approx_budget_batch(X, P, 16, b, 30, refine=refine)
    gn = {k: v.cpu().numpy() for k, v in g.items()}
    assert np.all(gn["status"] == 0)
    rate = "H" if refine else "H_IB"
    for r in range(X.shape[0]):
        th = gn["theta"][r]
        if 0 < th < 1:
            assert th * gn[rate + "1"][r] + (1 - th) * gn[rate + "2"][r] == pytest.approx(b, rel=1e-12)
        d_gpu = th * gn["mse1"][r] + (1 - th) * gn["mse2"][r]
        d_ref = ref["theta"][r] * ref["mse1"][r] + (1 - ref["theta"][r]) * ref["mse2"][r]
        assert d_gpu == pytest.approx(d_ref, rel=RTOL32)
        assert gn[rate + "2"][r] <= b + 1e-15


def test_approx_degenerate_and_invalid_rows(E, O):
    X = W.random_case(12, 3, 500, "normal")
    X[1] = 0.25  # constant row
    P, _ = O.grid_batch(X, 32)
    P[2, 5] = P[2, 4]  # not strictly increasing
    g = E.solve_approx(_cu(X[:2]), _cu(P[:2]), 6, _cu(_lams(X[:2], 2)))
    assert list(g["status"].cpu().numpy()) == [0, 0]
    assert g["Q_len"][1, 0].item() == 1 and g["Q"][1, 0, 0].item() == 0 and g["objective"][1, 0].item() == 0.0
    cnt, A, B = _oracle_stats(O, X[:2], P[:2])
    Pb = P.copy()
    cnt3 = torch.cat([cnt, cnt[:1]])
    A3 = torch.cat([A, A[:1]])
    B3 = torch.cat([B, B[:1]])
    g = E.solve_approx_stats(cnt3, A3, B3, _cu(Pb), 500, 6, _cu(_lams(X, 1)))
    st = g["status"].cpu().numpy()
    assert st[0] == 0 and st[2] == -1
    assert g["Q_len"][2, 0].item() == 0 and np.all(g["Q"][2, 0].cpu().numpy() == -1)


def test_approx_out_of_range_entries_are_flagged(E, O):
    X = W.random_case(13, 2, 300, "normal")
    P, _ = O.grid_batch(X, 16)
    X2 = X.copy()
    X2[1, 3] = P[1, -1] + 1.0
    g = E.solve_approx(_cu(X2), _cu(P), 5, _cu(_lams(X, 1)))
    assert list(g["status"].cpu().numpy()) == [0, -2]


@pytest.mark.parametrize("fp64", [False, True])
def test_approx_p512_global_tables(E, O, fp64):
    """p = 512, s = 32: cost table and layers in the global slab."""
    X, P = _setup(O, 14, 1, 20000, 512, "normal")
    lam = _lams(X, 3)[:, 1:]
    g = E.solve_approx(_cu(X), _cu(P), 32, _cu(lam), fp64=fp64)
    ref = O.solve_approx_batch(X, P, 32, lam)
    tol = RTOL64 if fp64 else RTOL32
    for t in range(lam.shape[1]):
        q = g["Q"][0, t, : g["Q_len"][0, t]].cpu().numpy()
        mse, _, _ = O.eval_raw(X[0], P[0][q])
        J = mse + lam[0, t] * O.eval_raw_ib(X[0], P[0][q])
        assert J <= ref["J"][0, t] * (1 + tol)
