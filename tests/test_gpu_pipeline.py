"""quantize(): one call from X to indices equals the C ABI calls it composes,
for the budget and fixed-lambda solvers, exact and approximate, on the uniform
grid and on a given alphabet; the time-shared indices are bit-exact against
the oracle's encoder."""
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


def _eq(a, b):
    assert torch.equal(a, b)


@pytest.mark.parametrize("solver", ["exact", "approx"])
def test_quantize_budget_matches_the_calls(E, O, solver):
    from entropy_constrained_unbiased_b200.pipeline import quantize
    X = W.random_case(91, 5, 3001, "student_t")
    Xd = torch.from_numpy(X).cuda()
    p, s, b, seed = 64, 8, 2.0, 1234
    q = quantize(Xd, p, s, b=b, seed=seed, solver=solver)
    P, cnt, A, B, _ = E.grid_bucket(Xd, p)
    if solver == "exact":
        g = E.solve_budget_stats(cnt, A, B, P, X.shape[1], s, b)
    else:
        g = E.solve_approx_budget_stats(cnt, A, B, P, X.shape[1], s, b)
    for k in ("Q1", "Q1_len", "Q2", "Q2_len", "theta"):
        _eq(getattr(q, k), g[k])
    _eq(q.P, P)
    idx, hist, _ = E.encode(Xd, P, s, g["Q1"], g["Q1_len"], seed, g["Q2"], g["Q2_len"], g["theta"])
    _eq(q.idx, idx)
    _eq(q.hist, hist)
    _eq(q.H_emp, E.entropy(hist))
    assert set(q.stats) >= {"status", "mse1", "mse2", "H1", "H2"}
    Xh, _ = E.dequantize(idx, P, s, g["Q1"], g["Q1_len"], seed, g["Q2"], g["Q2_len"], g["theta"])
    _eq(q.dequantize(), Xh)
    # the time-shared indices against the oracle's encoder
    Pn, gn = P.cpu().numpy(), {k: v.cpu().numpy() for k, v in g.items()}
    io, ho, so = O.encode_batch(X, Pn, gn["Q1"], gn["Q1_len"], s, seed, gn["Q2"], gn["Q2_len"], gn["theta"])
    assert np.all(so == 0)
    np.testing.assert_array_equal(q.idx.cpu().numpy(), io)
    np.testing.assert_array_equal(q.hist.cpu().numpy(), ho)


def test_quantize_lambda_and_given_alphabet(E):
    from entropy_constrained_unbiased_b200.pipeline import quantize
    X = W.random_case(92, 3, 2000, "laplace")
    Xd = torch.from_numpy(X).cuda()
    p, s, lam = 48, 6, 0.02
    P, _ = E.uniform_grid(Xd, p)
    q = quantize(Xd, p, s, lam=lam, seed=5, P=P, hirschberg=True)
    g = E.solve(Xd, P, s, torch.full((3, 1), lam, dtype=torch.float64, device="cuda"), hirschberg=True)
    _eq(q.Q1, g["Q"][:, 0, :])
    _eq(q.Q1_len, g["Q_len"][:, 0])
    assert q.Q2 is None and q.theta is None
    idx, hist, _ = E.encode(Xd, P, s, q.Q1, q.Q1_len, 5)
    _eq(q.idx, idx)
    assert torch.allclose(q.stats["objective"], g["objective"], rtol=0, atol=0)


def test_quantize_rejects_bad_arguments(E):
    from entropy_constrained_unbiased_b200.pipeline import quantize
    Xd = torch.from_numpy(W.random_case(93, 2, 100)).cuda()
    with pytest.raises(E.EcasqError):
        quantize(Xd, 16, 4)  # neither b nor lam
    with pytest.raises(E.EcasqError):
        quantize(Xd, 16, 4, b=1.0, lam=0.1)
    with pytest.raises(E.EcasqError):
        quantize(Xd, 16, 4, b=1.0, solver="other")
    with pytest.raises(E.EcasqError):
        quantize(Xd, 16, 4, b=1.0, P=torch.zeros(2, 8, dtype=torch.float64, device="cuda"))
