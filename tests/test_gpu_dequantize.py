"""Reconstruction X^ from the emitted indices on the GPU: bit-exact against the
oracle's (one code, two time-shared codes, unaligned and ragged rows, a large
alphabet), the mean over seeds of a full-size row equal to X within the
rounding's binomial error (E[X^] = X, "Entropy-Constrained Adaptive
Stochastic Quantization (ECASQ)", gist.science/pt/paper/2608.18147, §1), and
an index outside its code flagged."""
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


@pytest.mark.parametrize("n,d,two", [(3, 40001, False), (4, 12345, True), (2, 7, True), (1, 65536, True)])
def test_dequantize_matches_oracle(E, O, n, d, two):
    X = W.random_case(300 + d, n, d, "laplace")
    p, s, b = 64, 8, 2.0
    Xd = _cu(X)
    P, cnt, A, B, _ = E.grid_bucket(Xd, p)
    g = E.solve_budget_stats(cnt, A, B, P, d, s, b)
    Q2, L2, th = (g["Q2"], g["Q2_len"], g["theta"]) if two else (None, None, None)
    seed = 0x1234567890AB
    idx, hist, st = E.encode(Xd, P, s, g["Q1"], g["Q1_len"], seed, Q2, L2, th)
    assert int(st.abs().sum()) == 0
    Xh, st2 = E.dequantize(idx, P, s, g["Q1"], g["Q1_len"], seed, Q2, L2, th)
    assert int(st2.abs().sum()) == 0
    gn = {k: v.cpu().numpy() for k, v in g.items()}
    ref, so = O.dequantize_batch(idx.cpu().numpy(), P.cpu().numpy(), gn["Q1"], gn["Q1_len"], s, seed,
                                 gn["Q2"] if two else None, gn["Q2_len"] if two else None,
                                 gn["theta"] if two else None)
    assert np.all(so == 0)
    np.testing.assert_array_equal(Xh.cpu().numpy(), ref)


def test_dequantize_unaligned_rows(E, O):
    """Rows of odd length start at unaligned addresses: the scalar path."""
    X = W.random_case(310, 5, 1001, "normal")
    Xd = _cu(X)
    s = 6
    P, cnt, A, B, _ = E.grid_bucket(Xd, 48)
    g = E.solve_budget_stats(cnt, A, B, P, 1001, s, 1.5)
    idx, _, _ = E.encode(Xd, P, s, g["Q1"], g["Q1_len"], 9, g["Q2"], g["Q2_len"], g["theta"])
    Xh, st = E.dequantize(idx, P, s, g["Q1"], g["Q1_len"], 9, g["Q2"], g["Q2_len"], g["theta"])
    gn = {k: v.cpu().numpy() for k, v in g.items()}
    ref, _ = O.dequantize_batch(idx.cpu().numpy(), P.cpu().numpy(), gn["Q1"], gn["Q1_len"], s, 9, gn["Q2"],
                                gn["Q2_len"], gn["theta"])
    assert int(st.abs().sum()) == 0
    np.testing.assert_array_equal(Xh.cpu().numpy(), ref)


def test_mean_over_seeds_equals_x(E):
    """One 2^20-entry row, one 8-value code, 64 seeds: the mean of X^ minus X,
    scaled by each entry's binomial standard error, has mean ~0 and variance ~1."""
    X = W.random_case(320, 1, 1 << 20, "normal")
    Xd = _cu(X)
    P, cnt, A, B, _ = E.grid_bucket(Xd, 128)
    s = 8
    g = E.solve_stats(cnt, A, B, P, X.shape[1], s, _cu(np.array([[0.05]])))
    Q = g["Q"][:, 0, :].contiguous()
    m = g["Q_len"][:, 0].contiguous()
    acc = torch.zeros(X.shape[1], dtype=torch.float64, device="cuda")
    seeds = 64
    for k in range(seeds):
        idx, _, _ = E.encode(Xd, P, s, Q, m, 777 + k)
        Xh, st = E.dequantize(idx, P, s, Q, m, 777 + k)
        assert int(st.abs().sum()) == 0
        acc += Xh[0].double()
    mean = (acc / seeds).cpu().numpy()
    x = X[0].astype(np.float64)
    q = P[0].cpu().numpy()[Q[0, : int(m[0])].cpu().numpy()]
    i = np.clip(np.searchsorted(q, x, side="right") - 1, 0, q.size - 2)
    w = q[i + 1] - q[i]
    u = (x - q[i]) / w
    se = w * np.sqrt(u * (1 - u) / seeds)
    ok = se > 0
    z = (mean[ok] - x[ok]) / se[ok]
    assert abs(z.mean()) < 0.02 and abs(z.var() - 1.0) < 0.05
    assert np.all(mean[~ok] == x[~ok].astype(np.float32))


def test_index_outside_code_flagged(E):
    X = W.random_case(330, 2, 64, "normal")
    Xd = _cu(X)
    P, _ = E.uniform_grid(Xd, 16)
    Q = _cu(np.tile(np.array([0, 15, -1, -1], np.int32), (2, 1)))
    m = _cu(np.array([2, 2], np.int32))
    idx = torch.zeros((2, 64), dtype=torch.uint8, device="cuda")
    idx[1, 10] = 3
    _, st = E.dequantize(idx, P, 4, Q, m, 1)
    assert st.cpu().tolist() == [0, -2]
