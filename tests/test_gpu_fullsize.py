"""Full-size workloads on the GPU, in the launch configuration bench.py times,
checked against the fp64 oracle on sampled rows.

Each workload runs over all its rows on the device (grid, bucketing, solver,
encoder, entropy); the oracle recomputes a deterministic row sample one row at
a time. Tolerances as in test_gpu_parity.py: objective 1e-5 relative for the
fp32 DP (the throughput path bench.py times), codes re-scored by the oracle,
encodings bit-exact for the same code and seed.
"""
import numpy as np
import pytest
import torch

from entropy_constrained_unbiased_b200 import workloads as W

pytestmark = pytest.mark.gpu

RTOL32 = 1e-5
RTOL64 = 1e-9


@pytest.fixture(scope="module")
def E():
    from entropy_constrained_unbiased_b200 import build, ecasq
    assert torch.cuda.is_available()
    build.build()
    ecasq.load()
    return ecasq


def _sample(n, k):
    if n <= k:
        return np.arange(n)
    return np.unique(np.linspace(0, n - 1, k).round().astype(int))


def _full(E, w):
    X = W.make_inputs(w)
    Xd = torch.from_numpy(X).cuda()
    P, st = E.uniform_grid(Xd, w.p)
    cnt, A, B, st2 = E.bucket(Xd, P)
    assert int(st.abs().sum()) == 0 and int(st2.abs().sum()) == 0
    return X, Xd, P, cnt, A, B


@pytest.mark.parametrize("name,rows", [("small", 1), ("sweep", 12), ("mixture", 3)])
def test_fullsize_lambda_workloads(E, O, name, rows):
    w = W.WORKLOADS[name]
    X, Xd, P, cnt, A, B = _full(E, w)
    lam = w.lambdas()
    g = E.solve_stats(cnt, A, B, P, w.d, w.s, torch.from_numpy(lam).cuda(), hirschberg=w.hirschberg)
    assert int(g["status"].abs().sum()) == 0
    Q = g["Q"].cpu().numpy()
    m = g["Q_len"].cpu().numpy()
    Pn = P.cpu().numpy()
    idx = _sample(w.n, rows)
    Po, _ = O.grid_batch(X[idx], w.p)
    np.testing.assert_array_equal(Pn[idx], Po)
    ref = O.solve_batch(X[idx], Po, w.s, lam[idx])
    for a, r in enumerate(idx):
        for t in range(lam.shape[1]):
            mse, H, _ = O.eval_raw(X[r], Po[a][Q[r, t, : m[r, t]]])
            J = mse + lam[r, t] * H
            assert J <= ref["J"][a, t] * (1 + RTOL32), (r, t, J, ref["J"][a, t])
            assert g["objective"][r, t].item() == pytest.approx(J, rel=RTOL64)
    # encode every row with its first code; sampled rows bit-exact vs the oracle
    Q0 = g["Q"][:, 0, :].contiguous()
    m0 = g["Q_len"][:, 0].contiguous()
    code, hist, est = E.encode(Xd, P, w.s, Q0, m0, w.seed_encode)
    assert int(est.abs().sum()) == 0
    Q0n, m0n = Q0.cpu().numpy(), m0.cpu().numpy()
    for a, r in enumerate(idx):
        io, ho = O.encode_row(X[r], Po[a], Q0n[r], m0n[r], w.s, w.seed_encode, int(r))
        np.testing.assert_array_equal(code[r].cpu().numpy(), io)
        np.testing.assert_array_equal(hist[r].cpu().numpy(), ho)


@pytest.mark.parametrize("name,rows", [("weights", 16), ("gradients", 8)])
def test_fullsize_budget_workloads(E, O, name, rows):
    w = W.WORKLOADS[name]
    X, Xd, P, cnt, A, B = _full(E, w)
    g = E.solve_budget_stats(cnt, A, B, P, w.d, w.s, w.b, w.steps)
    gn = {k: v.cpu().numpy() for k, v in g.items()}
    assert np.all(gn["status"] == 0)
    idx = _sample(w.n, rows)
    Po, _ = O.grid_batch(X[idx], w.p)
    ref = O.solve_budget_batch(X[idx], Po, w.s, w.b, w.steps)
    lams = np.zeros((len(idx), 2))
    Js = np.zeros((len(idx), 2))
    for a, r in enumerate(idx):
        th = gn["theta"][r]
        if 0 < th < 1:
            assert th * gn["H1"][r] + (1 - th) * gn["H2"][r] == pytest.approx(w.b, rel=1e-12)
        d_gpu = th * gn["mse1"][r] + (1 - th) * gn["mse2"][r]
        d_ref = ref["theta"][a] * ref["mse1"][a] + (1 - ref["theta"][a]) * ref["mse2"][a]
        assert d_gpu == pytest.approx(d_ref, rel=RTOL32), (r, d_gpu, d_ref)
        for qk, mk, lk in (("Q1", "Q1_len", "lambda_lo"), ("Q2", "Q2_len", "lambda_hi")):
            mse, H, _ = O.eval_raw(X[r], Po[a][gn[qk][r, : gn[mk][r]]])
            assert gn["H1" if qk == "Q1" else "H2"][r] == pytest.approx(H, rel=RTOL64)
            assert gn["mse1" if qk == "Q1" else "mse2"][r] == pytest.approx(mse, rel=RTOL64)
            lams[a, 0 if qk == "Q1" else 1] = gn[lk][r]
            Js[a, 0 if qk == "Q1" else 1] = mse + gn[lk][r] * H
    # both codes are Lagrangian optima at the GPU's own multipliers: the
    # oracle's exact DP at lambda_lo and lambda_hi reaches the same objective
    # (to the fp32 DP's 1e-5)
    opt = O.solve_batch(X[idx], Po, w.s, lams)
    for a in range(len(idx)):
        for t in range(2):
            assert Js[a, t] <= opt["J"][a, t] * (1 + RTOL32) + 1e-300, (idx[a], t, Js[a, t], opt["J"][a, t])
    # time-shared encode of every row; sampled rows bit-exact
    code, hist, est = E.encode(Xd, P, w.s, g["Q1"], g["Q1_len"], w.seed_encode, g["Q2"], g["Q2_len"], g["theta"])
    assert int(est.abs().sum()) == 0
    Hemp = E.entropy(hist).cpu().numpy()
    hn = hist.cpu().numpy()
    for a, r in enumerate(idx):
        io, ho = O.encode_row(X[r], Po[a], gn["Q1"][r], gn["Q1_len"][r], w.s, w.seed_encode, int(r),
                              gn["Q2"][r], gn["Q2_len"][r], gn["theta"][r])
        np.testing.assert_array_equal(code[r].cpu().numpy(), io)
        np.testing.assert_array_equal(hn[r], ho)
        assert Hemp[r] == pytest.approx(O.entropy(ho, w.s), rel=1e-12)
    # empirical rate tracks the budget
    assert abs(float(np.mean(Hemp)) - w.b) < 0.05



def test_fullsize_weights_fp64_parity(E, O):
    """The fp64 DP (the 1e-9 parity mode) on full-size weight rows: the budget
    solve of the first 256 rows of the weights workload (4096 entries each) in
    fp64 layers; sampled rows against the oracle's bisection to 1e-9."""
    import dataclasses

    w = dataclasses.replace(W.WORKLOADS["weights"], n=256)
    X, Xd, P, cnt, A, B = _full(E, w)
    g = E.solve_budget_stats(cnt, A, B, P, w.d, w.s, w.b, w.steps, fp64=True)
    gn = {k: v.cpu().numpy() for k, v in g.items()}
    assert np.all(gn["status"] == 0)
    idx = _sample(w.n, 8)
    Po, _ = O.grid_batch(X[idx], w.p)
    ref = O.solve_budget_batch(X[idx], Po, w.s, w.b, w.steps)
    for a, r in enumerate(idx):
        for k_g, k_o in (("theta", "theta"), ("lambda_lo", "lam_lo"), ("lambda_hi", "lam_hi"), ("H1", "H1"),
                         ("H2", "H2"), ("mse1", "mse1"), ("mse2", "mse2")):
            assert gn[k_g][r] == pytest.approx(ref[k_o][a], rel=RTOL64, abs=1e-15), (r, k_g)


# -- approximation on H(I,B) and refinement at full size ---------------------------

@pytest.mark.parametrize("refine", [0, 8])
@pytest.mark.parametrize("name,rows", [("weights", 12), ("gradients", 3)])
def test_fullsize_approx_budget(E, O, name, rows, refine):
    """All rows on the device (fp32 layers, as bench.py times them); sampled rows
    against the oracle: time-shared MSE to 1e-5, the rate identity, and the
    GPU's fp64 figures of each code against the oracle's raw evaluation."""
    w = W.WORKLOADS[name]
    X, Xd, P, cnt, A, B = _full(E, w)
    g = E.solve_approx_budget_stats(cnt, A, B, P, w.d, w.s, w.b, refine=refine, steps=w.steps)
    gn = {k: v.cpu().numpy() for k, v in g.items()}
    assert np.all(gn["status"] == 0)
    idx = _sample(w.n, rows)
    Po, _ = O.grid_batch(X[idx], w.p)
    ref = O.solve_approx_budget_batch(X[idx], Po, w.s, w.b, w.steps, refine=refine)
    rate = "H" if refine else "H_IB"
    for a, r in enumerate(idx):
        th = gn["theta"][r]
        if 0 < th < 1:
            assert th * gn[rate + "1"][r] + (1 - th) * gn[rate + "2"][r] == pytest.approx(w.b, rel=1e-12)
        d_gpu = th * gn["mse1"][r] + (1 - th) * gn["mse2"][r]
        d_ref = ref["theta"][a] * ref["mse1"][a] + (1 - ref["theta"][a]) * ref["mse2"][a]
        assert d_gpu == pytest.approx(d_ref, rel=RTOL32), (r, d_gpu, d_ref)
        for q, m, k in (("Q1", "Q1_len", "1"), ("Q2", "Q2_len", "2")):
            code = gn[q][r, : gn[m][r]]
            mse, H, _ = O.eval_raw(X[r], Po[a][code])
            assert gn["mse" + k][r] == pytest.approx(mse, rel=RTOL64)
            assert gn["H" + k][r] == pytest.approx(H, rel=RTOL64)
            assert gn["H_IB" + k][r] == pytest.approx(O.eval_raw_ib(X[r], Po[a][code]), rel=RTOL64)


@pytest.mark.parametrize("name,rows", [("sweep", 6), ("mixture", 2), ("small", 1)])
def test_fullsize_approx_lambda(E, O, name, rows):
    w = W.WORKLOADS[name]
    X, Xd, P, cnt, A, B = _full(E, w)
    lam = w.lambdas()
    g = E.solve_approx_stats(cnt, A, B, P, w.d, w.s, torch.from_numpy(lam).cuda())
    assert int(g["status"].abs().sum()) == 0
    Q, m = g["Q"].cpu().numpy(), g["Q_len"].cpu().numpy()
    idx = _sample(w.n, rows)
    Po, _ = O.grid_batch(X[idx], w.p)
    ref = O.solve_approx_batch(X[idx], Po, w.s, lam[idx])
    for a, r in enumerate(idx):
        for t in range(lam.shape[1]):
            code = Q[r, t, : m[r, t]]
            mse, _, _ = O.eval_raw(X[r], Po[a][code])
            J = mse + lam[r, t] * O.eval_raw_ib(X[r], Po[a][code])
            assert J <= ref["J"][a, t] * (1 + RTOL32), (r, t, J, ref["J"][a, t])
            assert g["objective"][r, t].item() == pytest.approx(J, rel=RTOL64)
