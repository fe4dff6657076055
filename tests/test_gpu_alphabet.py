"""GPU hardware-aware permissible set vs the oracle, through the C ABI, and the
solver on that alphabet ("Entropy-Constrained Adaptive Stochastic Quantization
(ECASQ)", gist.science/pt/paper/2608.18147, §5 "Generalidade").

The alphabet is integer/bit work: P, its length and the status must be
bit-exact. The solver on a BF16 alphabet is held to the objective tolerances of
the other parity tests (fp64 1e-9, fp32 1e-5) and every value of its codes is a
BF16 number.
"""
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


def _rows(seed, n, d):
    rng = np.random.default_rng([47, seed])
    out = np.empty((n, d), np.float32)
    for r in range(n):
        scale = 10.0 ** rng.uniform(-30, 2)
        shift = rng.uniform(-3, 3) * scale
        out[r] = shift + scale * rng.standard_normal(d)
    return out


@pytest.mark.parametrize("seed,n,d", [(0, 6, 1000), (1, 3, 70001), (2, 5, 1)])
def test_bf16_alphabet_bit_exact(E, O, seed, n, d):
    X = _rows(seed, n, d)
    p_max = 65536
    P, p_len, st = E.bf16_alphabet(torch.from_numpy(X).cuda(), p_max)
    P, p_len, st = P.cpu().numpy(), p_len.cpu().numpy(), st.cpu().numpy()
    for r in range(n):
        ref, cnt = O.bf16_alphabet(X[r], p_max)
        assert p_len[r] == cnt
        assert st[r] == (0 if cnt <= p_max else -1)
        np.testing.assert_array_equal(P[r, :cnt], ref)
        assert np.all(np.isnan(P[r, cnt:]))


def test_bf16_alphabet_truncation_and_errors(E, O):
    X = np.stack([np.linspace(-1, 1, 64, dtype=np.float32), np.linspace(1, 1.5, 64, dtype=np.float32),
                  np.linspace(1, 2, 64, dtype=np.float32)])
    X[2, 5] = np.nan
    P, p_len, st = E.bf16_alphabet(torch.from_numpy(X).cuda(), 512)
    P, p_len, st = P.cpu().numpy(), p_len.cpu().numpy(), st.cpu().numpy()
    assert list(st) == [-1, 0, -2]
    assert p_len[0] == 32513 and p_len[1] == 65 and p_len[2] == 0
    ref, _ = O.bf16_alphabet(X[0], 512)
    np.testing.assert_array_equal(P[0], ref)


@pytest.mark.parametrize("fp64,tol", [(True, 1e-9), (False, 1e-5)])
def test_solver_on_a_bf16_alphabet(E, O, fp64, tol):
    """Rows spanning [1, 1.5] exactly: one 65-value BF16 alphabet (spacing 2^-7)."""
    rng = np.random.default_rng(53)
    X = (1.0 + 0.5 * rng.beta(2, 5, size=(4, 5000))).astype(np.float32)
    X[:, 0], X[:, 1] = 1.0, 1.5
    Pd, p_len, st = E.bf16_alphabet(torch.from_numpy(X).cuda(), 65)
    assert int(st.abs().sum()) == 0 and np.all(p_len.cpu().numpy() == 65)
    P = Pd.cpu().numpy()
    lam = np.var(X.astype(np.float64), axis=1)[:, None] * np.array([[0.0, 0.01, 0.1]])
    g = E.solve(torch.from_numpy(X).cuda(), Pd, 10, torch.from_numpy(lam).cuda(), fp64=fp64)
    ref = O.solve_batch(X, P, 10, lam)
    Q, m = g["Q"].cpu().numpy(), g["Q_len"].cpu().numpy()
    for r in range(X.shape[0]):
        for t in range(lam.shape[1]):
            vals = P[r][Q[r, t, : m[r, t]]]
            assert np.all((vals.astype(np.float32).view(np.uint32) & 0xFFFF) == 0)
            mse, H, _ = O.eval_raw(X[r], vals)
            assert mse + lam[r, t] * H <= ref["J"][r, t] * (1 + tol) + 1e-300


# -- large alphabets (p > 512): bucketing, the approximation, encoding -------------

def _wide_rows(seed, n, d):
    """Rows whose BF16 alphabet is the same 1237 values (0.0498 .. 40): each row
    holds 0.05 and 40, the rest lognormal in between."""
    rng = np.random.default_rng([59, seed])
    X = np.exp(rng.uniform(np.log(0.05), np.log(40.0), size=(n, d)) + 0.3 * rng.standard_normal((n, d)))
    X = np.clip(X, 0.05, 40.0).astype(np.float32)
    X[:, 0], X[:, 1] = np.float32(0.05), np.float32(40.0)
    return X


@pytest.fixture(scope="module")
def wide(E):
    X = _wide_rows(0, 3, 20000)
    Pd, p_len, st = E.bf16_alphabet(torch.from_numpy(X).cuda(), 2048)
    p = int(p_len[0].item())
    assert int(st.abs().sum()) == 0 and np.all(p_len.cpu().numpy() == p) and p > 512
    P = Pd[:, :p].contiguous()
    return X, P, p


def test_bucket_large_alphabet(E, O, wide):
    X, P, p = wide
    cnt, A, B, st = E.bucket(torch.from_numpy(X).cuda(), P)
    assert int(st.abs().sum()) == 0
    Pn = P.cpu().numpy()
    for r in range(X.shape[0]):
        co, Ao, Bo, so = O.bucket(X[r], Pn[r])
        assert so == 0
        np.testing.assert_array_equal(cnt[r].cpu().numpy(), co)
        span = Pn[r, -1] - Pn[r, 0]
        np.testing.assert_allclose(A[r].cpu().numpy(), Ao, rtol=1e-9, atol=1e-12 * span)
        np.testing.assert_allclose(B[r].cpu().numpy(), Bo, rtol=1e-9, atol=1e-12 * span ** 2)


@pytest.mark.parametrize("refine", [0, 4])
def test_approx_large_alphabet(E, O, wide, refine):
    """The approximation on a 1237-value BF16 alphabet (fp32 layers, pair terms
    from prefix sums): the code's objective within 1e-5 of the oracle's optimum
    (plain), the GPU's fp64 figures of its code equal to the oracle's raw
    evaluation, every code value a BF16 number; refined codes never worse
    than the plain ones on the exact objective."""
    X, P, p = wide
    Xd = torch.from_numpy(X).cuda()
    lam = np.var(X.astype(np.float64), axis=1)[:, None] * np.array([[0.0, 0.003, 0.03]])
    s = 12
    g = E.solve_approx(Xd, P, s, torch.from_numpy(lam).cuda(), refine=refine)
    assert int(g["status"].abs().sum()) == 0
    Pn = P.cpu().numpy()
    Q, m = g["Q"].cpu().numpy(), g["Q_len"].cpu().numpy()
    ref = O.solve_approx_batch(X, Pn, s, lam, refine=0)
    for r in range(X.shape[0]):
        for t in range(lam.shape[1]):
            vals = Pn[r][Q[r, t, : m[r, t]]]
            assert np.all((vals.astype(np.float32).view(np.uint32) & 0xFFFF) == 0)
            mse, H, _ = O.eval_raw(X[r], vals)
            hib = O.eval_raw_ib(X[r], vals)
            assert g["mse"][r, t].item() == pytest.approx(mse, rel=1e-9)
            assert g["H"][r, t].item() == pytest.approx(H, rel=1e-9, abs=1e-12)
            assert g["H_IB"][r, t].item() == pytest.approx(hib, rel=1e-9, abs=1e-12)
            J_ib = mse + lam[r, t] * hib
            if refine == 0:
                assert J_ib <= ref["J"][r, t] * (1 + 1e-5), (r, t, J_ib, ref["J"][r, t])
                assert g["objective"][r, t].item() == pytest.approx(J_ib, rel=1e-9)
            else:
                assert g["objective"][r, t].item() == pytest.approx(mse + lam[r, t] * H, rel=1e-9)
                # refinement starts from the plain code and only moves on a decrease
                mse0, H0, _ = O.eval_raw(X[r], Pn[r][ref["Q"][r, t, : ref["m"][r, t]]])
                assert mse + lam[r, t] * H <= (mse0 + lam[r, t] * H0) * (1 + 1e-5) + 1e-300


def test_approx_budget_and_encode_large_alphabet(E, O, wide):
    X, P, p = wide
    Xd = torch.from_numpy(X).cuda()
    s, b = 12, 2.5
    g = E.solve_approx_budget(Xd, P, s, b, refine=0, steps=30)
    gn = {k: v.cpu().numpy() for k, v in g.items()}
    assert np.all(gn["status"] == 0)
    Pn = P.cpu().numpy()
    ref = O.solve_approx_budget_batch(X, Pn, s, b, 30, refine=0)
    for r in range(X.shape[0]):
        th = gn["theta"][r]
        if 0 < th < 1:
            assert th * gn["H_IB1"][r] + (1 - th) * gn["H_IB2"][r] == pytest.approx(b, rel=1e-12)
        d_gpu = th * gn["mse1"][r] + (1 - th) * gn["mse2"][r]
        d_ref = ref["theta"][r] * ref["mse1"][r] + (1 - ref["theta"][r]) * ref["mse2"][r]
        assert d_gpu == pytest.approx(d_ref, rel=1e-5), (r, d_gpu, d_ref)
    # time-shared encoding on the large alphabet: bit-exact against the oracle
    idx, hist, est = E.encode(Xd, P, s, g["Q1"], g["Q1_len"], 7, g["Q2"], g["Q2_len"], g["theta"])
    assert int(est.abs().sum()) == 0
    io, ho, so = O.encode_batch(X, Pn, gn["Q1"], gn["Q1_len"], s, 7, gn["Q2"], gn["Q2_len"], gn["theta"])
    assert np.all(so == 0)
    np.testing.assert_array_equal(idx.cpu().numpy(), io)
    np.testing.assert_array_equal(hist.cpu().numpy(), ho)
    # and the reconstruction on the large alphabet
    Xh, sd = E.dequantize(idx, P, s, g["Q1"], g["Q1_len"], 7, g["Q2"], g["Q2_len"], g["theta"])
    ref, sr = O.dequantize_batch(io, Pn, gn["Q1"], gn["Q1_len"], s, 7, gn["Q2"], gn["Q2_len"], gn["theta"])
    assert int(sd.abs().sum()) == 0 and np.all(sr == 0)
    np.testing.assert_array_equal(Xh.cpu().numpy(), ref)


@pytest.mark.parametrize("s", [6, 24, 40])
def test_approx_large_alphabet_code_sizes(E, O, wide, s):
    """Code sizes on each side of the tiled layer sweep's register blocks (up to
    8, 16 and 32 layers after the first) and past them (the layer-by-layer
    sweep): the objective within 1e-5 of the oracle's optimum and the fp64
    figures equal to the oracle's raw evaluation."""
    X, P, p = wide
    Xd = torch.from_numpy(X).cuda()
    lam = np.var(X.astype(np.float64), axis=1)[:, None] * np.array([[0.001, 0.01]])
    g = E.solve_approx(Xd, P, s, torch.from_numpy(lam).cuda())
    assert int(g["status"].abs().sum()) == 0
    Pn = P.cpu().numpy()
    Q, m = g["Q"].cpu().numpy(), g["Q_len"].cpu().numpy()
    ref = O.solve_approx_batch(X, Pn, s, lam, refine=0)
    for r in range(X.shape[0]):
        for t in range(lam.shape[1]):
            assert 2 <= m[r, t] <= s
            vals = Pn[r][Q[r, t, : m[r, t]]]
            mse, _, _ = O.eval_raw(X[r], vals)
            J_ib = mse + lam[r, t] * O.eval_raw_ib(X[r], vals)
            assert J_ib <= ref["J"][r, t] * (1 + 1e-5), (r, t, J_ib, ref["J"][r, t])
            assert g["objective"][r, t].item() == pytest.approx(J_ib, rel=1e-9)


def test_approx_4097_value_alphabet_single_column_tail(E, O):
    """A 4097-value BF16 alphabet (every BF16 value in [2^-16, 2^16]): the tiled
    sweep's last X-tile holds one column (4097 = 128 x 32 + 1). One row at one
    lambda (the oracle's O(p^2) tables take seconds here) against the oracle's
    optimum, fp64 figures against its raw evaluation."""
    X = W.pinned_range_rows(7, 1, 65536, 2.0 ** -16, 2.0 ** 16)
    Xd = torch.from_numpy(X).cuda()
    Pd, p_len, st = E.bf16_alphabet(Xd, 8192)
    p = int(p_len[0].item())
    assert p == 4097 and int(st.abs().sum()) == 0
    P = Pd[:, :p].contiguous()
    lam = np.var(X.astype(np.float64), axis=1)[:, None] * np.array([[0.01]])
    s = 16
    g = E.solve_approx(Xd, P, s, torch.from_numpy(lam).cuda())
    assert int(g["status"].abs().sum()) == 0
    Pn = P.cpu().numpy()
    ref = O.solve_approx_batch(X, Pn, s, lam, refine=0)
    Q, m = g["Q"].cpu().numpy(), g["Q_len"].cpu().numpy()
    for t in range(lam.shape[1]):
        vals = Pn[0][Q[0, t, : m[0, t]]]
        mse, _, _ = O.eval_raw(X[0], vals)
        J_ib = mse + lam[0, t] * O.eval_raw_ib(X[0], vals)
        assert J_ib <= ref["J"][0, t] * (1 + 1e-5), (t, J_ib, ref["J"][0, t])
        assert g["objective"][0, t].item() == pytest.approx(J_ib, rel=1e-9)
