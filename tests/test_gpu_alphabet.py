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
