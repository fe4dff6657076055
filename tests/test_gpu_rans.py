"""GPU entropy coder (rANS) for the emitted indices vs the oracle, through the C
ABI ("Entropy-Constrained Adaptive Stochastic Quantization (ECASQ)",
gist.science/pt/paper/2608.18147, §1 "Contexto"). Byte work: the coded words
and lengths must be bit-exact, and both decoders must return the indices.
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


def _cu(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _check(E, O, idx, hist, seed, theta=None, two=False):
    n, d = idx.shape
    th = None if theta is None else _cu(theta)
    w, L, st = E.rans_encode(_cu(idx), _cu(hist), seed, th, two)
    wo, Lo, sto = O.rans_encode(idx, hist, seed, theta, two)
    st = st.cpu().numpy()
    np.testing.assert_array_equal(st, sto)
    Ln = L.cpu().numpy()
    wn = w.cpu().numpy().view(np.uint16)
    for r in range(n):
        if sto[r] != 0:
            continue
        np.testing.assert_array_equal(Ln[r], Lo[r])
        for g in range(Ln.shape[1]):
            np.testing.assert_array_equal(wn[r, g, : Ln[r, g]], wo[r, g, : Lo[r, g]])
    ok = sto == 0
    if ok.any():
        dec, dst = E.rans_decode(w, L, _cu(hist), d, seed, th, two)
        dec, dst = dec.cpu().numpy(), dst.cpu().numpy()
        assert np.all(dst[ok] == 0)
        np.testing.assert_array_equal(dec[ok], idx[ok])
        deco, dsto = O.rans_decode(wn, Ln, d, hist, seed, theta, two)
        np.testing.assert_array_equal(deco[ok], idx[ok])
    return Ln


@pytest.mark.parametrize("d", [1, 31, 1001, 16384, 16384 * 2 + 77])
def test_rans_random_bit_exact(E, O, d):
    rng = np.random.default_rng(d)
    n, s = 4, 16
    probs = rng.dirichlet(np.ones(s) * 0.4)
    idx = rng.choice(s, size=(n, d), p=probs).astype(np.uint8)
    hist = np.zeros((n, 2, s), np.int64)
    for r in range(n):
        hist[r, 0] = np.bincount(idx[r], minlength=s)
    idx[3] = 5  # a certain symbol in one row
    hist[3, 0] = 0
    hist[3, 0, 5] = d
    _check(E, O, idx, hist, 11)


def test_rans_after_time_shared_encode(E, O):
    """The coder on the encoder's own output: two codes, theta per row (mixed,
    all-first, all-second), the part of each entry recomputed from the seed."""
    X = W.random_case(61, 3, 20000, "student_t")
    P, _ = O.grid_batch(X, 64)
    g = O.solve_budget_batch(X, P, 8, 2.0, 30)
    theta = g["theta"].copy()
    theta[1], theta[2] = 1.0, 0.0
    idx, hist, st = O.encode_batch(X, P, g["Q1"], g["m1"], 8, 9, g["Q2"], g["m2"], theta)
    assert np.all(st == 0)
    L = _check(E, O, idx, hist, 9, theta, True)
    d = X.shape[1]
    bits = 16 * L.sum(axis=1) / d
    for r in range(3):
        # the final states (32 states of 32 bits per segment) on top of the entropy
        H = O.entropy(hist[r], 8)
        assert bits[r] <= H + 1024 * L.shape[1] / d + 0.01, (r, bits[r], H)


def test_rans_zero_frequency_is_flagged(E, O):
    idx = np.array([[0, 1, 2, 1] * 10], np.uint8)
    hist = np.zeros((1, 2, 3), np.int64)
    hist[0, 0] = [10, 20, 0]
    _check(E, O, idx, hist, 1)


def test_rans_fullsize_weights(E, O):
    """The weights workload end to end on the device (budget solve, encode,
    coder); sampled rows bit-exact vs the oracle, every row decoded."""
    w = W.WORKLOADS["weights"]
    X = W.make_inputs(w)
    Xd = torch.from_numpy(X).cuda()
    P, _ = E.uniform_grid(Xd, w.p)
    cnt, A, B, _ = E.bucket(Xd, P)
    o = E.solve_budget_stats(cnt, A, B, P, w.d, w.s, w.b, w.steps)
    idx, hist, est = E.encode(Xd, P, w.s, o["Q1"], o["Q1_len"], w.seed_encode, o["Q2"], o["Q2_len"], o["theta"])
    words, L, st = E.rans_encode(idx, hist, w.seed_encode, o["theta"], True)
    assert int(st.abs().sum()) == 0
    dec, dst = E.rans_decode(words, L, hist, w.d, w.seed_encode, o["theta"], True)
    assert int(dst.abs().sum()) == 0 and torch.equal(dec, idx)
    Hemp = E.entropy(hist).cpu().numpy()
    bits = 16 * L.sum(dim=1).cpu().numpy() / w.d
    assert np.all(bits <= Hemp + 0.3)  # 32 final states of 32 bits on 4096 entries: <= 0.25 bit/entry
    # the row index enters the part selector: the oracle codes the whole batch
    idxn, histn, th = idx.cpu().numpy(), hist.cpu().numpy(), o["theta"].cpu().numpy()
    full_w, full_L, full_st = O.rans_encode(idxn, histn, w.seed_encode, th, True)
    assert np.all(full_st == 0)
    Ln = L.cpu().numpy()
    wn = words.cpu().numpy().view(np.uint16)
    np.testing.assert_array_equal(Ln, full_L)
    for r in (0, 1777, 4095):
        np.testing.assert_array_equal(wn[r, 0, : Ln[r, 0]], full_w[r, 0, : full_L[r, 0]])
