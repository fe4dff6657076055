"""Pins of the oracle's reconstruction X^ from the emitted indices, and through
it of the encoder's stochastic rounding ("Entropy-Constrained Adaptive
Stochastic Quantization (ECASQ)", gist.science/pt/paper/2608.18147, §1 "O
Problema ECASQ": unbiased stochastic quantization, E[X^] = X; §2.1: two-way
time-sharing on a random partition).

Pins, each checked against numpy rather than the oracle itself:
- every reconstructed value is one of the two code values that bracket its
  entry;
- over many seeds the mean of X^ is X, within the binomial error of the
  rounding;
- the share of entries in the first code is theta, within its binomial error.
"""
import numpy as np
import pytest


def _case(seed, n, d, p, code):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((n, d)).astype(np.float32)
    return X, np.array(code, np.int32)


def test_values_bracket_their_entries(O):
    X, code = _case(1, 3, 2000, 64, [0, 7, 20, 33, 50, 63])
    s = 8
    P, _ = O.grid_batch(X, 64)
    Q = np.full((3, s), -1, np.int32)
    Q[:, : code.size] = code
    m = np.full(3, code.size, np.int32)
    idx, _, st = O.encode_batch(X, P, Q, m, s, 11)
    assert np.all(st == 0)
    Xh, st2 = O.dequantize_batch(idx, P, Q, m, s, 11)
    assert np.all(st2 == 0)
    for r in range(3):
        q = P[r][code]
        i = np.clip(np.searchsorted(q, X[r].astype(np.float64), side="right") - 1, 0, code.size - 2)
        lo, hi = q[i].astype(np.float32), q[i + 1].astype(np.float32)
        assert np.all((Xh[r] == lo) | (Xh[r] == hi))


def test_mean_over_seeds_is_unbiased(O):
    X, code = _case(2, 1, 48, 32, [0, 4, 13, 22, 31])
    s = 5
    P, _ = O.grid_batch(X, 32)
    Q = code[None, :]
    m = np.array([code.size], np.int32)
    seeds = 3000
    acc = np.zeros(X.shape[1])
    for seed in range(seeds):
        idx, _, _ = O.encode_batch(X, P, Q, m, s, 1000 + seed)
        Xh, _ = O.dequantize_batch(idx, P, Q, m, s, 1000 + seed)
        acc += Xh[0].astype(np.float64)
    mean = acc / seeds
    q = P[0][code]
    x = X[0].astype(np.float64)
    i = np.clip(np.searchsorted(q, x, side="right") - 1, 0, code.size - 2)
    w = q[i + 1] - q[i]
    u = (x - q[i]) / w  # probability of rounding up
    sd = w * np.sqrt(u * (1 - u) / seeds)
    # 5 standard errors per entry (plus the float32 rounding of the values)
    assert np.all(np.abs(mean - x) <= 5 * sd + 1e-6 * np.abs(q).max())


def test_time_sharing_share(O):
    X, _ = _case(3, 2, 40000, 32, [0])
    s = 4
    P, _ = O.grid_batch(X, 32)
    Q1 = np.tile(np.array([0, 10, 31, -1], np.int32), (2, 1))
    Q2 = np.tile(np.array([0, 20, 31, -1], np.int32), (2, 1))
    m = np.full(2, 3, np.int32)
    theta = np.array([0.3, 0.75])
    idx, hist, st = O.encode_batch(X, P, Q1, m, s, 5, Q2, m, theta)
    assert np.all(st == 0)
    d = X.shape[1]
    share = hist[:, 0, :].sum(axis=1) / d
    assert np.all(np.abs(share - theta) <= 5 * np.sqrt(theta * (1 - theta) / d))
    Xh, st2 = O.dequantize_batch(idx, P, Q1, m, s, 5, Q2, m, theta)
    assert np.all(st2 == 0)
    # entries reconstructed to a value only Q2 holds were in part 1
    only2 = P[:, 20][:, None].astype(np.float32)
    assert np.all((Xh == only2).sum(axis=1) <= hist[:, 1, :].sum(axis=1))


def test_index_outside_code_is_an_error(O):
    X, code = _case(4, 1, 100, 16, [0, 15])
    P, _ = O.grid_batch(X, 16)
    idx = np.full((1, 100), 2, np.uint8)  # code has 2 values: index 2 is outside
    _, st = O.dequantize_batch(idx, P, code[None, :], np.array([2], np.int32), 2, 1)
    assert st[0] == -1
