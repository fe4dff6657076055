"""Pins of the oracle's entropy coder for the emitted indices (CPU): static-model
rANS ("Entropy-Constrained Adaptive Stochastic Quantization (ECASQ)",
gist.science/pt/paper/2608.18147, §1 "Contexto": a lossless entropy coder gives
frequent values shorter bit strings; rANS after Duda, arXiv:1311.2540).

Pins: the quantised model on hand-worked counts; the exact stream of a uniform
two-symbol model (each state doubles per symbol, so a state emits one zero word
every 16 symbols and ends at 2^(16 + T mod 16)); round trips through the
decoder for every layout case (ragged tails, several segments, time-shared
parts, a part that never occurs, a certain symbol); and the coded size against
the ideal code length sum log2(M/f) plus the final states.
"""
import math

import numpy as np
import pytest

M = 1 << 15


def _hist_of(idx, s, parts=None):
    n, d = idx.shape
    h = np.zeros((n, 2, s), np.int64)
    for r in range(n):
        pr = np.zeros(d, np.int64) if parts is None else parts[r]
        for p in (0, 1):
            h[r, p] = np.bincount(idx[r][pr == p], minlength=s)
    return h


@pytest.mark.parametrize("cnt,f", [
    ([3, 1], [24576, 8192]),
    ([1, 0, 0, 1000000], [1, 0, 0, 32767]),
    ([5, 5, 5], [10924, 10922, 10922]),        # floors 10922 x 3 = 32766: the shortfall 2 goes to the first maximum
    ([1] * 200 + [1000000], [1] * 200 + [32568]),  # 200 floors bumped to 1: excess taken from the largest
    ([0, 0, 7], [0, 0, 32768]),
])
def test_model_hand_worked(O, cnt, f):
    fo, cum = O.rans_model(np.array(cnt))
    assert list(fo) == f
    assert cum[-1] == M and list(np.diff(cum)) == f


@pytest.mark.parametrize("T", [1, 15, 16, 17, 40, 512])
def test_uniform_two_symbol_stream_closed_form(O, T):
    d = 32 * T
    idx = np.zeros((1, d), np.uint8)
    hist = np.zeros((1, 2, 2), np.int64)
    hist[0, 0] = [1, 1]  # model f = (M/2, M/2); every entry is symbol 0
    words, seg_len, st = O.rans_encode(idx, hist, 1)
    assert st[0] == 0
    e = T // 16
    assert seg_len[0, 0] == 32 * e + 64
    w = words[0, 0, : seg_len[0, 0]]
    assert np.all(w[: 32 * e] == 0)
    xT = 1 << (16 + T % 16)
    assert np.all(w[32 * e:: 2] == (xT & 0xFFFF)) and np.all(w[32 * e + 1:: 2] == (xT >> 16))


@pytest.mark.parametrize("case", ["ragged", "segments", "timeshare", "certain", "skewed"])
def test_round_trip_and_size(O, case):
    rng = np.random.default_rng(abs(hash(case)) % 1000)
    n, s, two, theta, parts = 3, 16, False, None, None
    d = {"ragged": 1001, "segments": 16384 * 2 + 77, "timeshare": 5000, "certain": 3000, "skewed": 40000}[case]
    probs = rng.dirichlet(np.ones(s) * 0.3)
    idx = rng.choice(s, size=(n, d), p=probs).astype(np.uint8)
    if case == "certain":
        idx[:] = 3
    if case == "timeshare":
        two = True
        theta = np.array([0.3, 0.0, 1.0])
        # the parts the coder derives from the seed, read back through a second model-free pass
        parts = np.zeros((n, d), np.int64)
        parts[1] = 1
        from oracle import oracle as OO
        L = OO.lib()
        # part of entry j for row 0: Philox stream 1 word vs theta
        for j in range(d):
            ctr = np.array([j >> 2, 0, 1, 0], np.uint32)
            out = OO.philox4x32(ctr, np.array([5, 0], np.uint32))
            parts[0, j] = 0 if out[j & 3] * 2.0 ** -32 < 0.3 else 1
        del L
    hist = _hist_of(idx, s, parts)
    words, seg_len, st = O.rans_encode(idx, hist, 5, theta, two)
    assert np.all(st == 0)
    dec, st2 = O.rans_decode(words, seg_len, d, hist, 5, theta, two)
    assert np.all(st2 == 0) and np.array_equal(dec, idx)
    nseg = seg_len.shape[1]
    for r in range(n):
        ideal = 0.0
        for p in (0, 1):
            f, _ = O.rans_model(hist[r, p])
            c = hist[r, p]
            ideal += sum(int(c[i]) * math.log2(M / int(f[i])) for i in range(s) if c[i] > 0)
        bits = 16 * int(seg_len[r].sum())
        assert ideal - 64 * nseg <= bits <= ideal * 1.002 + 1024 * nseg + 64 * nseg, (case, r, bits, ideal)


def test_zero_frequency_symbol_is_an_error(O):
    idx = np.array([[0, 1, 2, 1]], np.uint8)
    hist = np.zeros((1, 2, 3), np.int64)
    hist[0, 0] = [1, 2, 0]  # symbol 2 has no frequency
    _, _, st = O.rans_encode(idx, hist, 1)
    assert st[0] == -1
