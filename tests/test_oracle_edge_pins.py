"""Pins of the oracle's edges: status values, batch layouts, output padding,
degenerate alphabets and the entropy coder's segment count and tie rules.

Each check fixes a behaviour that a slip in the oracle's plumbing could
change without moving any per-vector result: a row offset in a batch loop, the
-1 padding of a code shorter than s, the sign of an error status, an
off-by-one in a segment count, the order in which tied frequencies are
adjusted. The expected values come from the definitions (single-row calls,
the header's status constants, the stated model rule worked by hand), not from
the batch code under test.
"""
import re
from pathlib import Path

import numpy as np
import pytest

from oracle import oracle as O

ROOT = Path(__file__).resolve().parents[1]


def _abi_status(name):
    text = (ROOT / "include" / "ecasq.h").read_text()
    m = re.search(r"#define\s+%s\s+\((-?\d+)\)" % name, text)
    assert m, name
    return int(m.group(1))


ERR_RANGE = _abi_status("ECASQ_ERR_RANGE")
ERR_ARG = _abi_status("ECASQ_ERR_ARG")


def _rows(seed, n, d, scale=1.0):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((n, d)) * scale).astype(np.float32)


# -- status values -------------------------------------------------------------------

def test_range_status_is_the_abi_value():
    """An entry outside [P_0, P_{p-1}] (bucketing), outside the code's range
    (encoding), or off a one-value code gives ECASQ_ERR_RANGE, not just any
    nonzero value."""
    x = _rows(1, 1, 200)[0]
    P, st = O.uniform_grid(x, 16)
    assert st == 0
    x_out = x.copy()
    x_out[17] = np.float32(P[-1] + 1.0)
    assert O.bucket(x_out, P)[3] == ERR_RANGE
    x_low = x.copy()
    x_low[3] = np.float32(P[0] - 1.0)
    assert O.bucket(x_low, P)[3] == ERR_RANGE

    X = x[None, :]
    Pb = P[None, :]
    # code ends below max X
    Q = np.array([[0, 4, 9, -1]], np.int32)
    _, _, st = O.encode_batch(X, Pb, Q, np.array([3], np.int32), 4, seed=1)
    assert st[0] == ERR_RANGE
    # one-value code on a row that is not constant
    Q1 = np.array([[0, -1, -1, -1]], np.int32)
    _, _, st = O.encode_batch(X, Pb, Q1, np.array([1], np.int32), 4, seed=1)
    assert st[0] == ERR_RANGE
    # the raw evaluation of a code that does not cover the row, and of a
    # one-value code on a row that is not constant (the C call's own status)
    import ctypes as C
    mse, H = C.c_double(), C.c_double()
    for q in (np.ascontiguousarray(P[[0, 4, 9]]), np.ascontiguousarray(P[[3]])):
        mu = np.zeros(q.size)
        st = O.lib().eo_eval_raw(x, x.size, q, q.size, C.byref(mse), C.byref(H), mu.ctypes.data_as(C.c_void_p))
        assert st == ERR_RANGE


def test_constant_row_solves_to_one_value():
    """A constant vector: the grid collapses to one point, Q = {P_0} with J = 0;
    any entry off that point is out of range."""
    x = np.full(64, 0.25, np.float32)
    P, st = O.uniform_grid(x, 8)
    assert st == 0 and np.all(P == np.float64(np.float32(0.25)))
    out = O.solve_batch(x[None, :], P[None, :], 4, np.array([[0.1]]))
    assert out["status"][0, 0] == 0
    assert out["m"][0, 0] == 1 and out["Q"][0, 0, 0] == 0
    assert np.all(out["Q"][0, 0, 1:] == -1)
    assert out["J"][0, 0] == 0.0 and out["mse"][0, 0] == 0.0 and out["H"][0, 0] == 0.0
    y = x.copy()
    y[5] = np.float32(0.5)
    out = O.solve_batch(y[None, :], P[None, :], 4, np.array([[0.1]]))
    assert out["status"][0, 0] == ERR_RANGE
    # the approximation and both budget drivers take the same branch
    ap = O.solve_approx_batch(x[None, :], P[None, :], 4, np.array([0.1]), refine=2)
    assert ap["status"][0, 0] == 0 and ap["m"][0, 0] == 1 and ap["Q"][0, 0, 0] == 0 and ap["J"][0, 0] == 0.0
    for bud in (O.solve_budget_batch(x[None, :], P[None, :], 4, 1.0, 30),
                O.solve_approx_budget_batch(x[None, :], P[None, :], 4, 1.0, 30, refine=2)):
        assert bud["status"][0] == 0 and bud["m1"][0] == 1 and bud["Q1"][0, 0] == 0
        assert bud["mse1"][0] == 0.0 and bud["H1"][0] == 0.0


def test_two_values_allowed_keeps_the_ends():
    """s = 2: min X and max X must be in Q, so Q = {P_0, P_{p-1}} at any lambda,
    for the exact solver and the approximation."""
    X, P = _distinct_rows(75, 2, 300, 20)
    lam = np.array([[0.0, 0.3], [0.01, 1.0]])
    ex = O.solve_batch(X, P, 2, lam)
    assert np.all(ex["status"] == 0) and np.all(ex["m"] == 2)
    assert np.all(ex["Q"][..., 0] == 0) and np.all(ex["Q"][..., 1] == 19)
    for li in range(2):
        ap = O.solve_approx_batch(X, P, 2, lam[:, li])
        assert np.all(ap["status"] == 0) and np.all(ap["m"] == 2)
        assert np.all(ap["Q"][:, 0, 0] == 0) and np.all(ap["Q"][:, 0, 1] == 19)


# -- batch layouts and padding ---------------------------------------------------------

def _distinct_rows(seed, n, d, p):
    # rows on different scales, so that their grids and codes differ
    X = np.stack([_rows(seed + r, 1, d, scale=0.5 + r)[0] for r in range(n)])
    P, st = O.grid_batch(X, p)
    assert np.all(st == 0)
    return X, P


def _assert_padded(Q, m):
    Q = np.asarray(Q)
    for idx in np.ndindex(*m.shape):
        q = Q[idx]
        assert np.all(q[m[idx]:] == -1), (idx, q, m[idx])
        assert np.all(np.diff(q[:m[idx]]) > 0)


def test_solve_batch_rows_and_lambdas_match_single_calls():
    X, P = _distinct_rows(10, 3, 500, 24)
    lam = np.array([[0.001, 0.05], [0.01, 0.2], [0.003, 0.5]])
    s = 6
    out = O.solve_batch(X, P, s, lam)
    _assert_padded(out["Q"], out["m"])
    for r in range(3):
        for li in range(2):
            one = O.solve_batch(X[r:r + 1], P[r:r + 1], s, lam[r:r + 1, li:li + 1])
            assert out["m"][r, li] == one["m"][0, 0]
            np.testing.assert_array_equal(out["Q"][r, li], one["Q"][0, 0])
            assert out["J"][r, li] == one["J"][0, 0]
    # the rows do differ, so a row offset slip cannot pass by accident
    assert not np.array_equal(out["Q"][0, 0], out["Q"][2, 0]) or out["J"][0, 0] != out["J"][2, 0]


def test_budget_batch_rows_match_single_calls():
    X, P = _distinct_rows(20, 3, 400, 20)
    s = 5
    out = O.solve_budget_batch(X, P, s, 1.7, 30)
    _assert_padded(out["Q1"], out["m1"])
    _assert_padded(out["Q2"], out["m2"])
    for r in range(3):
        one = O.solve_budget_batch(X[r:r + 1], P[r:r + 1], s, 1.7, 30)
        for k in ("Q1", "Q2"):
            np.testing.assert_array_equal(out[k][r], one[k][0])
        for k in ("m1", "m2", "theta", "H1", "H2", "mse1", "mse2"):
            assert out[k][r] == one[k][0], k


def test_encode_batch_rows_match_single_row_encoding():
    """Row r of a batch is coded with Philox counter row r: the same as
    encode_row(…, row=r) on that row alone, with that row's own code."""
    X, P = _distinct_rows(30, 3, 301, 16)
    s = 5
    Q1 = np.array([[0, 3, 8, 15, -1], [0, 6, 15, -1, -1], [0, 1, 2, 7, 15]], np.int32)
    m1 = np.array([4, 3, 5], np.int32)
    Q2 = np.array([[0, 15, -1, -1, -1], [0, 2, 4, 9, 15], [0, 5, 15, -1, -1]], np.int32)
    m2 = np.array([2, 5, 3], np.int32)
    th = np.array([0.3, 0.7, 0.5])
    idx, hist, st = O.encode_batch(X, P, Q1, m1, s, 11, Q2, m2, th)
    assert np.all(st == 0)
    for r in range(3):
        i1, h1 = O.encode_row(X[r], P[r], Q1[r], m1[r], s, 11, r, Q2[r], m2[r], th[r])
        np.testing.assert_array_equal(idx[r], i1)
        np.testing.assert_array_equal(hist[r], h1)


def test_dequantize_batch_uses_each_rows_codes():
    """theta = 1 codes every entry on Q1 and theta = 0 on Q2, so X^ is
    P[Q_part[idx]] with no randomness; the rows have different codes."""
    X, P = _distinct_rows(40, 3, 97, 12)
    s = 4
    Q1 = np.array([[0, 5, 11, -1], [0, 2, 7, 11], [0, 11, -1, -1]], np.int32)
    m1 = np.array([3, 4, 2], np.int32)
    Q2 = np.array([[0, 3, 6, 11], [0, 11, -1, -1], [0, 4, 11, -1]], np.int32)
    m2 = np.array([4, 2, 3], np.int32)
    rng = np.random.default_rng(41)
    for th_val, Q, m in ((1.0, Q1, m1), (0.0, Q2, m2)):
        idx = np.stack([rng.integers(0, m[r], 97) for r in range(3)]).astype(np.uint8)
        th = np.full(3, th_val)
        Xh, st = O.dequantize_batch(idx, P, Q1, m1, s, 5, Q2, m2, th)
        assert np.all(st == 0)
        for r in range(3):
            want = P[r][Q[r][idx[r].astype(np.int64)]].astype(np.float32)
            np.testing.assert_array_equal(Xh[r], want)


def test_approx_batch_rows_match_single_calls():
    X, P = _distinct_rows(50, 3, 600, 32)
    s = 6
    lam = np.array([0.02, 0.05, 0.1])
    for refine in (0, 4):
        out = O.solve_approx_batch(X, P, s, lam, refine=refine)
        _assert_padded(out["Q"], out["m"])
        for r in range(3):
            one = O.solve_approx_batch(X[r:r + 1], P[r:r + 1], s, lam[r:r + 1], refine=refine)
            np.testing.assert_array_equal(out["Q"][r], one["Q"][0])
            assert out["J"][r, 0] == one["J"][0, 0]


def test_approx_batch_with_several_lambdas_per_row():
    X, P = _distinct_rows(55, 2, 400, 24)
    lam = np.array([[0.01, 0.1], [0.03, 0.3]])
    out = O.solve_approx_batch(X, P, 6, lam)
    _assert_padded(out["Q"], out["m"])
    for r in range(2):
        for li in range(2):
            one = O.solve_approx_batch(X[r:r + 1], P[r:r + 1], 6, lam[r:r + 1, li])
            np.testing.assert_array_equal(out["Q"][r, li], one["Q"][0, 0])
            assert out["J"][r, li] == one["J"][0, 0]


def test_approx_bad_arguments_status():
    X, P = _distinct_rows(56, 1, 100, 8)
    out = O.solve_approx_batch(X, P, 1, np.array([0.1]))
    assert out["status"][0, 0] == ERR_ARG


def test_encode_theta_at_the_ends_uses_one_code():
    """theta = 1 puts every entry on Q1 and theta = 0 every entry on Q2: the
    other part's histogram stays empty and the indices are those of the
    one-code encoding."""
    X, P = _distinct_rows(57, 2, 333, 16)
    s = 4
    Q1 = np.array([[0, 5, 15, -1], [0, 7, 11, 15]], np.int32)
    m1 = np.array([3, 4], np.int32)
    Q2 = np.array([[0, 3, 9, 15], [0, 15, -1, -1]], np.int32)
    m2 = np.array([4, 2], np.int32)
    i1, h1, st1 = O.encode_batch(X, P, Q1, m1, s, 4)
    i2, h2, st2 = O.encode_batch(X, P, Q2, m2, s, 4)
    ia, ha, sta = O.encode_batch(X, P, Q1, m1, s, 4, Q2, m2, np.ones(2))
    ib, hb, stb = O.encode_batch(X, P, Q1, m1, s, 4, Q2, m2, np.zeros(2))
    assert np.all(st1 == 0) and np.all(st2 == 0) and np.all(sta == 0) and np.all(stb == 0)
    np.testing.assert_array_equal(ia, i1)
    np.testing.assert_array_equal(ha[:, 0], h1[:, 0])
    assert np.all(ha[:, 1] == 0)
    np.testing.assert_array_equal(ib, i2)
    np.testing.assert_array_equal(hb[:, 1], h2[:, 0])
    assert np.all(hb[:, 0] == 0)


def test_entropy_of_an_empty_histogram_is_zero():
    assert O.entropy(np.zeros((2, 5), np.int64), 5) == 0.0


def test_approx_budget_outputs_are_valid_codes():
    """Both codes of the approximate budget solve are increasing index lists
    from P_0 to P_{p-1} (min X and max X lie in Q), padded with -1, and the
    reported H and MSE are those of the code they belong to."""
    X, P = _distinct_rows(60, 2, 800, 24)
    s = 6
    out = O.solve_approx_budget_batch(X, P, s, 1.5, 30, refine=4)
    assert np.all(out["status"] == 0)
    _assert_padded(out["Q1"], out["m1"])
    _assert_padded(out["Q2"], out["m2"])
    for r in range(2):
        for q, m, H, mse in ((out["Q1"][r], out["m1"][r], out["H1"][r], out["mse1"][r]),
                             (out["Q2"][r], out["m2"][r], out["H2"][r], out["mse2"][r])):
            assert m >= 2 and q[0] == 0 and q[m - 1] == P.shape[1] - 1
            mse_e, H_e, _ = O.eval_raw(X[r], P[r][q[:m]])
            assert mse == pytest.approx(mse_e, rel=1e-9, abs=1e-15)
            assert H == pytest.approx(H_e, rel=1e-9, abs=1e-15)


def test_two_value_alphabet_is_solved():
    """p = 2: the only code is {P_0, P_1}; every solver accepts it."""
    X = _rows(70, 2, 50)
    P, st = O.grid_batch(X, 2)
    assert np.all(st == 0)
    ex = O.solve_batch(X, P, 4, np.array([[0.1], [0.1]]))
    ap = O.solve_approx_batch(X, P, 4, np.array([0.1, 0.1]))
    for out in (ex, ap):
        assert np.all(out["status"] == 0)
        assert np.all(out["m"] == 2)
        np.testing.assert_array_equal(out["Q"][:, 0, :2], [[0, 1], [0, 1]])
        assert np.all(out["Q"][:, 0, 2:] == -1)


# -- entropy coder ---------------------------------------------------------------------

@pytest.mark.parametrize("d,segs", [(16382, 1), (16383, 1), (16384, 1), (16385, 2), (32767, 2), (32768, 2),
                                    (32769, 3)])
def test_rans_segment_count(d, segs):
    """Segments of 16,384 entries: ceil(d / 16384) per row, round trip intact."""
    rng = np.random.default_rng(d)
    idx = rng.integers(0, 4, (1, d)).astype(np.uint8)
    hist = np.zeros((1, 2, 4), np.int64)
    hist[0, 0] = np.bincount(idx[0], minlength=4)
    words, seg_len, st = O.rans_encode(idx, hist, seed=3)
    assert st[0] == 0
    assert words.shape[1] == segs and seg_len.shape[1] == segs
    back, st2 = O.rans_decode(words, seg_len, d, hist, seed=3)
    assert st2[0] == 0
    np.testing.assert_array_equal(back, idx)


def test_rans_two_full_segments_closed_form():
    """Two full segments (2 x 16384 entries) of the uniform two-symbol model,
    every entry symbol 0: each state doubles per symbol, so each segment holds
    512 steps = 32 zero words per state and the final state 2^(16 + 512 mod 16)
    = 2^16 as the (low, high) pair (0, 1); nothing of one segment leaks into
    the other."""
    d = 2 * 16384
    idx = np.zeros((1, d), np.uint8)
    hist = np.zeros((1, 2, 2), np.int64)
    hist[0, 0] = [1, 1]
    words, seg_len, st = O.rans_encode(idx, hist, 1)
    assert st[0] == 0
    for g in range(2):
        assert seg_len[0, g] == 32 * 32 + 64
        w = words[0, g, :seg_len[0, g]]
        assert np.all(w[:32 * 32] == 0)
        assert np.all(w[32 * 32::2] == 0) and np.all(w[32 * 32 + 1::2] == 1)


def test_rans_segment_capacity():
    """A state in [2^16, 2^32) with M = 2^15 sheds at most one 16-bit word per
    symbol, so a segment of 512 steps x 32 states needs at most 16384 words,
    plus two per state for the final states: 16448."""
    idx = np.zeros((1, 10), np.uint8)
    hist = np.zeros((1, 2, 2), np.int64)
    hist[0, 0] = [1, 1]
    words, _, _ = O.rans_encode(idx, hist, 1)
    assert words.shape[2] == 32 * 512 + 2 * 32


def test_rans_parts_are_the_encoders():
    """Time-shared row: Q1 has 6 values, Q2 only 2, so an index >= 2 can only
    come from part 1 (Q1). The coder recomputes each entry's part from seed and
    theta; with the encoder's rule every index has a frequency in its part's
    model and the row codes and decodes; with another seed, entries with an
    index >= 2 fall on Q2's model and the row is rejected."""
    rng = np.random.default_rng(80)
    x = rng.standard_normal(5000).astype(np.float32)
    P, _ = O.uniform_grid(x, 16)
    s = 6
    Q1 = np.array([0, 3, 6, 9, 12, 15], np.int32)
    Q2 = np.array([0, 15, -1, -1, -1, -1], np.int32)
    idx, hist = O.encode_row(x, P, Q1, 6, s, 21, 0, Q2, 2, 0.5)
    th = np.array([0.5])
    words, seg_len, st = O.rans_encode(idx[None, :], hist[None], 21, theta=th, two_codes=True)
    assert st[0] == 0
    back, st2 = O.rans_decode(words, seg_len, x.size, hist[None], 21, theta=th, two_codes=True)
    assert st2[0] == 0
    np.testing.assert_array_equal(back[0], idx)
    _, _, st3 = O.rans_encode(idx[None, :], hist[None], 22, theta=th, two_codes=True)
    assert st3[0] == ERR_ARG


def test_rans_malformed_stream_is_an_argument_error():
    """A segment length too short to hold the final states is rejected with
    ECASQ_ERR_ARG, as the header states for a malformed stream."""
    idx = np.zeros((1, 100), np.uint8)
    hist = np.zeros((1, 2, 2), np.int64)
    hist[0, 0] = [1, 1]
    words, seg_len, st = O.rans_encode(idx, hist, 1)
    assert st[0] == 0
    bad = seg_len.copy()
    bad[0, 0] = 2 * 32 - 1
    _, st2 = O.rans_decode(words, bad, 100, hist, 1)
    assert st2[0] == ERR_ARG


def test_rans_model_shortfall_goes_to_lowest_index_of_tied_counts():
    """M = 2^15, counts (5, 5, 1): floor(5M/11) = 14894 twice and
    floor(M/11) = 2978 sum to M - 2; the shortfall of 2 goes to the most
    frequent symbol, the lower index of the tie."""
    f, cum = O.rans_model(np.array([5, 5, 1]))
    np.testing.assert_array_equal(f, [14896, 14894, 2978])
    np.testing.assert_array_equal(cum, [0, 14896, 29790, 32768])


def test_rans_model_excess_comes_from_lowest_index_of_tied_frequencies():
    """Counts (10^5, 10^5, 1, 1, 1), n = 200003 > 3M: the three singletons
    round to 0 and are raised to 1; with floor(10^5 M / n) = 16383 twice the
    sum is M + 1, and the excess of 1 is taken from the largest frequency,
    the lower index of the tie."""
    f, _ = O.rans_model(np.array([100000, 100000, 1, 1, 1]))
    np.testing.assert_array_equal(f, [16382, 16383, 1, 1, 1])
    assert int(f.sum()) == 1 << 15


def test_rans_model_of_an_empty_part_is_empty():
    """A part with no entries (theta = 0 or 1 leaves one empty) gets no
    frequencies at all: nothing can be coded on it."""
    f, cum = O.rans_model(np.zeros(5, np.int64))
    assert np.all(f == 0) and np.all(cum == 0)


def test_rans_rejects_an_index_beyond_the_alphabet():
    """An index equal to s (one past the last symbol) is an error, even where
    the next part's model would give that position a nonzero frequency (two
    codes, theta = 1: every entry on part 0, part 1's model built anyway)."""
    idx = np.array([[0, 1, 2, 3, 1, 0]], np.uint8)
    hist = np.zeros((1, 2, 3), np.int64)
    hist[0, 0] = [2, 2, 1]  # s = 3: symbol 3 does not exist
    hist[0, 1] = [1, 1, 1]
    _, _, st = O.rans_encode(idx, hist, seed=1, theta=np.array([1.0]), two_codes=True)
    assert st[0] == ERR_ARG
    ok = idx.copy()
    ok[0, 3] = 2
    hist[0, 0] = [2, 2, 2]
    _, _, st = O.rans_encode(ok, hist, seed=1, theta=np.array([1.0]), two_codes=True)
    assert st[0] == 0


# -- refinement: the order of the value classes ---------------------------------------

def _one_iteration(V, R, L, d, lam, Q, cls_of):
    """One refinement iteration composed from the separately pinned local cost
    and binary search: classes 0, 1, 2 in turn; a value moves to the search's
    index only on a strict decrease of its local cost."""
    Q = np.array(Q, np.int32)
    for cls in range(3):
        for t in range(1, Q.size - 1):
            if cls_of(t) != cls:
                continue
            c = O.refine_point(V, R, L, d, lam, Q, t)
            if c != Q[t] and O.refine_local(V, R, L, d, lam, Q, t, c) < O.refine_local(V, R, L, d, lam, Q, t,
                                                                                           int(Q[t])):
                Q[t] = c
    return Q


def test_refinement_search_stays_inside_the_open_interval():
    """A value searches (c_{t-1}, c_{t+1}) only: it never lands on a neighbour,
    also where the local cost still falls at the interval's right end (cases
    of that kind are required to occur, so the check has teeth)."""
    right_end = 0
    for seed in range(200):
        rng = np.random.default_rng(1000 + seed)
        x = (rng.standard_normal(400) * rng.uniform(0.5, 2.0)).astype(np.float32)
        P, _ = O.uniform_grid(x, 32)
        cnt, A, B, _ = O.bucket(x, P)
        V, R, L = O.tables(cnt, A, B, P)
        lam = float(rng.uniform(0.01, 0.3)) * float(np.var(x.astype(np.float64)))
        Q, _ = O.approx_dp(V, R, L, 8, x.size, lam)
        Q = np.asarray(Q, np.int32)
        for t in range(1, Q.size - 1):
            lo, hi = int(Q[t - 1]) + 1, int(Q[t + 1]) - 1
            if hi - lo < 1:
                continue
            c = O.refine_point(V, R, L, x.size, lam, Q, t)
            assert lo <= c <= hi, (seed, t, c, lo, hi)
            f = [O.refine_local(V, R, L, x.size, lam, Q, t, k) for k in (hi - 1, hi)]
            if f[1] < f[0]:
                right_end += 1
    assert right_end >= 3


def test_refinement_classes_run_in_position_order():
    """Q_c = {t : (t - 1) mod 3 = c} over the interior positions 1 .. m-2, so Q0
    holds position 1; one iteration runs Q0, Q1, Q2. Checked on cases where
    the other assignment (t mod 3) ends elsewhere after one iteration."""
    found = 0
    for seed in range(200):
        rng = np.random.default_rng(seed)
        x = (rng.standard_normal(600) * rng.uniform(0.5, 2.0)).astype(np.float32)
        P, _ = O.uniform_grid(x, 40)
        cnt, A, B, _ = O.bucket(x, P)
        V, R, L = O.tables(cnt, A, B, P)
        lam = float(rng.uniform(0.01, 0.2)) * float(np.var(x.astype(np.float64)))
        Qa, _ = O.approx_dp(V, R, L, 10, x.size, lam)
        mine = _one_iteration(V, R, L, x.size, lam, Qa, lambda t: (t - 1) % 3)
        other = _one_iteration(V, R, L, x.size, lam, Qa, lambda t: t % 3)
        if np.array_equal(mine, other):
            continue
        Qr, _, it = O.refine(V, R, L, x.size, lam, Qa, 1)
        assert it == 1
        np.testing.assert_array_equal(Qr, mine)
        found += 1
        if found == 3:
            break
    assert found == 3


# -- accuracy of the oracle's sums and the BF16 alphabet's statuses ---------------------

def test_bucket_sums_are_compensated():
    """A_k and B_k are sums of the fp64 terms y = x - P_k and y^2 over about
    66,000 entries per bucket. Compensated summation keeps them within
    3 eps sum|y| of the correctly rounded sum (math.fsum of the same terms);
    plain summation drifts by about sqrt(n) eps, far beyond that bound."""
    import math
    rng = np.random.default_rng(90)
    x = rng.standard_normal(200000).astype(np.float32)
    P, st = O.uniform_grid(x, 4)
    assert st == 0
    cnt, A, B, st = O.bucket(x, P)
    assert st == 0
    xd = x.astype(np.float64)
    k = np.clip(np.searchsorted(P[:-1], xd, side="right") - 1, 0, P.size - 2)
    eps = np.finfo(np.float64).eps
    for b in range(P.size - 1):
        y = xd[k == b] - P[b]
        assert cnt[b] == y.size
        for got, terms in ((A[b], y), (B[b], y * y)):
            exact = math.fsum(terms.tolist())
            bound = 3 * eps * float(np.abs(terms).sum())
            assert abs(got - exact) <= bound, (b, got, exact, bound)


def test_bf16_alphabet_status_values():
    """A non-finite entry, and an entry above the largest finite BF16 value
    (so that no BF16 value >= max X exists), give ECASQ_ERR_RANGE."""
    P = np.zeros(16)
    for bad in (np.float32("nan"), np.float32(np.finfo(np.float32).max)):
        x = np.array([0.5, bad, -1.0], np.float32)
        assert O.lib().eo_bf16_alphabet(x, x.size, P, P.size) == ERR_RANGE
    x = np.array([0.5, -1.0], np.float32)
    assert O.lib().eo_bf16_alphabet(x, x.size, P, P.size) > 0


def test_budget_bisection_runs_the_given_number_of_steps():
    """The lambda bracket starts as [0, (P_{p-1} - P_0)^2] and halves once per
    step, so after `steps` steps lambda_hi - lambda_lo is that width x
    2^-steps (up to the rounding of the midpoints, about 2^-23 relative), for
    the exact and the approximate budget drivers, wherever the budget binds."""
    X, P = _distinct_rows(95, 3, 700, 24)
    for steps in (12, 30):
        for out in (O.solve_budget_batch(X, P, 6, 1.6, steps),
                    O.solve_approx_budget_batch(X, P, 6, 1.6, steps, refine=0)):
            for r in range(3):
                assert out["status"][r] == 0 and 0.0 < out["theta"][r] < 1.0
                width = (P[r, -1] - P[r, 0]) ** 2 * 2.0 ** -steps
                assert out["lam_hi"][r] - out["lam_lo"][r] == pytest.approx(width, rel=1e-5)


def test_rans_truncated_stream_is_an_argument_error():
    """A segment length that drops renormalisation words leaves the decoder
    short of words: ECASQ_ERR_ARG."""
    d = 16384
    idx = np.zeros((1, d), np.uint8)
    hist = np.zeros((1, 2, 2), np.int64)
    hist[0, 0] = [1, 1]
    words, seg_len, st = O.rans_encode(idx, hist, 1)
    assert st[0] == 0 and seg_len[0, 0] == 32 * 32 + 64
    bad = seg_len.copy()
    bad[0, 0] = 64 + 100
    _, st2 = O.rans_decode(words, bad, d, hist, 1)
    assert st2[0] == ERR_ARG
