"""Pins of the fp64 oracle to things other than itself (CPU only).

Definitions: "Entropy-Constrained Adaptive Stochastic Quantization (ECASQ)"
(gist.science/pt/paper/2608.18147): §1 problem (unbiased stochastic rounding,
MSE, H(X^) <= b, |Q| <= s), §2.1 Lagrangian relaxation and two-way
time-sharing, §2.2 pair-state DP, §2.3 bound H(X^) <= H(I,B) <= H(X^) + 1.

The pins: hand-worked closed forms (tests/golden), two independent evaluations
of the objective (raw entries vs bucket tables), brute force over every code on
tiny inputs, the textbook MSE-only DP at lambda = 0, invariants, reflection and
scaling symmetries, lambda-sweep monotonicity, the time-sharing identity, and a
library Philox (numpy) for the generator's round structure.
"""
import itertools
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from entropy_constrained_unbiased_b200 import workloads as W

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _expr(s):
    return float(eval(s, {"__builtins__": {}}, {"log2": math.log2}))


def _load_cases():
    cases, cur = [], None
    for line in open(os.path.join(GOLD, "worked_examples.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        if line.startswith("case "):
            cur = {"name": line.split()[1]}
            cases.append(cur)
            continue
        k, v = (t.strip() for t in line.split("=", 1))
        cur[k] = v
    return cases


@pytest.mark.parametrize("case", _load_cases(), ids=lambda c: c["name"])
def test_worked_examples_raw_and_tables(O, case):
    x = np.array([float(Fraction(t)) for t in case["x"].split()], np.float32)
    q = np.array([float(Fraction(t)) for t in case["q"].split()])
    mse_ref = _expr(case["mse"])
    H_ref = _expr(case["H"])
    mu_ref = np.array([_expr(t) for t in case["mu"].split()])
    mse, H, mu = O.eval_raw(x, q)
    assert mse == pytest.approx(mse_ref, rel=1e-14, abs=1e-15)
    assert H == pytest.approx(H_ref, rel=1e-14, abs=1e-15)
    np.testing.assert_allclose(mu, mu_ref, rtol=1e-14, atol=1e-14)
    # Same objective through buckets + interval tables on P = the code itself.
    cnt, A, B, st = O.bucket(x, q)
    assert st == 0
    V, R, L = O.tables(cnt, A, B, q)
    mse_t, H_t, mu_t = O.eval_tables(V, R, L, x.size, np.arange(q.size))
    assert mse_t == pytest.approx(mse_ref, rel=1e-14, abs=1e-15)
    assert H_t == pytest.approx(H_ref, rel=1e-14, abs=1e-15)
    np.testing.assert_allclose(mu_t, mu_ref, rtol=1e-14, atol=1e-14)


def _dp_cases():
    out = []
    for line in open(os.path.join(GOLD, "dp_worked_examples.txt")):
        line = line.strip()
        if line.startswith("dp "):
            parts = line.split()
            lam = float(Fraction(parts[1]))
            rest = line.split(None, 2)[2]
            qs, jexpr = rest.rsplit("  ", 1) if "  " in rest else (None, None)
            out.append((lam, [int(t) for t in qs.split()], _expr(jexpr.strip())))
    return out


DP_X = np.array([0, 0.5, 0.5, 1], np.float32)
DP_P = np.array([0.0, 0.5, 1.0])


@pytest.mark.parametrize("lam,Q_ref,J_ref", _dp_cases())
def test_dp_worked_example(O, lam, Q_ref, J_ref):
    r = O.solve_batch(DP_X[None], DP_P[None], 3, np.array([[lam]]))
    m = r["m"][0, 0]
    assert list(r["Q"][0, 0, :m]) == Q_ref
    assert r["J"][0, 0] == pytest.approx(J_ref, rel=1e-15, abs=1e-15)


def test_budget_worked_example(O):
    line = [l for l in open(os.path.join(GOLD, "dp_worked_examples.txt")) if l.startswith("budget ")][0]
    kv = dict(t.split("=") for t in line.split()[1:])
    r = O.solve_budget_batch(DP_X[None], DP_P[None], 3, float(Fraction(kv["b"])), 30)
    assert r["status"][0] == 0
    assert list(r["Q1"][0, : r["m1"][0]]) == [int(t) for t in kv["Q1"].split(",")]
    assert list(r["Q2"][0, : r["m2"][0]]) == [int(t) for t in kv["Q2"].split(",")]
    for k in ("H1", "H2", "mse1", "mse2", "theta", "lam_hi"):
        ref = float(Fraction(kv[k]))
        key = k
        assert r[key][0] == pytest.approx(ref, rel=1e-14, abs=1e-15), k


# -- random tiny instances -----------------------------------------------------

def _nonuniform_P(rng, x, p):
    lo, hi = float(x.min()), float(x.max())
    inner = np.sort(rng.uniform(lo, hi, size=p - 2))
    P = np.concatenate([[lo], inner, [hi]])
    assert np.all(np.diff(P) > 0)
    return P


def _tiny(seed, d, p, uniform):
    rng = np.random.default_rng([7, seed])
    dist = ["normal", "laplace", "student_t", "lognormal", "outlier"][seed % 5]
    x = W.draw(dist, rng, 1, d)[0]
    if uniform:
        P, st = None, 0
    else:
        P = _nonuniform_P(rng, x, p)
    return x, P, dist


@pytest.mark.parametrize("seed", range(10))
def test_tables_match_raw_evaluation(O, seed):
    """Bucket tables and the raw O(d) pass give the same objective for random codes."""
    rng = np.random.default_rng([11, seed])
    x, P, _ = _tiny(seed, 300, 24, uniform=bool(seed % 2))
    if P is None:
        P, st = O.uniform_grid(x, 24)
        assert st == 0
    cnt, A, B, st = O.bucket(x, P)
    assert st == 0 and cnt.sum() == x.size
    V, R, L = O.tables(cnt, A, B, P)
    assert np.all(V >= 0)
    for _ in range(20):
        k = rng.integers(0, P.size - 2 + 1)
        inner = np.sort(rng.choice(np.arange(1, P.size - 1), size=k, replace=False))
        Q = np.concatenate([[0], inner, [P.size - 1]]).astype(np.int32)
        mse_t, H_t, mu_t = O.eval_tables(V, R, L, x.size, Q)
        mse_r, H_r, mu_r = O.eval_raw(x, P[Q])
        assert mse_t == pytest.approx(mse_r, rel=1e-11, abs=1e-14)
        assert H_t == pytest.approx(H_r, rel=1e-11, abs=1e-14)
        np.testing.assert_allclose(mu_t, mu_r, rtol=1e-10, atol=1e-9)
        assert mu_t.sum() == pytest.approx(x.size, rel=1e-12)


def _brute(O, x, P, s, lam):
    p = P.size
    best = (math.inf, None)
    for k in range(0, min(s, p) - 1):
        for inner in itertools.combinations(range(1, p - 1), k):
            Q = [0, *inner, p - 1]
            mse, H, _ = O.eval_raw(x, P[Q])
            J = mse + lam * H
            if J < best[0]:
                best = (J, Q)
    return best


@pytest.mark.parametrize("seed", range(12))
@pytest.mark.parametrize("lam", [0.0, 1e-3, 1e-1, 10.0])
def test_dp_equals_brute_force(O, seed, lam):
    """The DP's optimum equals exhaustive search over every code (p <= 12, s <= 4;
    p = 16, s = 6), uniform and random non-uniform P."""
    p, s = (12, 4) if seed < 8 else (16, 6)
    x, P, _ = _tiny(seed, 64 + 13 * seed, p, uniform=(seed % 3 == 0))
    if P is None:
        P, _ = O.uniform_grid(x, p)
    scale = float(np.var(x.astype(np.float64))) if lam > 0 else 1.0
    lam_eff = lam * scale  # put MSE and lambda*H on comparable scales
    J_bf, Q_bf = _brute(O, x, P, s, lam_eff)
    r = O.solve_batch(x[None], P[None], s, np.array([[lam_eff]]))
    m = r["m"][0, 0]
    Q = r["Q"][0, 0, :m]
    assert Q[0] == 0 and Q[-1] == p - 1 and m <= s and np.all(np.diff(Q) > 0)
    mse, H, _ = O.eval_raw(x, P[Q])
    assert mse + lam_eff * H == pytest.approx(J_bf, rel=1e-12, abs=1e-15)
    assert r["J"][0, 0] == pytest.approx(J_bf, rel=1e-12, abs=1e-15)


def _asq_textbook(V, p, s, d):
    """MSE-only adaptive stochastic quantization (lambda = 0): the separable 2-D DP
    G_i(c) = min_{a<c} G_{i-1}(a) + V(a, c), G_1(0) = 0, answer min_i G_i(p-1)."""
    INF = math.inf
    G = [[INF] * p for _ in range(s + 1)]
    G[1][0] = 0.0
    for i in range(2, s + 1):
        for c in range(1, p):
            G[i][c] = min(G[i - 1][a] + V[a, c] for a in range(c) if G[i - 1][a] < INF) if any(
                G[i - 1][a] < INF for a in range(c)) else INF
    return min(G[i][p - 1] for i in range(2, s + 1)) / d


@pytest.mark.parametrize("seed", range(6))
def test_lambda_zero_is_textbook_asq(O, seed):
    rng = np.random.default_rng([13, seed])
    x = W.draw(["normal", "laplace", "lognormal"][seed % 3], rng, 1, 400)[0]
    p, s = 40, 6
    P, _ = O.uniform_grid(x, p)
    cnt, A, B, _ = O.bucket(x, P)
    V, R, L = O.tables(cnt, A, B, P)
    ref = _asq_textbook(V, p, s, x.size)
    r = O.solve_batch(x[None], P[None], s, np.array([[0.0]]))
    assert r["mse"][0, 0] == pytest.approx(ref, rel=1e-12)
    assert r["J"][0, 0] == pytest.approx(ref, rel=1e-12)
    # More values never raise the MSE: at lambda = 0 all s slots are used unless idle.
    assert r["m"][0, 0] == s


@pytest.mark.parametrize("seed", range(6))
def test_invariants(O, seed):
    rng = np.random.default_rng([17, seed])
    x = W.draw(["normal", "student_t", "outlier"][seed % 3], rng, 1, 2000)[0]
    p, s = 48, 8
    P, _ = O.uniform_grid(x, p)
    assert P[0] == float(x.min()) and P[-1] == float(x.max())
    cnt, A, B, _ = O.bucket(x, P)
    V, R, L = O.tables(cnt, A, B, P)
    v = float(np.var(x.astype(np.float64)))
    for lam in (0.0, 0.01 * v, v):
        Q, J = O.dp(V, R, L, s, x.size, lam)
        m = Q.size
        # min X and max X are code values (unbiasedness at the ends)
        assert P[Q[0]] == x.min() and P[Q[-1]] == x.max()
        mse, H, mu = O.eval_tables(V, R, L, x.size, Q)
        assert mu.sum() == pytest.approx(x.size, rel=1e-12)
        assert H <= math.log2(m) + 1e-12
        # H(X^) <= H(I,B) <= H(X^) + 1 (§2.3), H(I,B) from the interval masses
        hib = 0.0
        for t in range(m - 1):
            for mass in (L[Q[t], Q[t + 1]], R[Q[t], Q[t + 1]]):
                if mass > 0:
                    hib -= mass / x.size * math.log2(mass / x.size)
        assert H <= hib + 1e-12 <= H + 1 + 2e-12
        assert J == pytest.approx(mse + lam * H, rel=1e-12, abs=1e-15)


@pytest.mark.parametrize("seed", range(4))
def test_reflection_and_scaling(O, seed):
    rng = np.random.default_rng([19, seed])
    x = W.draw(["lognormal", "student_t", "laplace", "outlier"][seed], rng, 1, 500)[0]
    p, s = 32, 6
    P, _ = O.uniform_grid(x, p)
    lam = 0.05 * float(np.var(x.astype(np.float64)))
    r = O.solve_batch(x[None], P[None], s, np.array([[lam]]))
    m = r["m"][0, 0]
    Q = r["Q"][0, 0, :m]
    J = r["J"][0, 0]
    # reflection: x -> -x, P -> -reverse(P): mirrored code, same objective
    rr = O.solve_batch((-x)[None], (-P[::-1])[None].copy(), s, np.array([[lam]]))
    assert rr["J"][0, 0] == pytest.approx(J, rel=1e-11)
    mm = rr["m"][0, 0]
    Qr = rr["Q"][0, 0, :mm]
    Jr_of_mirror = O.eval_raw(x, P[(p - 1 - Qr)[::-1]])
    assert Jr_of_mirror[0] + lam * Jr_of_mirror[1] == pytest.approx(J, rel=1e-11)
    # scaling by c = 4 (exact in fp32): P -> cP, lambda -> c^2 lambda, J -> c^2 J
    c = 4.0
    rs = O.solve_batch((c * x)[None], (c * P)[None], s, np.array([[c * c * lam]]))
    assert rs["J"][0, 0] == pytest.approx(c * c * J, rel=1e-11)
    assert list(rs["Q"][0, 0, : rs["m"][0, 0]]) == list(Q)


def test_lambda_sweep_monotone(O):
    w = W.WORKLOADS["sweep"]
    x = W.make_inputs(w, rows=1)[:, :2048]
    P, _ = O.grid_batch(x, 48)
    lam = w.lambdas()[:1]
    r = O.solve_batch(x, P, 8, lam)
    mse, H = r["mse"][0], r["H"][0]
    assert np.all(np.diff(mse) >= -1e-12 * mse[1:])
    assert np.all(np.diff(H) <= 1e-12)


@pytest.mark.parametrize("seed", range(4))
def test_time_sharing_identity(O, seed):
    rng = np.random.default_rng([23, seed])
    x = W.draw(["student_t", "normal", "grad", "laplace"][seed], rng, 1, 1500)
    P, _ = O.grid_batch(x, 40)
    for b in (1.5, 2.0, 2.7):
        r = O.solve_budget_batch(x, P, 10, b, 30)
        assert r["status"][0] == 0
        th, H1, H2 = r["theta"][0], r["H1"][0], r["H2"][0]
        assert H2 <= b + 1e-15
        if th > 0:
            assert H1 > b
            assert th * H1 + (1 - th) * H2 == pytest.approx(b, rel=1e-12)
        # both codes are Lagrangian optima at their lambdas
        for key_q, key_m, lam in (("Q1", "m1", r["lam_lo"][0]), ("Q2", "m2", r["lam_hi"][0])):
            m = r[key_m][0]
            Q = r[key_q][0, :m]
            mse, H, _ = O.eval_raw(x[0], P[0][Q])
            ref = O.solve_batch(x, P, 10, np.array([[lam]]))
            assert mse + lam * H == pytest.approx(ref["J"][0, 0], rel=1e-11)


# -- Philox ------------------------------------------------------------------

@pytest.mark.parametrize("ctr,key", [((0, 0, 0, 0), (0, 0)), ((5, 7, 11, 13), (0x1234, 0xFFFF)),
                                     ((2**64 - 1, 3, 2**63, 9), (2**64 - 1, 42))])
def test_philox_round_structure_matches_numpy(O, ctr, key):
    """numpy's Philox bit generator is Philox4x64-10; it increments its 256-bit
    counter once before its first block. The oracle's 4x64 instance of the
    same round structure must reproduce it."""
    bg = np.random.Philox(key=np.array(key, np.uint64), counter=np.array(ctr, np.uint64))
    got = bg.random_raw(4)
    c = list(ctr)
    c[0] = (c[0] + 1) % 2**64
    carry = c[0] == 0
    i = 1
    while carry and i < 4:
        c[i] = (c[i] + 1) % 2**64
        carry = c[i] == 0
        i += 1
    ours = O.philox4x64(np.array(c, np.uint64), np.array(key, np.uint64))
    np.testing.assert_array_equal(ours, got)


def _philox_kat():
    rows = []
    with open(os.path.join(GOLD, "philox4x32_kat.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            w = [int(t, 16) for t in line.split()]
            assert len(w) == 10
            rows.append((tuple(w[0:4]), tuple(w[4:6]), tuple(w[6:10])))
    return rows


@pytest.mark.parametrize("ctr,key,want", _philox_kat())
def test_philox4x32_known_answers(O, ctr, key, want):
    """The published Philox4x32-10 known-answer vectors (Random123, Salmon et
    al. SC'11): a wrong multiplier, Weyl increment, word order or round count
    changes every output word."""
    got = O.philox4x32(ctr, key)
    assert [int(v) for v in got] == list(want), [f"{int(v):08x}" for v in got]


def test_philox4x32_uniformity(O):
    """Chi-square over 2^14 blocks (65536 words) in 64 cells."""
    words = []
    for j in range(1 << 14):
        words.extend(O.philox4x32((j, 3, 0, 0), (1, 0)))
    w = np.array(words, np.uint64)
    cells = np.bincount((w >> 26).astype(np.int64), minlength=64)
    exp = w.size / 64
    chi2 = float(((cells - exp) ** 2 / exp).sum())
    assert chi2 < 63 + 6 * math.sqrt(2 * 63)  # ~ 6 sigma
    assert np.unique(w).size > w.size * 0.999


# -- encoder -----------------------------------------------------------------

def test_encode_unbiased_and_histogram(O):
    rng = np.random.default_rng([29, 0])
    x = W.draw("laplace", rng, 1, 256)
    P, _ = O.grid_batch(x, 32)
    r = O.solve_batch(x, P, 6, np.array([[0.02]]))
    m = int(r["m"][0, 0])
    Q = r["Q"][0, 0]
    qv = P[0][Q[:m]]
    _, _, mu = O.eval_raw(x[0], qv)
    acc = np.zeros(x.shape[1])
    counts = np.zeros(m)
    seeds = 400
    for sd in range(seeds):
        idx, hist, st = O.encode_batch(x, P, Q[None], r["m"][:, 0], 6, seed=sd)
        assert st[0] == 0 and idx.max() < m
        assert hist[0, 0].sum() == x.shape[1] and hist[0, 1].sum() == 0
        np.testing.assert_array_equal(np.bincount(idx[0], minlength=6), hist[0, 0])
        acc += qv[idx[0]]
        counts += hist[0, 0, :m]
    # E[X^] = X: the mean over seeds is within 5 sigma of x for every entry
    mean = acc / seeds
    lo_hi = [(qv[max(np.searchsorted(qv, v, "right") - 1, 0)], qv[min(np.searchsorted(qv, v, "right"), m - 1)])
             for v in x[0].astype(np.float64)]
    sig = np.array([(h - l) / 2 for l, h in lo_hi]) / math.sqrt(seeds) + 1e-12
    assert np.all(np.abs(mean - x[0]) <= 5 * sig + 1e-7)
    # histogram mass matches mu (multinomial, 5 sigma)
    n_tot = seeds * x.shape[1]
    expect = mu * seeds
    sd_ = np.sqrt(n_tot * (mu / x.shape[1]) * (1 - mu / x.shape[1]))
    assert np.all(np.abs(counts - expect) <= 5 * sd_ + 1)


def test_encode_time_sharing_share(O):
    rng = np.random.default_rng([31, 0])
    x = W.draw("normal", rng, 1, 20000)
    P, _ = O.grid_batch(x, 32)
    r = O.solve_budget_batch(x, P, 8, 2.2, 30)
    assert 0 < r["theta"][0] < 1
    idx, hist, st = O.encode_batch(x, P, r["Q1"], r["m1"], 8, 1, r["Q2"], r["m2"], r["theta"])
    share = hist[0, 0].sum() / x.shape[1]
    th = r["theta"][0]
    assert abs(share - th) < 5 * math.sqrt(th * (1 - th) / x.shape[1])
    Hemp = O.entropy(hist[0], 8)
    Hts = th * r["H1"][0] + (1 - th) * r["H2"][0]
    assert abs(Hemp - Hts) < 0.05


def test_entropy_of_histogram(O):
    hist = np.zeros((2, 4), np.int64)
    hist[0, :3] = [1, 1, 2]          # H = 1.5 bits over 4 entries
    hist[1, :2] = [2, 2]             # H = 1 bit over 4 entries
    assert O.entropy(hist, 4) == pytest.approx((4 * 1.5 + 4 * 1.0) / 8, rel=1e-15)


def _grid_cases():
    rng = np.random.default_rng([41, 0])
    cases = []
    for p in (2, 3, 7, 17, 64, 128, 256, 512):
        for lo, hi in ((-1.0, 1.0), (0.0, 3.0), (-2.5e-3, 7.0e-2), (1000.0, 1000.5), (-3.0e5, -2.0e5)):
            cases.append((p, lo, hi))
    for _ in range(6):
        a, b = np.sort(rng.standard_normal(2) * 10.0 ** rng.integers(-3, 4, 2))
        cases.append((int(rng.integers(2, 513)), float(a), float(b)))
    return cases


@pytest.mark.parametrize("p,lo,hi", _grid_cases())
def test_grid_interior_is_uniform(O, p, lo, hi):
    """A uniform grid spanning [min X, max X]: P_k equals the exact rational
    lo + (hi - lo) k / (p - 1) to within the rounding of a few fp64 operations,
    and every spacing P_{k+1} - P_k equals (hi - lo)/(p - 1) likewise. A grid
    built with k/p (or any other slip in the spacing) is off by span/p at the
    interior points, far beyond these bounds."""
    rng = np.random.default_rng([43, p])
    x = rng.uniform(lo, hi, size=257).astype(np.float32)
    x[0], x[-1] = np.float32(lo), np.float32(hi)
    flo, fhi = float(x.min()), float(x.max())
    P, st = O.uniform_grid(x, p)
    Pb, stb = O.grid_batch(x[None, :], p)
    assert st == 0 and stb[0] == 0
    np.testing.assert_array_equal(P, Pb[0])
    span = Fraction(fhi) - Fraction(flo)
    tol = 4 * np.spacing(max(abs(flo), abs(fhi), float(span)))
    for k in range(p):
        exact = Fraction(flo) + span * k / (p - 1)
        assert abs(Fraction(float(P[k])) - exact) <= Fraction(tol), (k, float(P[k]), float(exact))
    assert P[0] == flo and P[-1] == fhi
    step = float(span / (p - 1))
    assert np.all(np.abs(np.diff(P) - step) <= 2 * tol)


def test_grid_is_exact_endpoints(O):
    x = W.random_case(3, 1, 777, "lognormal")
    P, st = O.uniform_grid(x[0], 17)
    assert st == 0 and P[0] == x.min() and P[-1] == x.max()
    assert np.all(np.diff(P) > 0)
    bad = x.copy()
    bad[0, 5] = np.nan
    _, st = O.uniform_grid(bad[0], 17)
    assert st == -2
