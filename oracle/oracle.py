"""ctypes front end of the fp64 CPU oracle (oracle/ecasq_oracle.cpp).

TEST INFRASTRUCTURE ONLY: imported by tests/, by __graft_entry__.smoke() and by
bench.py's cpu_baseline / reference leg. The product package never imports it.

Every function takes and returns numpy arrays. Definitions follow the ECASQ
technical summary (gist.science/pt/paper/2608.18147), §1 (problem), §2.1
(Lagrangian relaxation, time-sharing) and §2.2 (the pair-state DP over a
permissible set P); the C++ source states each one.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_lib = None


def lib():
    global _lib
    if _lib is None:
        from . import build as _build  # type: ignore

        path = _build.build()
        L = C.CDLL(path)
        f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
        f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
        i64p = np.ctypeslib.ndpointer(np.int64, flags="C_CONTIGUOUS")
        i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
        u8p = np.ctypeslib.ndpointer(np.uint8, flags="C_CONTIGUOUS")
        u32p = np.ctypeslib.ndpointer(np.uint32, flags="C_CONTIGUOUS")
        u64p = np.ctypeslib.ndpointer(np.uint64, flags="C_CONTIGUOUS")
        u16p = np.ctypeslib.ndpointer(np.uint16, flags="C_CONTIGUOUS")
        I, I64, D, U64 = C.c_int, C.c_int64, C.c_double, C.c_uint64
        sig = {
            "eo_uniform_grid": (I, [f32p, I64, I, f64p]),
            "eo_bucket": (I, [f32p, I64, f64p, I, i64p, f64p, f64p]),
            "eo_tables": (None, [i64p, f64p, f64p, f64p, I, f64p, f64p, f64p]),
            "eo_eval_tables": (None, [f64p, f64p, f64p, I, I64, i32p, I, C.POINTER(D), C.POINTER(D), C.c_void_p]),
            "eo_eval_raw": (I, [f32p, I64, f64p, I, C.POINTER(D), C.POINTER(D), C.c_void_p]),
            "eo_dp": (I, [f64p, f64p, f64p, I, I, I64, D, i32p, C.POINTER(C.c_int32), C.POINTER(D)]),
            "eo_philox4x32_10": (None, [u32p, u32p, u32p]),
            "eo_philox4x64_10": (None, [u64p, u64p, u64p]),
            "eo_entropy": (D, [i64p, I]),
            "eo_threads": (I, []),
            "eo_solve_batch": (I, [f32p, I, I64, f64p, I, I, f64p, I, i32p, i32p, f64p, f64p, f64p, i32p]),
            "eo_solve_budget_batch": (I, [f32p, I, I64, f64p, I, I, D, I, i32p, i32p, i32p, i32p,
                                          f64p, f64p, f64p, f64p, f64p, f64p, f64p, i32p]),
            "eo_encode_batch": (I, [f32p, I, I64, f64p, I, i32p, i32p, C.c_void_p, C.c_void_p, C.c_void_p,
                                    I, U64, u8p, i64p, i32p]),
            "eo_grid_batch": (I, [f32p, I, I64, I, f64p, i32p]),
            "eo_dequantize_batch": (I, [u8p, I, I64, f64p, I, i32p, i32p, C.c_void_p, C.c_void_p, C.c_void_p,
                                        I, U64, f32p, i32p]),
            "eo_hib_tables": (D, [f64p, f64p, f64p, I, I64, i32p, I]),
            "eo_bf16_alphabet": (I, [f32p, I64, f64p, I]),
            "eo_rans_segment_words": (C.c_int64, []),
            "eo_rans_segments": (C.c_int64, [I64]),
            "eo_rans_model": (None, [i64p, I, u32p, u32p]),
            "eo_rans_encode_batch": (I, [u8p, I, I64, I, i64p, C.c_void_p, I, U64, u16p, i32p, i32p]),
            "eo_rans_decode_batch": (I, [u16p, i32p, I, I64, I, i64p, C.c_void_p, I, U64, u8p, i32p]),
            "eo_eval_raw_ib": (I, [f32p, I64, f64p, I, C.POINTER(D)]),
            "eo_approx_dp": (I, [f64p, f64p, f64p, I, I, I64, D, i32p, C.POINTER(C.c_int32), C.POINTER(D)]),
            "eo_refine_local": (D, [f64p, f64p, f64p, I, I64, D, i32p, I, I, I]),
            "eo_refine_point": (I, [f64p, f64p, f64p, I, I64, D, i32p, I, I]),
            "eo_refine": (I, [f64p, f64p, f64p, I, I64, D, i32p, I, I, C.POINTER(C.c_int32)]),
            "eo_solve_approx_batch": (I, [f32p, I, I64, f64p, I, I, f64p, I, I, i32p, i32p, f64p, f64p, f64p,
                                          f64p, i32p]),
            "eo_solve_approx_budget_batch": (I, [f32p, I, I64, f64p, I, I, D, I, I, i32p, i32p, i32p, i32p,
                                                 f64p, f64p, f64p, f64p, f64p, f64p, f64p, f64p, f64p, i32p]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _f32(x):
    return np.ascontiguousarray(x, dtype=np.float32)


def _f64(x):
    return np.ascontiguousarray(x, dtype=np.float64)


def threads() -> int:
    return int(lib().eo_threads())


# -- single-vector building blocks -------------------------------------------

def uniform_grid(x, p):
    x = _f32(x).ravel()
    P = np.empty(p, np.float64)
    st = lib().eo_uniform_grid(x, x.size, p, P)
    return P, st


def bucket(x, P):
    x = _f32(x).ravel()
    P = _f64(P)
    p = P.size
    cnt = np.zeros(p - 1, np.int64)
    A = np.zeros(p - 1, np.float64)
    B = np.zeros(p - 1, np.float64)
    st = lib().eo_bucket(x, x.size, P, p, cnt, A, B)
    return cnt, A, B, st


def tables(cnt, A, B, P):
    P = _f64(P)
    p = P.size
    V = np.zeros((p, p))
    R = np.zeros((p, p))
    L = np.zeros((p, p))
    lib().eo_tables(np.ascontiguousarray(cnt, np.int64), _f64(A), _f64(B), P, p, V, R, L)
    return V, R, L


def eval_tables(V, R, L, d, Q):
    Q = np.ascontiguousarray(Q, np.int32)
    p = V.shape[0]
    mse, H = C.c_double(), C.c_double()
    mu = np.zeros(max(Q.size, 1))
    lib().eo_eval_tables(_f64(V), _f64(R), _f64(L), p, d, Q, Q.size, C.byref(mse), C.byref(H),
                         mu.ctypes.data_as(C.c_void_p))
    return mse.value, H.value, mu[: Q.size]


def eval_raw(x, qvals):
    x = _f32(x).ravel()
    q = _f64(qvals)
    mse, H = C.c_double(), C.c_double()
    mu = np.zeros(max(q.size, 1))
    st = lib().eo_eval_raw(x, x.size, q, q.size, C.byref(mse), C.byref(H), mu.ctypes.data_as(C.c_void_p))
    if st:
        raise ValueError("entry outside the code range")
    return mse.value, H.value, mu[: q.size]


def dp(V, R, L, s, d, lam):
    p = V.shape[0]
    Q = np.full(min(s, p), -1, np.int32)
    m = C.c_int32()
    J = C.c_double()
    st = lib().eo_dp(_f64(V), _f64(R), _f64(L), p, s, d, lam, Q, C.byref(m), C.byref(J))
    if st:
        raise ValueError("oracle dp failed")
    return Q[: m.value].copy(), J.value


# -- approximation on H(I,B) and iterative refinement (§2.3, §2.4) ------------

def bf16_alphabet(x, p_max=65536):
    """Every finite BF16 value from the largest <= min x to the smallest >= max x."""
    x = _f32(x).ravel()
    P = np.zeros(p_max)
    n = int(lib().eo_bf16_alphabet(x, x.size, P, p_max))
    if n < 0:
        raise ValueError("non-finite entry or range outside BF16")
    return P[: min(n, p_max)].copy(), n


def hib_tables(V, R, L, d, Q):
    Q = np.ascontiguousarray(Q, np.int32)
    return float(lib().eo_hib_tables(_f64(V), _f64(R), _f64(L), V.shape[0], d, Q, Q.size))


def eval_raw_ib(x, qvals):
    x = _f32(x).ravel()
    q = _f64(qvals)
    out = C.c_double()
    if lib().eo_eval_raw_ib(x, x.size, q, q.size, C.byref(out)):
        raise ValueError("entry outside the code range")
    return out.value


def approx_dp(V, R, L, s, d, lam):
    p = V.shape[0]
    Q = np.full(min(s, p), -1, np.int32)
    m = C.c_int32()
    J = C.c_double()
    if lib().eo_approx_dp(_f64(V), _f64(R), _f64(L), p, s, d, lam, Q, C.byref(m), C.byref(J)):
        raise ValueError("oracle approx dp failed")
    return Q[: m.value].copy(), J.value


def refine_local(V, R, L, d, lam, Q, t, c):
    Q = np.ascontiguousarray(Q, np.int32)
    return float(lib().eo_refine_local(_f64(V), _f64(R), _f64(L), V.shape[0], d, lam, Q, Q.size, t, c))


def refine_point(V, R, L, d, lam, Q, t):
    Q = np.ascontiguousarray(Q, np.int32)
    return int(lib().eo_refine_point(_f64(V), _f64(R), _f64(L), V.shape[0], d, lam, Q, Q.size, t))


def refine(V, R, L, d, lam, Q, iters):
    """Returns (refined Q, moves, iterations run)."""
    Q = np.ascontiguousarray(Q, np.int32).copy()
    done = C.c_int32()
    moves = lib().eo_refine(_f64(V), _f64(R), _f64(L), V.shape[0], d, lam, Q, Q.size, iters, C.byref(done))
    return Q, int(moves), int(done.value)


def solve_approx_batch(X, P, s, lam, refine=0):
    """lam: [n] or [n, L]. J is MSE + lam*H(I,B) (refine == 0) or MSE + lam*H (refine > 0)."""
    X = _f32(X)
    n, d = X.shape
    P = _f64(P)
    p = P.shape[1]
    lam = _f64(lam).reshape(n, -1)
    nl = lam.shape[1]
    out = dict(Q=np.full((n, nl, s), -1, np.int32), m=np.zeros((n, nl), np.int32))
    for k in ("J", "mse", "H", "HIB"):
        out[k] = np.zeros((n, nl))
    out["status"] = np.zeros((n, nl), np.int32)
    out["threads"] = lib().eo_solve_approx_batch(X, n, d, P, p, s, lam, nl, int(refine), out["Q"], out["m"],
                                                 out["J"], out["mse"], out["H"], out["HIB"], out["status"])
    return out


def solve_approx_budget_batch(X, P, s, b, steps=30, refine=0):
    X = _f32(X)
    n, d = X.shape
    P = _f64(P)
    p = P.shape[1]
    out = dict(Q1=np.full((n, s), -1, np.int32), m1=np.zeros(n, np.int32),
               Q2=np.full((n, s), -1, np.int32), m2=np.zeros(n, np.int32))
    for k in ("theta", "lam_lo", "lam_hi", "H1", "H2", "HIB1", "HIB2", "mse1", "mse2"):
        out[k] = np.zeros(n)
    out["status"] = np.zeros(n, np.int32)
    out["threads"] = lib().eo_solve_approx_budget_batch(
        X, n, d, P, p, s, float(b), steps, int(refine), out["Q1"], out["m1"], out["Q2"], out["m2"],
        out["theta"], out["lam_lo"], out["lam_hi"], out["H1"], out["H2"], out["HIB1"], out["HIB2"],
        out["mse1"], out["mse2"], out["status"])
    return out


# -- entropy coder (rANS) for the emitted indices (§1 "Contexto") ---------------

def rans_model(cnt):
    cnt = np.ascontiguousarray(cnt, np.int64)
    s = cnt.size
    f = np.zeros(s, np.uint32)
    cum = np.zeros(s + 1, np.uint32)
    lib().eo_rans_model(cnt, s, f, cum)
    return f, cum


def rans_encode(idx, hist, seed, theta=None, two_codes=False):
    """idx [n, d] u8, hist [n, 2, s]. Returns words [n, segments, cap] u16,
    seg_len [n, segments], status [n]."""
    idx = np.ascontiguousarray(idx, np.uint8)
    n, d = idx.shape
    hist = np.ascontiguousarray(hist, np.int64).reshape(n, 2, -1)
    s = hist.shape[2]
    nseg = int(lib().eo_rans_segments(d))
    cap = int(lib().eo_rans_segment_words())
    words = np.zeros((n, nseg, cap), np.uint16)
    seg_len = np.zeros((n, nseg), np.int32)
    st = np.zeros(n, np.int32)
    th = None if theta is None else np.ascontiguousarray(theta, np.float64).reshape(n)
    lib().eo_rans_encode_batch(idx, n, d, s, hist, None if th is None else th.ctypes.data_as(C.c_void_p),
                               int(bool(two_codes)), C.c_uint64(seed), words, seg_len, st)
    return words, seg_len, st


def rans_decode(words, seg_len, d, hist, seed, theta=None, two_codes=False):
    words = np.ascontiguousarray(words, np.uint16)
    seg_len = np.ascontiguousarray(seg_len, np.int32)
    n = words.shape[0]
    hist = np.ascontiguousarray(hist, np.int64).reshape(n, 2, -1)
    s = hist.shape[2]
    idx = np.zeros((n, d), np.uint8)
    st = np.zeros(n, np.int32)
    th = None if theta is None else np.ascontiguousarray(theta, np.float64).reshape(n)
    lib().eo_rans_decode_batch(words, seg_len, n, d, s, hist, None if th is None else th.ctypes.data_as(C.c_void_p),
                               int(bool(two_codes)), C.c_uint64(seed), idx, st)
    return idx, st


def philox4x32(ctr, key):
    out = np.zeros(4, np.uint32)
    lib().eo_philox4x32_10(np.asarray(ctr, np.uint32), np.asarray(key, np.uint32), out)
    return out


def philox4x64(ctr, key):
    out = np.zeros(4, np.uint64)
    lib().eo_philox4x64_10(np.asarray(ctr, np.uint64), np.asarray(key, np.uint64), out)
    return out


def entropy(hist, s):
    return float(lib().eo_entropy(np.ascontiguousarray(hist, np.int64).ravel(), s))


# -- batched drivers (OpenMP over vectors) -------------------------------------

def grid_batch(X, p):
    X = _f32(X)
    n, d = X.shape
    P = np.zeros((n, p))
    st = np.zeros(n, np.int32)
    lib().eo_grid_batch(X, n, d, p, P, st)
    return P, st


def solve_batch(X, P, s, lam):
    """lam: [n] or [n, L]. Returns dict of [n, L] arrays (Q is [n, L, s], -1 padded)."""
    X = _f32(X)
    n, d = X.shape
    P = _f64(P)
    p = P.shape[1]
    lam = _f64(lam).reshape(n, -1)
    nl = lam.shape[1]
    Q = np.full((n, nl, s), -1, np.int32)
    m = np.zeros((n, nl), np.int32)
    J = np.zeros((n, nl))
    mse = np.zeros((n, nl))
    H = np.zeros((n, nl))
    st = np.zeros((n, nl), np.int32)
    thr = lib().eo_solve_batch(X, n, d, P, p, s, lam, nl, Q, m, J, mse, H, st)
    return dict(Q=Q, m=m, J=J, mse=mse, H=H, status=st, threads=thr)


def solve_budget_batch(X, P, s, b, steps=30):
    X = _f32(X)
    n, d = X.shape
    P = _f64(P)
    p = P.shape[1]
    out = dict(Q1=np.full((n, s), -1, np.int32), m1=np.zeros(n, np.int32),
               Q2=np.full((n, s), -1, np.int32), m2=np.zeros(n, np.int32))
    for k in ("theta", "lam_lo", "lam_hi", "H1", "H2", "mse1", "mse2"):
        out[k] = np.zeros(n)
    out["status"] = np.zeros(n, np.int32)
    thr = lib().eo_solve_budget_batch(X, n, d, P, p, s, float(b), steps, out["Q1"], out["m1"], out["Q2"],
                                      out["m2"], out["theta"], out["lam_lo"], out["lam_hi"], out["H1"],
                                      out["H2"], out["mse1"], out["mse2"], out["status"])
    out["threads"] = thr
    return out


def encode_batch(X, P, Q1, m1, s, seed, Q2=None, m2=None, theta=None):
    X = _f32(X)
    n, d = X.shape
    P = _f64(P)
    p = P.shape[1]
    Q1 = np.ascontiguousarray(Q1, np.int32).reshape(n, s)
    m1 = np.ascontiguousarray(m1, np.int32).reshape(n)
    idx = np.zeros((n, d), np.uint8)
    hist = np.zeros((n, 2, s), np.int64)
    st = np.zeros(n, np.int32)
    keep = []
    if Q2 is not None:
        Q2 = np.ascontiguousarray(Q2, np.int32).reshape(n, s)
        m2 = np.ascontiguousarray(m2, np.int32).reshape(n)
        th = _f64(theta).reshape(n)
        keep = [Q2, m2, th]
        q2p, m2p, thp = (a.ctypes.data_as(C.c_void_p) for a in keep)
    else:
        q2p = m2p = thp = None
    lib().eo_encode_batch(X, n, d, P, p, Q1, m1, q2p, m2p, thp, s, C.c_uint64(seed), idx, hist, st)
    del keep
    return idx, hist, st


def dequantize_batch(idx, P, Q1, m1, s, seed, Q2=None, m2=None, theta=None):
    """X^ [n, d] float32 from the indices of encode_batch (same codes, seed and
    theta); status -1 for a row with an index outside its code."""
    idx = np.ascontiguousarray(idx, np.uint8)
    n, d = idx.shape
    P = _f64(P)
    p = P.shape[1]
    Q1 = np.ascontiguousarray(Q1, np.int32).reshape(n, s)
    m1 = np.ascontiguousarray(m1, np.int32).reshape(n)
    out = np.zeros((n, d), np.float32)
    st = np.zeros(n, np.int32)
    keep = []
    if Q2 is not None:
        Q2 = np.ascontiguousarray(Q2, np.int32).reshape(n, s)
        m2 = np.ascontiguousarray(m2, np.int32).reshape(n)
        th = _f64(theta).reshape(n)
        keep = [Q2, m2, th]
        q2p, m2p, thp = (a.ctypes.data_as(C.c_void_p) for a in keep)
    else:
        q2p = m2p = thp = None
    lib().eo_dequantize_batch(idx, n, d, P, p, Q1, m1, q2p, m2p, thp, s, C.c_uint64(seed), out, st)
    del keep
    return out, st


def encode_row(x, P_row, Q1, m1, s, seed, row, Q2=None, m2=0, theta=0.0):
    """Encode one vector that is row `row` of its batch (the Philox counter
    carries the row index). Returns idx [d] u8 and hist [2, s]."""
    L = lib()
    fn = L.eo_encode
    fn.restype = C.c_int
    fn.argtypes = [C.c_void_p, C.c_int64, C.c_void_p, C.c_int, C.c_void_p, C.c_int, C.c_void_p, C.c_int,
                   C.c_double, C.c_int, C.c_uint64, C.c_uint32, C.c_void_p, C.c_void_p]
    x = _f32(x).ravel()
    P_row = _f64(P_row).ravel()
    q1 = np.ascontiguousarray(Q1, np.int32).ravel()
    q2 = np.ascontiguousarray(Q2, np.int32).ravel() if Q2 is not None else None
    idx = np.zeros(x.size, np.uint8)
    hist = np.zeros(2 * s, np.int64)
    st = fn(x.ctypes.data, x.size, P_row.ctypes.data, P_row.size, q1.ctypes.data, int(m1),
            q2.ctypes.data if q2 is not None else None, int(m2), float(theta), s, C.c_uint64(seed), row,
            idx.ctypes.data, hist.ctypes.data)
    if st:
        raise ValueError("oracle encode failed")
    return idx, hist.reshape(2, s)
