"""Thin ctypes binding of libecasq.so (C ABI in include/ecasq.h).

Argument marshalling only: every step of the solver runs in the library's CUDA
kernels. torch provides device memory and the current stream. There is no CPU
fallback: loading raises if the library is missing or no CUDA device exists.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libecasq.so")

OK, ERR_ARG, ERR_RANGE, ERR_WORKSPACE, ERR_CUDA, WARN_BUDGET = 0, -1, -2, -3, -4, 1

EXPORTS = [
    "ecasq_workspace_size", "ecasq_aux_workspace_size", "ecasq_uniform_grid", "ecasq_bf16_alphabet", "ecasq_bucket",
    "ecasq_bucket_noalloc", "ecasq_grid_bucket",
    "ecasq_solve", "ecasq_solve_stats", "ecasq_solve_budget", "ecasq_solve_budget_stats",
    "ecasq_approx_workspace_size", "ecasq_solve_approx", "ecasq_solve_approx_stats", "ecasq_solve_approx_budget",
    "ecasq_solve_approx_budget_stats",
    "ecasq_encode", "ecasq_dequantize", "ecasq_entropy", "ecasq_rans_segments", "ecasq_rans_segment_words",
    "ecasq_rans_encode", "ecasq_rans_decode", "ecasq_status_string", "ecasq_launch_count",
]


class EcasqError(RuntimeError):
    pass


class Opts(C.Structure):
    _fields_ = [("dp_fp64", C.c_int), ("hirschberg", C.c_int), ("bisect_steps", C.c_int),
                ("reserved", C.c_int)]


_lib = None


def load(path: str = LIB_PATH):
    """Load the library and declare its signatures (no CUDA call is made)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise EcasqError(f"libecasq.so not built ({path}); run __graft_entry__.build()")
    L = C.CDLL(path)
    P, I, I64, D, SZ, U64 = C.c_void_p, C.c_int, C.c_int64, C.c_double, C.c_size_t, C.c_uint64
    OP = C.POINTER(Opts)
    sig = {
        "ecasq_workspace_size": (SZ, [I, I64, I, I, I, OP]),
        "ecasq_aux_workspace_size": (SZ, [I, I64, I]),
        "ecasq_uniform_grid": (I, [P, I, I64, I, P, P, P, SZ, P]),
        "ecasq_bf16_alphabet": (I, [P, I, I64, I, P, P, P, P, SZ, P]),
        "ecasq_bucket": (I, [P, P, I, I64, I, P, P, P, P, P, SZ, P]),
        "ecasq_grid_bucket": (I, [P, I, I64, I, P, P, P, P, P, P, SZ, P]),
        "ecasq_bucket_noalloc": (I, [P, P, I, I64, I, P, P, P, P, P]),
        "ecasq_solve": (I, [P, P, I, I64, I, I, P, I, P, P, P, P, P, P, OP, P, SZ, P]),
        "ecasq_solve_stats": (I, [P, P, P, P, I, I64, I, I, P, I, P, P, P, P, P, P, OP, P, SZ, P]),
        "ecasq_solve_budget": (I, [P, P, I, I64, I, I, D] + [P] * 12 + [OP, P, SZ, P]),
        "ecasq_solve_budget_stats": (I, [P, P, P, P, I, I64, I, I, D] + [P] * 12 + [OP, P, SZ, P]),
        "ecasq_approx_workspace_size": (SZ, [I, I64, I, I, OP]),
        "ecasq_solve_approx": (I, [P, P, I, I64, I, I, P, I, I, P, P, P, P, P, P, P, OP, P, SZ, P]),
        "ecasq_solve_approx_stats": (I, [P, P, P, P, I, I64, I, I, P, I, I, P, P, P, P, P, P, P, OP, P, SZ, P]),
        "ecasq_solve_approx_budget": (I, [P, P, I, I64, I, I, D, I] + [P] * 14 + [OP, P, SZ, P]),
        "ecasq_solve_approx_budget_stats": (I, [P, P, P, P, I, I64, I, I, D, I] + [P] * 14 + [OP, P, SZ, P]),
        "ecasq_encode": (I, [P, P, I, I64, I, I, P, P, P, P, P, U64, P, P, P, P]),
        "ecasq_entropy": (I, [P, I, I, P, P]),
        "ecasq_dequantize": (I, [P, P, I, I64, I, I, P, P, P, P, P, U64, P, P, P]),
        "ecasq_rans_segments": (I64, [I64]),
        "ecasq_rans_segment_words": (I64, []),
        "ecasq_rans_encode": (I, [P, P, P, I, I, I64, I, U64, P, P, P, P]),
        "ecasq_rans_decode": (I, [P, P, P, P, I, I, I64, I, U64, P, P, P]),
        "ecasq_status_string": (C.c_char_p, [I]),
        "ecasq_launch_count": (C.c_uint64, [I]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def _need_cuda():
    if not torch.cuda.is_available():
        raise EcasqError("ECASQ needs a CUDA device; there is no CPU fallback")
    return load()


def _ptr(t):
    return C.c_void_p(t.data_ptr()) if t is not None else C.c_void_p(0)


def _stream():
    return C.c_void_p(torch.cuda.current_stream().cuda_stream)


def _check(rc: int, what: str):
    if rc != OK:
        msg = load().ecasq_status_string(rc).decode()
        raise EcasqError(f"{what}: {msg} ({rc})")


def _dev(t, dtype, name):
    if not (t.is_cuda and t.dtype == dtype and t.is_contiguous()):
        raise EcasqError(f"{name} must be a contiguous CUDA {dtype} tensor")
    return t


_ws_cache: dict = {}


def workspace(nbytes: int, device) -> torch.Tensor:
    """A cached device buffer of at least nbytes (the library never allocates)."""
    key = torch.device(device)
    buf = _ws_cache.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=key)
        _ws_cache[key] = buf
    return buf


def opts(fp64: bool = False, steps: int = 30, hirschberg: bool = False) -> Opts:
    return Opts(int(fp64), int(hirschberg), int(steps), 0)


def launch_count(reset: bool = False) -> int:
    return int(load().ecasq_launch_count(int(reset)))


def uniform_grid(X: torch.Tensor, p: int):
    L = _need_cuda()
    _dev(X, torch.float32, "X")
    n, d = X.shape
    P = torch.empty((n, p), dtype=torch.float64, device=X.device)
    st = torch.empty(n, dtype=torch.int32, device=X.device)
    ws = workspace(L.ecasq_aux_workspace_size(n, d, p), X.device)
    _check(L.ecasq_uniform_grid(_ptr(X), n, d, p, _ptr(P), _ptr(st), _ptr(ws), ws.numel(), _stream()),
           "ecasq_uniform_grid")
    return P, st


def bf16_alphabet(X: torch.Tensor, p_max: int):
    """Per row, every BF16 value covering [min X, max X]. Returns P [n, p_max]
    (NaN past each row's count), p_len [n], status [n]."""
    L = _need_cuda()
    _dev(X, torch.float32, "X")
    n, d = X.shape
    P = torch.empty((n, p_max), dtype=torch.float64, device=X.device)
    p_len = torch.empty(n, dtype=torch.int32, device=X.device)
    st = torch.empty(n, dtype=torch.int32, device=X.device)
    ws = workspace(L.ecasq_aux_workspace_size(n, d, 2), X.device)
    _check(L.ecasq_bf16_alphabet(_ptr(X), n, d, p_max, _ptr(P), _ptr(p_len), _ptr(st), _ptr(ws), ws.numel(),
                                 _stream()), "ecasq_bf16_alphabet")
    return P, p_len, st


def bucket(X: torch.Tensor, P: torch.Tensor):
    L = _need_cuda()
    _dev(X, torch.float32, "X")
    _dev(P, torch.float64, "P")
    n, d = X.shape
    p = P.shape[1]
    cnt = torch.empty((n, p - 1), dtype=torch.int64, device=X.device)
    A = torch.empty((n, p - 1), dtype=torch.float64, device=X.device)
    B = torch.empty_like(A)
    st = torch.empty(n, dtype=torch.int32, device=X.device)
    ws = workspace(L.ecasq_aux_workspace_size(n, d, p), X.device)
    _check(L.ecasq_bucket(_ptr(X), _ptr(P), n, d, p, _ptr(cnt), _ptr(A), _ptr(B), _ptr(st), _ptr(ws), ws.numel(),
                          _stream()), "ecasq_bucket")
    return cnt, A, B, st


def grid_bucket(X: torch.Tensor, p: int):
    """Uniform grid and bucketing in one call (one read of X when rows fit in
    shared memory). Returns P [n,p] f64, cnt [n,p-1] i64, A, B [n,p-1] f64, status."""
    L = _need_cuda()
    _dev(X, torch.float32, "X")
    n, d = X.shape
    P = torch.empty((n, p), dtype=torch.float64, device=X.device)
    cnt = torch.empty((n, p - 1), dtype=torch.int64, device=X.device)
    A = torch.empty((n, p - 1), dtype=torch.float64, device=X.device)
    B = torch.empty((n, p - 1), dtype=torch.float64, device=X.device)
    st = torch.empty(n, dtype=torch.int32, device=X.device)
    ws = workspace(L.ecasq_aux_workspace_size(n, d, p), X.device)
    _check(L.ecasq_grid_bucket(_ptr(X), n, d, p, _ptr(P), _ptr(cnt), _ptr(A), _ptr(B), _ptr(st), _ptr(ws),
                               ws.numel(), _stream()), "ecasq_grid_bucket")
    return P, cnt, A, B, st


def bucket_noalloc(X: torch.Tensor, P: torch.Tensor):
    """ecasq_bucket through the workspace-free entry point: the library uses its
    own fixed device array instead of a workspace (for callers that cannot
    allocate device memory; calls on one GPU must not overlap)."""
    L = _need_cuda()
    _dev(X, torch.float32, "X")
    _dev(P, torch.float64, "P")
    n, d = X.shape
    p = P.shape[1]
    cnt = torch.empty((n, p - 1), dtype=torch.int64, device=X.device)
    A = torch.empty((n, p - 1), dtype=torch.float64, device=X.device)
    B = torch.empty_like(A)
    st = torch.empty(n, dtype=torch.int32, device=X.device)
    _check(L.ecasq_bucket_noalloc(_ptr(X), _ptr(P), n, d, p, _ptr(cnt), _ptr(A), _ptr(B), _ptr(st), _stream()),
           "ecasq_bucket_noalloc")
    return cnt, A, B, st


def _lam_table(lam, n, device):
    lam = torch.as_tensor(lam, dtype=torch.float64)
    if lam.dim() == 0:
        lam = lam.expand(n, 1)
    elif lam.dim() == 1:
        lam = lam.reshape(n, 1) if lam.numel() == n else lam.reshape(1, -1).expand(n, -1)
    return lam.to(device).contiguous()


def _solve_outputs(n, nl, s, device):
    return dict(Q=torch.empty((n, nl, s), dtype=torch.int32, device=device),
                Q_len=torch.empty((n, nl), dtype=torch.int32, device=device),
                objective=torch.empty((n, nl), dtype=torch.float64, device=device),
                mse=torch.empty((n, nl), dtype=torch.float64, device=device),
                H=torch.empty((n, nl), dtype=torch.float64, device=device),
                status=torch.empty(n, dtype=torch.int32, device=device))


def solve(X: torch.Tensor, P: torch.Tensor, s: int, lam, fp64: bool = False, hirschberg: bool = False):
    """Exact Lagrangian solve of each row at each of its lambdas ([n] or [n, L])."""
    L = _need_cuda()
    _dev(X, torch.float32, "X")
    _dev(P, torch.float64, "P")
    n, d = X.shape
    p = P.shape[1]
    lt = _lam_table(lam, n, X.device)
    nl = lt.shape[1]
    o = _solve_outputs(n, nl, s, X.device)
    op = opts(fp64, hirschberg=hirschberg)
    ws = workspace(L.ecasq_workspace_size(n, d, p, s, nl, C.byref(op)), X.device)
    _check(L.ecasq_solve(_ptr(X), _ptr(P), n, d, p, s, _ptr(lt), nl, _ptr(o["Q"]), _ptr(o["Q_len"]),
                         _ptr(o["objective"]), _ptr(o["mse"]), _ptr(o["H"]), _ptr(o["status"]), C.byref(op),
                         _ptr(ws), ws.numel(), _stream()), "ecasq_solve")
    return o


def solve_stats(cnt, A, B, P, d: int, s: int, lam, fp64: bool = False, hirschberg: bool = False):
    L = _need_cuda()
    n, p = P.shape
    lt = _lam_table(lam, n, P.device)
    nl = lt.shape[1]
    o = _solve_outputs(n, nl, s, P.device)
    op = opts(fp64, hirschberg=hirschberg)
    ws = workspace(L.ecasq_workspace_size(n, d, p, s, nl, C.byref(op)), P.device)
    _check(L.ecasq_solve_stats(_ptr(cnt), _ptr(A), _ptr(B), _ptr(P), n, d, p, s, _ptr(lt), nl, _ptr(o["Q"]),
                               _ptr(o["Q_len"]), _ptr(o["objective"]), _ptr(o["mse"]), _ptr(o["H"]),
                               _ptr(o["status"]), C.byref(op), _ptr(ws), ws.numel(), _stream()),
           "ecasq_solve_stats")
    return o


def _budget_outputs(n, s, device):
    o = dict(Q1=torch.empty((n, s), dtype=torch.int32, device=device),
             Q1_len=torch.empty(n, dtype=torch.int32, device=device),
             Q2=torch.empty((n, s), dtype=torch.int32, device=device),
             Q2_len=torch.empty(n, dtype=torch.int32, device=device))
    for k in ("theta", "lambda_lo", "lambda_hi", "H1", "H2", "mse1", "mse2"):
        o[k] = torch.empty(n, dtype=torch.float64, device=device)
    o["status"] = torch.empty(n, dtype=torch.int32, device=device)
    return o


_BUDGET_ORDER = ("Q1", "Q1_len", "Q2", "Q2_len", "theta", "lambda_lo", "lambda_hi", "H1", "H2", "mse1", "mse2",
                 "status")


def solve_budget(X: torch.Tensor, P: torch.Tensor, s: int, b: float, steps: int = 30, fp64: bool = False,
                 hirschberg: bool = False):
    """Entropy budget b: lambda bisection plus two-way time-sharing per row."""
    L = _need_cuda()
    _dev(X, torch.float32, "X")
    _dev(P, torch.float64, "P")
    n, d = X.shape
    p = P.shape[1]
    o = _budget_outputs(n, s, X.device)
    op = opts(fp64, steps, hirschberg)
    ws = workspace(L.ecasq_workspace_size(n, d, p, s, 1, C.byref(op)), X.device)
    _check(L.ecasq_solve_budget(_ptr(X), _ptr(P), n, d, p, s, float(b), *[_ptr(o[k]) for k in _BUDGET_ORDER],
                                C.byref(op), _ptr(ws), ws.numel(), _stream()), "ecasq_solve_budget")
    return o


def solve_budget_stats(cnt, A, B, P, d: int, s: int, b: float, steps: int = 30, fp64: bool = False,
                       hirschberg: bool = False):
    L = _need_cuda()
    n, p = P.shape
    o = _budget_outputs(n, s, P.device)
    op = opts(fp64, steps, hirschberg)
    ws = workspace(L.ecasq_workspace_size(n, d, p, s, 1, C.byref(op)), P.device)
    _check(L.ecasq_solve_budget_stats(_ptr(cnt), _ptr(A), _ptr(B), _ptr(P), n, d, p, s, float(b),
                                      *[_ptr(o[k]) for k in _BUDGET_ORDER], C.byref(op), _ptr(ws), ws.numel(),
                                      _stream()), "ecasq_solve_budget_stats")
    return o


# -- approximation on H(I,B) and iterative refinement ---------------------------

def solve_approx(X: torch.Tensor, P: torch.Tensor, s: int, lam, refine: int = 0, fp64: bool = False):
    """Approximate solve of each row at each of its lambdas ([n] or [n, L]); with
    refine > 0 the code is then refined on the exact objective. Adds H_IB."""
    L = _need_cuda()
    _dev(X, torch.float32, "X")
    _dev(P, torch.float64, "P")
    n, d = X.shape
    p = P.shape[1]
    lt = _lam_table(lam, n, X.device)
    nl = lt.shape[1]
    o = _solve_outputs(n, nl, s, X.device)
    o["H_IB"] = torch.empty((n, nl), dtype=torch.float64, device=X.device)
    op = opts(fp64)
    ws = workspace(L.ecasq_approx_workspace_size(n, d, p, s, C.byref(op)), X.device)
    _check(L.ecasq_solve_approx(_ptr(X), _ptr(P), n, d, p, s, _ptr(lt), nl, int(refine), _ptr(o["Q"]),
                                _ptr(o["Q_len"]), _ptr(o["objective"]), _ptr(o["mse"]), _ptr(o["H"]),
                                _ptr(o["H_IB"]), _ptr(o["status"]), C.byref(op), _ptr(ws), ws.numel(), _stream()),
           "ecasq_solve_approx")
    return o


def solve_approx_stats(cnt, A, B, P, d: int, s: int, lam, refine: int = 0, fp64: bool = False):
    L = _need_cuda()
    n, p = P.shape
    lt = _lam_table(lam, n, P.device)
    nl = lt.shape[1]
    o = _solve_outputs(n, nl, s, P.device)
    o["H_IB"] = torch.empty((n, nl), dtype=torch.float64, device=P.device)
    op = opts(fp64)
    ws = workspace(L.ecasq_approx_workspace_size(n, d, p, s, C.byref(op)), P.device)
    _check(L.ecasq_solve_approx_stats(_ptr(cnt), _ptr(A), _ptr(B), _ptr(P), n, d, p, s, _ptr(lt), nl, int(refine),
                                      _ptr(o["Q"]), _ptr(o["Q_len"]), _ptr(o["objective"]), _ptr(o["mse"]),
                                      _ptr(o["H"]), _ptr(o["H_IB"]), _ptr(o["status"]), C.byref(op), _ptr(ws),
                                      ws.numel(), _stream()), "ecasq_solve_approx_stats")
    return o


_APPROX_BUDGET_ORDER = ("Q1", "Q1_len", "Q2", "Q2_len", "theta", "lambda_lo", "lambda_hi", "H1", "H2", "H_IB1",
                        "H_IB2", "mse1", "mse2", "status")


def _approx_budget_outputs(n, s, device):
    o = _budget_outputs(n, s, device)
    for k in ("H_IB1", "H_IB2"):
        o[k] = torch.empty(n, dtype=torch.float64, device=device)
    return o


def solve_approx_budget(X: torch.Tensor, P: torch.Tensor, s: int, b: float, refine: int = 0, steps: int = 30,
                        fp64: bool = False):
    """Entropy budget b for the approximation (rate H(I,B)) or, with refine > 0,
    for the refined approximation (rate H)."""
    L = _need_cuda()
    _dev(X, torch.float32, "X")
    _dev(P, torch.float64, "P")
    n, d = X.shape
    p = P.shape[1]
    o = _approx_budget_outputs(n, s, X.device)
    op = opts(fp64, steps)
    ws = workspace(L.ecasq_approx_workspace_size(n, d, p, s, C.byref(op)), X.device)
    _check(L.ecasq_solve_approx_budget(_ptr(X), _ptr(P), n, d, p, s, float(b), int(refine),
                                       *[_ptr(o[k]) for k in _APPROX_BUDGET_ORDER], C.byref(op), _ptr(ws),
                                       ws.numel(), _stream()), "ecasq_solve_approx_budget")
    return o


def solve_approx_budget_stats(cnt, A, B, P, d: int, s: int, b: float, refine: int = 0, steps: int = 30,
                              fp64: bool = False):
    L = _need_cuda()
    n, p = P.shape
    o = _approx_budget_outputs(n, s, P.device)
    op = opts(fp64, steps)
    ws = workspace(L.ecasq_approx_workspace_size(n, d, p, s, C.byref(op)), P.device)
    _check(L.ecasq_solve_approx_budget_stats(_ptr(cnt), _ptr(A), _ptr(B), _ptr(P), n, d, p, s, float(b), int(refine),
                                             *[_ptr(o[k]) for k in _APPROX_BUDGET_ORDER], C.byref(op), _ptr(ws),
                                             ws.numel(), _stream()), "ecasq_solve_approx_budget_stats")
    return o


def encode(X: torch.Tensor, P: torch.Tensor, s: int, Q1, Q1_len, seed: int, Q2=None, Q2_len=None, theta=None):
    """Stochastic rounding onto Q1 (or time-shared Q1/Q2). Returns idx [n,d] u8, hist [n,2,s] i64, status."""
    L = _need_cuda()
    _dev(X, torch.float32, "X")
    _dev(P, torch.float64, "P")
    n, d = X.shape
    p = P.shape[1]
    idx = torch.empty((n, d), dtype=torch.uint8, device=X.device)
    hist = torch.empty((n, 2, s), dtype=torch.int64, device=X.device)
    st = torch.empty(n, dtype=torch.int32, device=X.device)
    _check(L.ecasq_encode(_ptr(X), _ptr(P), n, d, p, s, _ptr(Q1), _ptr(Q1_len), _ptr(Q2), _ptr(Q2_len), _ptr(theta),
                          C.c_uint64(seed), _ptr(idx), _ptr(hist), _ptr(st), _stream()), "ecasq_encode")
    return idx, hist, st


def dequantize(idx: torch.Tensor, P: torch.Tensor, s: int, Q1, Q1_len, seed: int, Q2=None, Q2_len=None,
               theta=None):
    """X^ [n,d] float32 from the indices of encode (same codes, s, seed and theta), and status."""
    L = _need_cuda()
    _dev(idx, torch.uint8, "idx")
    _dev(P, torch.float64, "P")
    n, d = idx.shape
    p = P.shape[1]
    Xh = torch.empty((n, d), dtype=torch.float32, device=idx.device)
    st = torch.empty(n, dtype=torch.int32, device=idx.device)
    _check(L.ecasq_dequantize(_ptr(idx), _ptr(P), n, d, p, s, _ptr(Q1), _ptr(Q1_len), _ptr(Q2), _ptr(Q2_len),
                              _ptr(theta), C.c_uint64(seed), _ptr(Xh), _ptr(st), _stream()), "ecasq_dequantize")
    return Xh, st


def entropy(hist: torch.Tensor):
    L = _need_cuda()
    n, _, s = hist.shape
    H = torch.empty(n, dtype=torch.float64, device=hist.device)
    _check(L.ecasq_entropy(_ptr(hist), n, s, _ptr(H), _stream()), "ecasq_entropy")
    return H


# -- entropy coder for the indices --------------------------------------------------

def rans_encode(idx: torch.Tensor, hist: torch.Tensor, seed: int, theta=None, two_codes: bool = False):
    """rANS-code idx [n, d] u8 with per-row models from hist [n, 2, s]. Returns
    words [n, segments, cap] u16 (stored as int16), seg_len [n, segments], status."""
    L = _need_cuda()
    _dev(idx, torch.uint8, "idx")
    _dev(hist, torch.int64, "hist")
    n, d = idx.shape
    s = hist.shape[-1]
    nseg, cap = int(L.ecasq_rans_segments(d)), int(L.ecasq_rans_segment_words())
    words = torch.empty((n, nseg, cap), dtype=torch.int16, device=idx.device)
    seg_len = torch.empty((n, nseg), dtype=torch.int32, device=idx.device)
    st = torch.empty(n, dtype=torch.int32, device=idx.device)
    if theta is not None:
        _dev(theta, torch.float64, "theta")
    _check(L.ecasq_rans_encode(_ptr(idx), _ptr(hist), _ptr(theta) if theta is not None else None, int(bool(two_codes)),
                               n, d, s, C.c_uint64(seed), _ptr(words), _ptr(seg_len), _ptr(st), _stream()),
           "ecasq_rans_encode")
    return words, seg_len, st


def rans_decode(words: torch.Tensor, seg_len: torch.Tensor, hist: torch.Tensor, d: int, seed: int, theta=None,
                two_codes: bool = False):
    L = _need_cuda()
    n = words.shape[0]
    s = hist.shape[-1]
    idx = torch.empty((n, d), dtype=torch.uint8, device=words.device)
    st = torch.empty(n, dtype=torch.int32, device=words.device)
    _check(L.ecasq_rans_decode(_ptr(words), _ptr(seg_len), _ptr(hist), _ptr(theta) if theta is not None else None,
                               int(bool(two_codes)), n, d, s, C.c_uint64(seed), _ptr(idx), _ptr(st), _stream()),
           "ecasq_rans_decode")
    return idx, st
