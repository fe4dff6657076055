"""The C-ABI library loads and exports every symbol include/ecasq.h declares.
CPU only: no call here reaches the GPU (argument checks return before any
CUDA work)."""
import ctypes as C
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from entropy_constrained_unbiased_b200 import build, ecasq
    build.build()
    return ecasq.load()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "ecasq.h")).read()
    return sorted(set(re.findall(r"\b(ecasq_[a-z0-9_]+)\s*\(", text)))


def test_header_lists_the_binding_exports():
    from entropy_constrained_unbiased_b200 import ecasq
    assert declared_symbols() == sorted(ecasq.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code in (0, -1, -2, -3, -4, 1):
        assert lib.ecasq_status_string(code)
    assert lib.ecasq_status_string(99) == b"unknown status"


def test_argument_errors_return_before_cuda(lib):
    null = C.c_void_p(0)
    # null input / bad sizes: ECASQ_ERR_ARG
    assert lib.ecasq_uniform_grid(null, 1, 16, 8, null, null, null, 0, null) == -1
    assert lib.ecasq_bucket(null, null, 1, 16, 1, null, null, null, null, null, 0, null) == -1
    assert lib.ecasq_aux_workspace_size(0, 16, 8) == 0
    # alphabet-sized passes (grid, bucketing, encoding, approximation) take up to
    # 65536 values, the exact solver up to 512
    assert lib.ecasq_aux_workspace_size(4, 16, 65537) == 0
    assert lib.ecasq_aux_workspace_size(4, 16, 600) > 0
    assert lib.ecasq_aux_workspace_size(4, 1024, 64) > 0
    assert lib.ecasq_workspace_size(4, 16, 600, 4, 1, None) == 0
    assert lib.ecasq_entropy(null, 1, 4, null, null) == -1
    assert lib.ecasq_encode(null, null, 1, 16, 8, 4, null, null, null, null, null, 1, null, null, null, null) == -1
    # approximation: null X, negative refinement count, bad sizes
    dummy = C.c_void_p(16)  # never dereferenced: the checks fail first
    assert lib.ecasq_approx_workspace_size(0, 16, 8, 4, None) == 0
    assert lib.ecasq_approx_workspace_size(4, 16, 65537, 4, None) == 0
    assert lib.ecasq_solve_approx(null, dummy, 1, 16, 8, 4, dummy, 1, 0, *[dummy] * 7, None, dummy, 64, null) == -1
    assert lib.ecasq_solve_approx_stats(dummy, dummy, dummy, dummy, 1, 16, 8, 4, dummy, 1, -1, *[dummy] * 7, None,
                                        dummy, 64, null) == -1
    assert lib.ecasq_solve_approx_budget(dummy, dummy, 1, 16, 8, 1, 2.0, 0, *[dummy] * 14, None, dummy, 64,
                                         null) == -1
    assert lib.ecasq_solve_approx_budget_stats(dummy, dummy, dummy, dummy, 1, 16, 8, 4, -1.0, 0, *[dummy] * 14,
                                               None, dummy, 64, null) == -1


def test_missing_workspace_is_reported(lib):
    dummy = C.c_void_p(16)  # never dereferenced: the check fails first
    assert lib.ecasq_uniform_grid(dummy, 1, 16, 8, dummy, dummy, C.c_void_p(0), 0, C.c_void_p(0)) == -3


def test_launch_counter(lib):
    lib.ecasq_launch_count(1)
    assert lib.ecasq_launch_count(0) == 0


def test_product_path_has_no_cpu_fallback(monkeypatch):
    from entropy_constrained_unbiased_b200 import ecasq
    import torch
    if torch.cuda.is_available():
        pytest.skip("GPU present")
    with pytest.raises(ecasq.EcasqError):
        ecasq.uniform_grid(torch.zeros(1, 8), 4)


def test_triple_count_matches_enumeration():
    """Per-solve triple count (bench metric): every (k, l, j) the recurrence
    visits, counted directly; layer 2 has only k = 0 because c_1 = P_0."""
    from bench import triples_per_solve
    for p, s in [(8, 4), (12, 5), (64, 8), (20, 20), (30, 3), (5, 2)]:
        S = min(s, p)
        t = 0
        for i in range(2, S):
            for l in range(i - 1, p - 1):
                ks = [0] if i == 2 else range(i - 2, l)
                js = [p - 1] if i == S - 1 else range(l + 1, p)
                t += len(list(ks)) * len(list(js))
        assert triples_per_solve(p, s) == t
    assert triples_per_solve(64, 8) == 151347
    assert triples_per_solve(128, 16) == 3522197


def _pass_enum(s0, e0, T, last_only):
    t_ = 0
    for t in range(2, T + 1):
        last = last_only and t == T
        for l in range(s0 + t - 1, e0):
            ks = [s0] if t == 2 else range(s0 + t - 2, l)
            js = [e0] if last else range(l + 1, e0 + 1)
            t_ += len(list(ks)) * len(list(js))
    return t_


def test_hirschberg_triple_count_matches_enumeration():
    """Triples of a Hirschberg-mode solve: the whole-alphabet pass plus, per
    segment, a forward and a reflected pass, each enumerated directly; the
    segments follow the split rule on random codes."""
    from bench import hirschberg_triples, pass_triples, triples_per_solve
    rng = np.random.default_rng(3)
    for p, s in [(12, 5), (30, 8), (40, 12), (9, 9)]:
        assert pass_triples(0, p - 1, min(s, p) - 1, True) == triples_per_solve(p, s)
        for _ in range(5):
            m = int(rng.integers(2, min(s, p) + 1))
            code = np.concatenate([[0], np.sort(rng.choice(np.arange(1, p - 1), m - 2, replace=False)), [p - 1]])
            want = _pass_enum(0, p - 1, min(s, p) - 1, True)
            segs = [(0, m - 2)] if m >= 4 else []
            while segs:
                lo, hi = segs.pop()
                mid = lo + (hi - lo - 1 + 1) // 2
                want += _pass_enum(code[lo], code[hi], mid - lo + 1, mid + 1 == hi)
                want += _pass_enum(p - 1 - code[hi], p - 1 - code[lo], hi - mid, False)
                segs += [sg for sg in ((lo, mid), (mid + 1, hi)) if sg[1] - sg[0] - 1 >= 1]
            assert hirschberg_triples(code, p, s) == want, (p, s, code)


def test_quantize_argument_checks_and_no_cpu_path():
    """quantize() checks its arguments before any call and, without a GPU,
    fails in the binding instead of computing anything on the CPU."""
    import torch
    from entropy_constrained_unbiased_b200 import ecasq
    from entropy_constrained_unbiased_b200.pipeline import quantize
    X = torch.zeros(1, 8)
    with pytest.raises(ecasq.EcasqError):
        quantize(X, 4, 2)
    with pytest.raises(ecasq.EcasqError):
        quantize(X, 4, 2, b=1.0, lam=0.1)
    with pytest.raises(ecasq.EcasqError):
        quantize(X, 4, 2, b=1.0, solver="other")
    if not torch.cuda.is_available():
        with pytest.raises(ecasq.EcasqError):
            quantize(X, 4, 2, b=1.0)
