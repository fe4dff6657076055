"""Pins of the oracle's hardware-aware permissible set (CPU): every BF16 value
from the largest one <= min X to the smallest one >= max X ("Entropy-Constrained
Adaptive Stochastic Quantization (ECASQ)", gist.science/pt/paper/2608.18147, §5
"Generalidade": arbitrary permissible alphabets such as the values BF16 can
represent).

Pins: closed-form counts from the BF16 format (8 bits of precision: 128 values
per binade, spacing 2^(e-7) in [2^e, 2^(e+1)), 127 subnormals per sign), the
outward rounding of the ends, and a second enumeration written with numpy bit
views.
"""
import numpy as np
import pytest


def _bf16_values_numpy():
    b = (np.arange(65536, dtype=np.uint32) << 16).view(np.float32)
    v = np.unique(b[np.isfinite(b)].astype(np.float64))  # -0 == +0
    return v


@pytest.mark.parametrize("x,count", [
    ([1.0, 1.5], 65),                      # [1, 1.5], spacing 2^-7
    ([1.0, 4.0], 257),                     # 128 in [1,2) + 128 in [2,4) + 4
    ([0.75, 1.25], 97),                    # 64 in [0.75, 1) (spacing 2^-8) + 33 in [1, 1.25]
    ([-3.0, -2.5], 33),                    # [2, 4) spacing 2^-6 on the negative side
    ([-1.0, 1.0], 2 * (127 + 126 * 128 + 1) + 1),  # per sign: subnormals, binades 2^-126..2^-1, 1.0; one zero
    ([2.0, 2.0], 1),                       # a single value
])
def test_bf16_alphabet_closed_form_counts(O, x, count):
    P, n = O.bf16_alphabet(np.array(x, np.float32))
    assert n == count and P.size == count
    assert P[0] == min(x) and P[-1] == max(x)
    assert np.all(np.diff(P) > 0)
    f = P.astype(np.float32)
    assert np.array_equal(f.astype(np.float64), P)
    assert np.all((f.view(np.uint32) & 0xFFFF) == 0)  # BF16-representable
    assert np.sum(P == 0.0) <= 1


def test_bf16_alphabet_rounds_the_ends_outward(O):
    x = np.array([1.001, 1.3, 1.499], np.float32)
    P, n = O.bf16_alphabet(x)
    assert P[0] == 1.0 and P[-1] == 1.5 and n == 65
    x = np.array([-1.499, -1.001], np.float32)
    P, n = O.bf16_alphabet(x)
    assert P[0] == -1.5 and P[-1] == -1.0 and n == 65


@pytest.mark.parametrize("seed", range(6))
def test_bf16_alphabet_matches_a_numpy_enumeration(O, seed):
    rng = np.random.default_rng([43, seed])
    scale = 10.0 ** rng.uniform(-40, 3)
    shift = rng.uniform(-2, 2) * scale
    x = (shift + scale * rng.standard_normal(50)).astype(np.float32)
    allv = _bf16_values_numpy()
    lo = allv[allv <= float(x.min())].max()
    hi = allv[allv >= float(x.max())].min()
    ref = allv[(allv >= lo) & (allv <= hi)]
    P, n = O.bf16_alphabet(x, p_max=70000)
    assert n == ref.size
    assert np.array_equal(P, ref)


def test_bf16_alphabet_truncates_at_p_max(O):
    P, n = O.bf16_alphabet(np.array([-1.0, 1.0], np.float32), p_max=512)
    assert n == 32513 and P.size == 512
    full, _ = O.bf16_alphabet(np.array([-1.0, 1.0], np.float32))
    assert np.array_equal(P, full[:512])
