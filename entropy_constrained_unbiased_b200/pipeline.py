"""One call from a batch of vectors to their quantised indices.

`quantize` composes the C ABI calls of the binding in the order of the
method ("Entropy-Constrained Adaptive Stochastic Quantization (ECASQ)",
gist.science/pt/paper/2608.18147, §1 "O Problema ECASQ" and §2):
- the alphabet: the uniform grid on each row's [min, max], or a given P;
- bucketing;
- the solver: exact or approximate, at a fixed λ or under an entropy budget
  with two-way time-sharing;
- stochastic-rounding encoding;
- the empirical entropy of the indices;
- on request (`Quantized.dequantize`), the reconstruction X^.

Every step runs in the library's kernels; this module only chooses the calls
and passes tensors between them. There is no CPU path.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

from . import ecasq as E


@dataclass
class Quantized:
    P: torch.Tensor             # [n, p] alphabet (fp64)
    Q1: torch.Tensor            # [n, s] code indices into P, -1 padded
    Q1_len: torch.Tensor        # [n]
    idx: torch.Tensor           # [n, d] uint8: position of each entry's value in its code
    hist: torch.Tensor          # [n, 2, s] index counts per time-sharing part
    H_emp: torch.Tensor         # [n] empirical entropy of idx, bits per entry
    Q2: torch.Tensor | None = None       # second code of a budget solve
    Q2_len: torch.Tensor | None = None
    theta: torch.Tensor | None = None    # [n] share of the entries coded with Q1
    stats: dict = field(default_factory=dict)  # the solver's fp64 figures (mse, H, lambda, ...)
    seed: int = 0

    def dequantize(self) -> torch.Tensor:
        """X^ [n, d] float32: each entry's value in the code its part used."""
        s = self.Q1.shape[1]
        Xh, st = E.dequantize(self.idx, self.P, s, self.Q1, self.Q1_len, self.seed, self.Q2, self.Q2_len,
                              self.theta)
        if int(st.abs().sum()) != 0:
            raise E.EcasqError(f"reconstruction rejected rows: {st.nonzero().flatten().tolist()[:8]}")
        return Xh


def quantize(X: torch.Tensor, p: int, s: int, *, b: float | None = None, lam: float | None = None,
             seed: int = 0, P: torch.Tensor | None = None, solver: str = "exact", refine: int = 0,
             fp64: bool = False, hirschberg: bool = False, steps: int = 30) -> Quantized:
    """Quantise the rows of X (float32 [n, d] on the GPU) to at most s values
    each, under an entropy budget b (bits per entry) or at a fixed λ (exactly
    one of the two).

    The alphabet is the uniform p-point grid on each row's range, or P
    (fp64 [n, p], ascending, covering each row). `solver` is "exact" (the
    pair-state DP) or "approx" (the layered shortest path on H(I,B), with
    `refine` refinement iterations). `seed` keys the Philox stream of the
    rounding and of the time-sharing partition.
    """
    if (b is None) == (lam is None):
        raise E.EcasqError("give exactly one of b (entropy budget) and lam (fixed lambda)")
    if solver not in ("exact", "approx"):
        raise E.EcasqError(f"solver must be 'exact' or 'approx', not {solver!r}")
    n, d = X.shape
    if P is None:
        P, cnt, A, B, st = E.grid_bucket(X, p)
    else:
        if P.shape != (n, p):
            raise E.EcasqError(f"P must be [{n}, {p}], got {list(P.shape)}")
        cnt, A, B, st = E.bucket(X, P)
    if int(st.abs().sum()) != 0:
        raise E.EcasqError(f"bucketing rejected rows: {st.nonzero().flatten().tolist()[:8]}")
    if b is not None:
        if solver == "exact":
            g = E.solve_budget_stats(cnt, A, B, P, d, s, b, steps=steps, fp64=fp64, hirschberg=hirschberg)
        else:
            g = E.solve_approx_budget_stats(cnt, A, B, P, d, s, b, refine=refine, steps=steps, fp64=fp64)
        idx, hist, est = E.encode(X, P, s, g["Q1"], g["Q1_len"], seed, g["Q2"], g["Q2_len"], g["theta"])
        out = Quantized(P=P, Q1=g["Q1"], Q1_len=g["Q1_len"], Q2=g["Q2"], Q2_len=g["Q2_len"], theta=g["theta"],
                        idx=idx, hist=hist, H_emp=E.entropy(hist), seed=seed)
        skip = ("Q1", "Q1_len", "Q2", "Q2_len", "theta")
    else:
        lam_t = torch.full((n, 1), float(lam), dtype=torch.float64, device=X.device)
        if solver == "exact":
            g = E.solve_stats(cnt, A, B, P, d, s, lam_t, fp64=fp64, hirschberg=hirschberg)
        else:
            g = E.solve_approx_stats(cnt, A, B, P, d, s, lam_t, refine=refine, fp64=fp64)
        Q1 = g["Q"][:, 0, :].contiguous()
        Q1_len = g["Q_len"][:, 0].contiguous()
        idx, hist, est = E.encode(X, P, s, Q1, Q1_len, seed)
        out = Quantized(P=P, Q1=Q1, Q1_len=Q1_len, idx=idx, hist=hist, H_emp=E.entropy(hist), seed=seed)
        skip = ("Q", "Q_len")
    if int(est.abs().sum()) != 0:
        raise E.EcasqError(f"encoding rejected rows: {est.nonzero().flatten().tolist()[:8]}")
    out.stats = {k: v for k, v in g.items() if k not in skip}
    return out
