"""Benchmark of the ECASQ solver hot path on B200.

One step = the whole path on one batch of synthetic vectors already in HBM:
uniform grid + bucketing -> DP solves (lambda bisection + time-sharing, or
fixed lambdas) -> stochastic-rounding encode -> empirical entropy.

Default workload: 4096 x 4096 weight-like rows (0.02 * Student-t, nu = 4),
p = 128, s = 16, budget b = 3.0 bits/entry, 30 bisection steps.

Metric: DP (k, l, j) triples per second over the whole step (triples counted
by formula, one solve = every triple the recurrence visits), with entries/s
and per-kernel roofline fractions alongside. The oracle (fp64 CPU) is timed
on a bounded sample of the same workload as the CPU baseline.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--fp64]
  python bench.py --impl reference ...   # the CPU oracle as the reference arm
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from entropy_constrained_unbiased_b200 import workloads as W  # noqa: E402

MUFU_LG2_PER_CLK_PER_SM = 16  # special-function unit results per clock per SM (sm_100)
METRIC = "ECASQ DP (k,l,j) triples/s"  # the same string in both arms
B200_SMS = 148

# DRAM bytes (read + write) per k_dp launch per row, from one ncu capture of
# k_dp on the first 296 rows of the weights workload (1.40 MB read, 1409 MB
# written, almost all of it the stored DP layers written back from L2), scaled
# by the rows of a launch. The figure belongs to the kernel source it was taken
# on; it is dropped (null) when that source has changed since.
DP_TRAFFIC = {"weights": {"bytes_per_row": (1403904 + 1409423616) / 296, "dp_source_sha1": "e0fddc885cc8318d"}}


def triples_per_solve(p: int, s: int) -> int:
    """(k, l, j) triples one exact solve evaluates: layer 2 has only k = 0
    (c_1 = P_0), layers 3 .. S-2 every k < l < j with k >= i-2, and the last
    layer S-1 only j = p-1."""
    S = min(s, p)
    t = 0
    for i in range(2, S):
        last = i == S - 1
        for l in range(i - 1, p - 1):
            K = 1 if i == 2 else l - i + 2
            NJ = 1 if last else p - 1 - l
            t += K * NJ
    return t


def _su(n: int) -> int:  # 1 + 2 + ... + n (0 for n <= 0)
    return n * (n + 1) // 2 if n > 0 else 0


def _sq(n: int) -> int:  # 1 + 4 + ... + n^2 (0 for n <= 0)
    return n * (n + 1) * (2 * n + 1) // 6 if n > 0 else 0


def pass_triples(s0: int, e0: int, T: int, last_only: bool) -> int:
    """(k, l, j) triples of one forward pass over the alphabet range s0..e0
    with T values from c_1 = P_s0: layer 2 has only k = s0; layer t >= 3 every
    s0 + t - 2 <= k < l < j <= e0 with l >= s0 + t - 1; the last layer only
    j = e0 when last_only. The whole-alphabet pass (0, p-1, S-1, True) is
    triples_per_solve(p, s)."""
    tot = 0
    for t in range(2, T + 1):
        last = last_only and t == T
        a, b = s0 + t - 1, e0 - 1  # rows l
        if a > b:
            continue
        if t == 2:
            tot += (b - a + 1) if last else _su(e0 - a) - _su(e0 - b - 1)
            continue
        kmin = s0 + t - 2
        ua, ub = a - kmin, b - kmin  # u = l - kmin >= 1: the k values of row l
        su = _su(ub) - _su(ua - 1)
        tot += su if last else (e0 - kmin) * su - (_sq(ub) - _sq(ua - 1))
    return tot


def hirschberg_triples(code, p: int, s: int) -> int:
    """Triples one Hirschberg-mode solve evaluates, given the code it found
    (indices into P, c_0 = 0 .. c_{m-1} = p-1): the whole-alphabet forward
    pass, then per segment (lo, hi) of unknown values c[lo+1 .. hi-1] with
    mid = lo + ceil((hi - lo - 1) / 2) a forward pass from c[lo] over
    c[lo] .. c[hi] with mid - lo + 1 values (only the last value c[hi] in its
    last layer when mid + 1 = hi) and a pass over the reflected range with
    hi - mid values; segments split at (c[mid], c[mid+1])."""
    S = min(s, p)
    tot = pass_triples(0, p - 1, S - 1, True)
    m = len(code)
    stack = [(0, m - 2)] if m >= 4 else []
    while stack:
        lo, hi = stack.pop()
        mid = lo + (hi - lo) // 2  # lo + ceil((hi - lo - 1) / 2)
        qlo, qhi = int(code[lo]), int(code[hi])
        tot += pass_triples(qlo, qhi, mid - lo + 1, mid + 1 == hi)
        tot += pass_triples(p - 1 - qhi, p - 1 - qlo, hi - mid, False)
        if mid - lo - 1 >= 1:
            stack.append((lo, mid))
        if hi - mid - 2 >= 1:
            stack.append((mid + 1, hi))
    return tot


def relaxations_per_solve(p: int, s: int) -> int:
    """(i, a, x) relaxations G_{i-1}(a) + w(a, x) one solve of the approximation's
    layered shortest path evaluates: layers i = 2 .. S, x = i-1 .. p-1, a = i-2 .. x-1."""
    S = min(s, p)
    return sum(x - i + 2 for i in range(2, S + 1) for x in range(i - 1, p))


SMEM_BYTES_PER_CLK_PER_SM = 128  # one 32-lane x 4-byte shared-memory wavefront per clock


def dp_traffic(w):
    import hashlib

    rec = DP_TRAFFIC.get(w.name)
    if rec is None:
        return None
    src = os.path.join(ROOT, "entropy_constrained_unbiased_b200", "csrc", "dp.cu")
    with open(src, "rb") as f:
        if hashlib.sha1(f.read()).hexdigest()[:16] != rec["dp_source_sha1"]:
            return None
    return rec["bytes_per_row"] * w.n


SPIN_CYCLES = 4_000_000  # about 2 ms of GPU clock


def device_ms(fn, stream, flush, reps=3, stat="mean"):
    """Mean (or median) device time (ms) of the launches fn makes, each rep
    after an L2 flush. A spin kernel queued before the first event keeps the
    stream busy while the host allocates and enqueues fn, so host overhead
    between the two events is not counted."""
    import torch

    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    out = []
    for k in range(reps):
        flush.fill_(k & 0xFF)
        torch.cuda._sleep(SPIN_CYCLES)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize()
        out.append(a.elapsed_time(b))
    return float(np.median(out) if stat == "median" else np.mean(out))


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f)
    except OSError:
        return {}


def describe(w: W.Workload) -> str:
    what = {"budget": f"budget b={w.b} bits/entry, {w.steps}-step lambda bisection + two-way time-sharing",
            "sweep": f"{w.n_lambda} log-spaced lambdas in [1e-4, 1]",
            "solve": f"fixed lambda={w.lam}"}[w.mode]
    return f"{w.name}: {w.n}x{w.d} fp32 ({w.dist}), uniform P p={w.p}, s={w.s}, {what}"


def solves_done(w: W.Workload, out) -> int:
    """DP solves actually executed, read from the solver's outputs."""
    if w.mode != "budget":
        return w.n * (w.n_lambda if w.mode == "sweep" else 1)
    st = out["status"].cpu().numpy()
    lam_hi = out["lambda_hi"].cpu().numpy()
    total = 0
    for r in range(w.n):
        if st[r] == 1:
            total += 2
        elif lam_hi[r] == 0.0:
            total += 1
        elif st[r] == 0:
            total += 2 + w.steps
    return total


class Clocks:
    """nvidia-smi sampling during the timed region."""

    def __init__(self, index: int):
        self.index = index
        self.rows = []
        self.proc = None

    def __enter__(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([c.strip() for c in line.split(",")])

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4) if len(r) > 5 + i and "Active" in r[5 + i]
                          and "Not" not in r[5 + i]})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.rows)}


# ---------------------------------------------------------------------------------

def run_ours(args, w: W.Workload, rank: int, world: int):
    import torch
    from entropy_constrained_unbiased_b200 import dist as D
    from entropy_constrained_unbiased_b200 import ecasq as E

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    E.load()
    fp64 = args.fp64
    X_host = W.make_inputs(w, rank=rank)
    X = torch.from_numpy(X_host).to(dev)
    n, d, p, s = w.n, w.d, w.p, w.s
    lam = torch.from_numpy(w.lambdas()).to(dev) if w.mode != "budget" else None
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # > 126 MB L2
    stream = torch.cuda.current_stream()

    def step(X):
        P, cnt, A, B, st = E.grid_bucket(X, p)
        ev_dp0.record(stream)
        if w.mode == "budget":
            out = E.solve_budget_stats(cnt, A, B, P, d, s, w.b, w.steps, fp64=fp64)
            ev_dp1.record(stream)
            idx, hist, est = E.encode(X, P, s, out["Q1"], out["Q1_len"], w.seed_encode, out["Q2"], out["Q2_len"],
                                      out["theta"])
        else:
            out = E.solve_stats(cnt, A, B, P, d, s, lam, fp64=fp64, hirschberg=w.hirschberg)
            ev_dp1.record(stream)
            Q = out["Q"][:, 0, :].contiguous()
            Ql = out["Q_len"][:, 0].contiguous()
            idx, hist, est = E.encode(X, P, s, Q, Ql, w.seed_encode)
        Hemp = E.entropy(hist)
        return out, idx, hist, Hemp

    ev_dp0 = torch.cuda.Event(enable_timing=True)
    ev_dp1 = torch.cuda.Event(enable_timing=True)
    unit_peaks = measure_unit_peaks()
    for _ in range(args.warmup):
        out, idx, hist, Hemp = step(X)
    torch.cuda.synchronize()
    n_solves = solves_done(w, out)
    tps = triples_per_solve(p, s)

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    dp_ms = []
    D.barrier()
    torch.cuda.synchronize()
    E.launch_count(reset=True)
    with Clocks(dev.index) as clk:
        for k in range(args.steps):
            flush.fill_(k & 0xFF)  # evict X and the tables from L2 between steps
            starts[k].record(stream)
            out, idx, hist, Hemp = step(X)
            ends[k].record(stream)
            torch.cuda.synchronize()
            dp_ms.append(ev_dp0.elapsed_time(ev_dp1))
    launches = E.launch_count(reset=True)
    step_ms = [starts[k].elapsed_time(ends[k]) for k in range(args.steps)]
    t_ms = D.max_over_ranks(float(sum(step_ms)))
    D.barrier()

    # e2e: same step through the C ABI with host buffers, copies inside the timed
    # region: pinned input, the step's results read back into pinned buffers;
    # one untimed pass (allocations), then as many timed steps as above
    Xpin = torch.from_numpy(X_host).pin_memory()
    keys = ("Q1", "Q2", "theta") if w.mode == "budget" else ()
    host_out = None
    e2e_ms = []
    for k in range(args.steps + 1):
        flush.fill_(k & 0xFF)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        Xd = Xpin.to(dev, non_blocking=True)
        o2, idx2, hist2, H2 = step(Xd)
        dev_out = [idx2, H2] + [o2[k2] for k2 in keys]
        if host_out is None:
            host_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in dev_out]
        for h, t in zip(host_out, dev_out):
            h.copy_(t, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        if k > 0:
            e2e_ms.append(e0.elapsed_time(e1))
    bo = n * d + n * 8 + (n * s * 4 * 2 + n * 8 if w.mode == "budget" else 0)

    peaks = measured_peaks()
    hbm = float(peaks.get("hbm_gbs", 6650.0))
    entries = n * d
    hbm_kernels = {}
    # Each stage alone, on the last step's data (device time, see device_ms)
    P_last, _ = E.uniform_grid(X, p)
    if w.mode == "budget":
        enc_args = (out["Q1"], out["Q1_len"], w.seed_encode, out["Q2"], out["Q2_len"], out["theta"])
    else:
        enc_args = (out["Q"][:, 0, :].contiguous(), out["Q_len"][:, 0].contiguous(), w.seed_encode)
    hbm_kernels.update(stage_figures(E, X, P_last, p, s, enc_args, stream, flush, hbm))
    hbm_kernels["input"] = f"this workload ({n} x {d})"
    sm_max = float(peaks.get("sm_max_mhz", 1965.0))
    mufu_peak = MUFU_LG2_PER_CLK_PER_SM * B200_SMS * sm_max * 1e6
    # The other workloads' exact solves, and the HBM-bound stages on the
    # gradients input (256 x 2^20 fp32 = 1 GiB, larger than L2) with codes from
    # the exact budget solver on it.
    dp_workloads = {}
    if w.name == "weights" and not args.no_other_workloads:
        hbm_kernels["gradients_input"], dp_workloads["gradients"] = gradients_figures(
            E, dev, stream, flush, hbm, mufu_peak, rank)
        dp_workloads.update(small_dp_figures(E, dev, stream, flush, mufu_peak, rank))
    large_alphabet = None
    if w.name == "weights" and not args.no_large_alphabet:
        large_alphabet = large_alphabet_figure(E, dev, stream, flush, rank)
    # hardware-aware alphabet (BF16 values covering each row), p_max = 512: one
    # read of X plus the alphabet rows written
    E.bf16_alphabet(X, 512)
    bf_bytes = entries * 4 + n * 512 * 8
    bf_t = device_ms(lambda: E.bf16_alphabet(X, 512), stream, flush)
    hbm_kernels["bf16_alphabet"] = {"ms": bf_t, "bytes": bf_bytes, "achieved_GBps": bf_bytes / (bf_t * 1e-3) / 1e9,
                                    "peak_GBps": hbm, "frac": bf_bytes / (bf_t * 1e-3) / 1e9 / hbm}
    # entropy coder on the last step's indices (rANS, per-row models from the
    # histogram), through the C ABI with its output buffers allocated once:
    # coded bits per entry against the empirical entropy
    import ctypes

    lib = E.load()
    th = out["theta"] if w.mode == "budget" else None
    nseg, cap = int(lib.ecasq_rans_segments(d)), int(lib.ecasq_rans_segment_words())
    words = torch.empty((n, nseg, cap), dtype=torch.int16, device=dev)
    seg_len = torch.empty((n, nseg), dtype=torch.int32, device=dev)
    rst = torch.empty(n, dtype=torch.int32, device=dev)

    def coder():
        rc = lib.ecasq_rans_encode(E._ptr(idx), E._ptr(hist), E._ptr(th), int(w.mode == "budget"), n, d, s,
                                   ctypes.c_uint64(w.seed_encode), E._ptr(words), E._ptr(seg_len), E._ptr(rst),
                                   E._stream())
        assert rc == 0, rc

    coder()
    rc_t = device_ms(coder, stream, flush)
    coded_bits = 16.0 * float(seg_len.sum().item())
    hbm_kernels["rans_encode"] = {"ms": rc_t, "entries_per_s": entries / (rc_t * 1e-3),
                                  "bits_per_entry": coded_bits / entries,
                                  "empirical_entropy_bits": float(Hemp.mean().item()),
                                  "bytes": entries + coded_bits / 8,
                                  "achieved_GBps": (entries + coded_bits / 8) / (rc_t * 1e-3) / 1e9, "peak_GBps": hbm,
                                  "frac": (entries + coded_bits / 8) / (rc_t * 1e-3) / 1e9 / hbm,
                                  "status_nonzero_rows": int((rst != 0).sum().item())}
    del words
    dp_avg_ms = float(np.mean(dp_ms))
    achieved = n_solves * tps / (dp_avg_ms * 1e-3)
    total_triples = world * n_solves * tps  # one step, all ranks
    value = total_triples * args.steps / (t_ms * 1e-3)
    approx, approx_outs = approx_timing(args, w, X, stream, flush, dp_avg_ms, sm_max)
    approx["vnmse"] = vnmse_report(w, X, out, approx_outs)
    if large_alphabet is not None:
        approx["large_alphabet"] = large_alphabet
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "triples/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": t_ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64" if fp64 else "f32",
        "data": "synthetic",
        "config": {"workload": describe(w), "n": n, "d": d, "p": p, "s": s, "l2": "flushed between steps",
                   "step": "uniform grid + bucketing + DP solves (bisection + time-sharing) + encode + entropy",
                   "dp_solves_per_step": n_solves, "triples_per_solve": tps,
                   "entries_per_s": world * n * d / (t_ms * 1e-3 / args.steps),
                   "parallelism": f"dp{world} (rows sharded, no collective)"},
        "roofline": {"bound": "alu", "kernel": "k_dp (DP layers + backtrack + bisection)", "achieved": achieved,
                     "peak": mufu_peak, "unit": "triples/s", "frac": achieved / mufu_peak, "traffic": dp_traffic(w),
                     "peak_basis": f"MUFU lg2 {MUFU_LG2_PER_CLK_PER_SM}/clk/SM x {B200_SMS} SMs x {sm_max:.0f} MHz "
                                   "(1 lg2 per triple)",
                     "measured_lg2_per_s": unit_peaks.get("lg2"),
                     "frac_of_measured_lg2": (achieved / unit_peaks["lg2"]) if unit_peaks.get("lg2") else None,
                     "measured_ffma_per_s": unit_peaks.get("ffma")},
        "e2e": {"value": total_triples / (float(np.mean(e2e_ms)) * 1e-3), "unit": "triples/s",
                "h2d_bytes_per_step": n * d * 4, "d2h_bytes_per_step": bo},
        "hbm_kernels": hbm_kernels,
        "dp_workloads": dp_workloads,
        "approx": approx,
        "gpu_launches": int(launches),
        "clocks": clk.summary(),
    }
    if w.hirschberg:
        ev = evaluated_triples(w, out)
        line["roofline"]["evaluated_triples_per_step"] = ev
        line["roofline"]["evaluated_frac"] = ev / (dp_avg_ms * 1e-3) / mufu_peak
        line["roofline"]["note"] = ("achieved/frac count the whole-alphabet pass; evaluated_* adds the divide and "
                                    "conquer's recovery passes")
    return line


def stage_figures(E, X, P, p, s, enc_args, stream, flush, hbm):
    """Device time of the uniform grid (min/max pass + grid), bucketing, the two
    in one call, encoding and the reconstruction, each call alone after an L2
    flush; algorithmic bytes: 4 B/entry read for the grid, for bucketing and for
    the combined call, 4 B read + 1 B written for encoding (the histograms are
    fused), 1 B read + 4 B written for the reconstruction."""
    entries = X.numel()
    idx, _, _ = E.encode(X, P, s, *enc_args)  # the reconstruction takes the encoder's arguments
    fns = {"grid": lambda: E.uniform_grid(X, p), "bucket": lambda: E.bucket(X, P),
           "grid_bucket": lambda: E.grid_bucket(X, p), "encode": lambda: E.encode(X, P, s, *enc_args),
           "dequantize": lambda: E.dequantize(idx, P, s, *enc_args)}
    out = {}
    # grid_bucket: the grid and bucketing in one call, one read of X (4 B/entry)
    # when rows fit in shared memory, else the two passes above (8 B/entry);
    # dequantize: 1 B of index read and 4 B of X^ written per entry
    for name, bpe in (("grid", 4), ("bucket", 4), ("grid_bucket", 4), ("encode", 5), ("dequantize", 5)):
        fns[name]()
        ms = device_ms(fns[name], stream, flush)
        gbs = entries * bpe / (ms * 1e-3) / 1e9
        out[name] = {"ms": ms, "bytes_per_entry": bpe, "achieved_GBps": gbs, "peak_GBps": hbm,
                     "frac": gbs / hbm, "entries_per_s": entries / (ms * 1e-3)}
    return out


def dp_figure(E, w: W.Workload, cnt, A, B, P, stream, flush, mufu_peak, reps=3):
    """Device time of one exact-solver call on a workload's bucket statistics
    (L2 flushed before each call; the median of the reps, so that one
    disturbed call does not move the figure) and its triples/s against the
    MUFU peak. Hirschberg's recovery passes are work the triple count leaves
    out."""
    import torch

    if w.mode == "budget":
        def call():
            return E.solve_budget_stats(cnt, A, B, P, w.d, w.s, w.b, w.steps)
    else:
        lam = torch.from_numpy(w.lambdas()).to(P.device)

        def call():
            return E.solve_stats(cnt, A, B, P, w.d, w.s, lam, hirschberg=w.hirschberg)
    out = call()
    torch.cuda.synchronize()
    ms = device_ms(call, stream, flush, reps=reps, stat="median")
    ns = solves_done(w, out)
    tps = triples_per_solve(w.p, w.s)
    ach = ns * tps / (ms * 1e-3)
    res = {"workload": describe(w), "ms": ms, "solves": ns, "triples_per_solve": tps, "achieved": ach,
           "frac": ach / mufu_peak, "status_nonzero_rows": int((out["status"] != 0).sum().item())}
    if w.hirschberg:
        ev = evaluated_triples(w, out)
        res["note"] = ("achieved/frac count the whole-alphabet pass only (the metric's triples); the "
                       "evaluated_* figures add the recovery passes of the divide and conquer")
        res["evaluated_triples"] = ev
        res["evaluated_achieved"] = ev / (ms * 1e-3)
        res["evaluated_frac"] = ev / (ms * 1e-3) / mufu_peak
    return res, out


def evaluated_triples(w: W.Workload, out) -> int:
    """Triples the Hirschberg-mode solves of a fixed-lambda call evaluated,
    from the codes they returned (rows with a nonzero status, lambda = 0 and
    constant rows are left out)."""
    Q = out["Q"].cpu().numpy()
    m = out["Q_len"].cpu().numpy()
    st = out["status"].cpu().numpy()
    lam = w.lambdas()
    tot = 0
    for r in range(Q.shape[0]):
        if st[r] != 0:
            continue
        for t in range(Q.shape[1]):
            if lam[r, t] > 0 and m[r, t] >= 2:
                tot += hirschberg_triples(Q[r, t, : m[r, t]], w.p, w.s)
    return tot


def gradients_figures(E, dev, stream, flush, hbm, mufu_peak, rank):
    """On the gradients input (256 x 2^20 fp32 = 1 GiB, larger than L2): the
    exact budget solve (k_dp) and the HBM-bound stages, with the codes of that
    solve for the encoder."""
    import torch

    g = W.WORKLOADS["gradients"]
    X = torch.from_numpy(W.make_inputs(g, rank=rank)).to(dev)
    P, _ = E.uniform_grid(X, g.p)
    cnt, A, B, _ = E.bucket(X, P)
    dp, o = dp_figure(E, g, cnt, A, B, P, stream, flush, mufu_peak)
    del cnt, A, B
    enc = (o["Q1"], o["Q1_len"], g.seed_encode, o["Q2"], o["Q2_len"], o["theta"])
    res = stage_figures(E, X, P, g.p, g.s, enc, stream, flush, hbm)
    res["input"] = f"gradients: {g.n} x {g.d} fp32, p={g.p}, s={g.s}, codes of the b={g.b} budget solve"
    del X, P, o
    torch.cuda.empty_cache()
    return res, dp


def large_alphabet_figure(E, dev, stream, flush, rank, n=148, d=65536, s=16):
    """The approximation on a hardware alphabet: rows covering [2^-16, 2^16],
    whose BF16 values there are 4097 (p > 512: pair terms from prefix sums,
    the tiled layer sweep); one fixed-lambda solve per row per call. Each pair
    cost (about 20 fp64 operations and two MUFU log2) is evaluated once per
    solve and relaxes the S - 1 layers."""
    import torch

    X = torch.from_numpy(W.pinned_range_rows(rank, n, d, 2.0 ** -16, 2.0 ** 16)).to(dev)
    Pd, p_len, st = E.bf16_alphabet(X, 8192)
    p = int(p_len[0].item())
    assert int(st.abs().sum()) == 0 and bool((p_len == p).all())
    P = Pd[:, :p].contiguous()
    cnt, A, B, st = E.bucket(X, P)
    assert int(st.abs().sum()) == 0
    lam = (X.double().var(dim=1, keepdim=True) * 0.01).contiguous()

    def call():
        return E.solve_approx_stats(cnt, A, B, P, d, s, lam)
    out = call()
    torch.cuda.synchronize()
    ms = device_ms(call, stream, flush, reps=2)
    pairs = p * (p - 1) // 2
    rel = relaxations_per_solve(p, s)
    res = {"rows": f"{n} x {d} fp32 covering [2^-16, 2^16]", "alphabet": "BF16 values", "p": p, "s": s,
           "ms": ms, "solves": n, "pairs_per_solve": pairs, "relaxations_per_solve": rel,
           "pairs_per_s": n * pairs / (ms * 1e-3), "relaxations_per_s": n * rel / (ms * 1e-3),
           "status_nonzero_rows": int((out["status"] != 0).sum().item())}
    del X, Pd, P, cnt, A, B, out
    torch.cuda.empty_cache()
    return res


def small_dp_figures(E, dev, stream, flush, mufu_peak, rank, names=("sweep", "mixture")):
    """k_dp on the lambda-sweep and Hirschberg workloads, each on its own input."""
    import torch

    res = {}
    for name in names:
        w = W.WORKLOADS[name]
        X = torch.from_numpy(W.make_inputs(w, rank=rank)).to(dev)
        P, cnt, A, B, _ = E.grid_bucket(X, w.p)
        res[name], _ = dp_figure(E, w, cnt, A, B, P, stream, flush, mufu_peak)
        del X, P, cnt, A, B
    torch.cuda.empty_cache()
    return res


def vnmse_report(w: W.Workload, X, exact, approx_out):
    """vNMSE = E||X^ - X||^2 / ||X||^2 per row (§4 "Precisão" reports the mean
    excess of the approximation and of its refinement over the optimum). Budget
    workloads compare the time-shared MSE at the same budget b; the exact and
    refined solvers constrain H(X^), the plain approximation H(I,B)."""
    import torch

    nx = X.double().pow(2).sum(dim=1)
    d = X.shape[1]

    def ts(o):
        if w.mode == "budget":
            th = o["theta"]
            return (th * o["mse1"] + (1.0 - th) * o["mse2"]) * d / nx
        return o["mse"][:, 0] * d / nx

    def rate(o):  # time-shared H(X^), bits per entry
        if w.mode == "budget":
            th = o["theta"]
            return th * o["H1"] + (1.0 - th) * o["H2"]
        return o["H"][:, 0]

    ve = ts(exact)
    ok = torch.isfinite(ve) & (ve > 0)
    res = {"definition": "d * MSE / ||x||^2 per row, mean over rows; rate_H = time-shared H(X^) in bits/entry",
           "exact": float(ve[ok].mean().item()), "exact_rate_H": float(rate(exact)[ok].mean().item())}
    for key, o in approx_out.items():
        va = ts(o)
        res[key] = float(va[ok].mean().item())
        res[f"{key}_rate_H"] = float(rate(o)[ok].mean().item())
        if w.mode == "budget":
            res[f"excess_{key}_over_exact"] = float((va[ok] / ve[ok] - 1.0).mean().item())
    if w.mode == "budget":
        res["note"] = ("at the same budget b the plain approximation constrains H(I,B) <= b, which leaves "
                       "H(X^) lower (H(I,B) <= H(X^) + 1); the refined one constrains H(X^) like the exact solver")
    res["pages_context"] = "mean excess 4.97% (approximation) and 1.37% (refined) on the pages' own inputs"
    return res


def approx_timing(args, w: W.Workload, X, stream, flush, dp_avg_ms: float, sm_max: float):
    """The approximation on H(I,B), plain and refined (8 iterations), on the same
    workload and bucket statistics as the exact solver above; CUDA events around
    the solver call alone, L2 flushed before each call. Roofline: every
    relaxation reads one 4-byte cost entry from shared memory (the G value is a
    broadcast), so at most 32 relaxations per clock per SM."""
    import torch
    from entropy_constrained_unbiased_b200 import ecasq as E

    fp64 = args.fp64
    P, _ = E.uniform_grid(X, w.p)
    cnt, A, B, _ = E.bucket(X, P)
    lam = torch.from_numpy(w.lambdas()).to(X.device) if w.mode != "budget" else None
    rps = relaxations_per_solve(w.p, w.s)
    peak = SMEM_BYTES_PER_CLK_PER_SM / 4 * B200_SMS * sm_max * 1e6
    res = {"kernel": "k_approx (layers + recovery + refinement + evaluation + bisection)",
           "relaxations_per_solve": rps, "bound": "smem", "peak": peak, "unit": "relaxations/s",
           "peak_basis": f"{SMEM_BYTES_PER_CLK_PER_SM} B/clk/SM shared memory / 4 B per relaxation x {B200_SMS} SMs "
                         f"x {sm_max:.0f} MHz"}

    def call(refine):
        if w.mode == "budget":
            return E.solve_approx_budget_stats(cnt, A, B, P, w.d, w.s, w.b, refine=refine, steps=w.steps, fp64=fp64)
        return E.solve_approx_stats(cnt, A, B, P, w.d, w.s, lam, refine=refine, fp64=fp64)

    outs = {}
    for refine in (0, 8):
        out = call(refine)  # warm-up
        outs["approx" if refine == 0 else "refined8"] = out
        torch.cuda.synchronize()
        t = device_ms(lambda: call(refine), stream, flush, reps=max(2, min(args.steps, 3)))
        ns = solves_done(w, out)
        ach = ns * rps / (t * 1e-3)
        res[f"refine{refine}"] = {"ms": t, "solves": ns, "achieved": ach, "frac": ach / peak,
                                  "speedup_vs_exact_dp": dp_avg_ms / t,
                                  "status_nonzero_rows": int((out["status"] != 0).sum().item())}
    return res, outs


def measure_unit_peaks():
    """MUFU lg2 and FFMA rates of this GPU from the microbenchmark library."""
    import ctypes

    from entropy_constrained_unbiased_b200 import build

    try:
        L = ctypes.CDLL(build.PEAKS_LIB)
    except OSError:
        return {}
    L.ecasq_peak_lg2_per_s.restype = ctypes.c_double
    L.ecasq_peak_ffma_per_s.restype = ctypes.c_double
    out = {"lg2": L.ecasq_peak_lg2_per_s(), "ffma": L.ecasq_peak_ffma_per_s()}
    return {k: v for k, v in out.items() if v > 0}


def oracle_sample(w: W.Workload, budget_s: float, stages: bool = True):
    """Time the fp64 oracle on a deterministic row sample of the workload: the
    exact DP solves (the metric), then, on the same rows, the other stages of
    the path (grid, bucketing, encoding with the solved codes, the
    approximation), so that each GPU stage has the oracle's rate beside it."""
    from oracle import oracle as O

    rows = 1
    X = W.make_inputs(w, rows=64 if w.n >= 64 else w.n)
    threads = O.threads()
    tps = triples_per_solve(w.p, w.s)
    done_rows, solves, t_tot = 0, 0, 0.0
    codes = []
    while done_rows < X.shape[0] and t_tot < budget_s:
        take = min(max(rows, threads), X.shape[0] - done_rows)
        Xs = np.ascontiguousarray(X[done_rows:done_rows + take])
        P, _ = O.grid_batch(Xs, w.p)
        t0 = time.perf_counter()
        if w.mode == "budget":
            r = O.solve_budget_batch(Xs, P, w.s, w.b, w.steps)
            st = r["status"]
            lam_hi = r["lam_hi"]
            solves += int(sum(2 if st[i] == 1 else (1 if lam_hi[i] == 0 else 2 + w.steps) for i in range(take)))
        else:
            lam = w.lambdas()[:take]
            r = O.solve_batch(Xs, P, w.s, lam)
            solves += take * lam.shape[1]
        t_tot += time.perf_counter() - t0
        codes.append(r)
        done_rows += take
    res = {"value": solves * tps / t_tot, "unit": "triples/s", "cores": threads, "kind": "oracle",
           "sample": f"first {done_rows} rows of {w.n} ({solves} fp64 DP solves, {t_tot:.1f} s)"}
    if not stages or done_rows == 0:
        return res
    Xs = np.ascontiguousarray(X[:done_rows])
    entries = Xs.size
    out = {}
    t0 = time.perf_counter()
    P, _ = O.grid_batch(Xs, w.p)
    out["grid"] = {"entries_per_s": entries / (time.perf_counter() - t0), "cores": threads}
    t0 = time.perf_counter()
    for i in range(done_rows):
        O.bucket(Xs[i], P[i])
    out["bucket"] = {"entries_per_s": entries / (time.perf_counter() - t0), "cores": 1}
    if w.mode == "budget":
        cat = {k: np.concatenate([c[k] for c in codes]) for k in ("Q1", "m1", "Q2", "m2", "theta")}
        t0 = time.perf_counter()
        O.encode_batch(Xs, P, cat["Q1"], cat["m1"], w.s, w.seed_encode, cat["Q2"], cat["m2"], cat["theta"])
    else:
        Q = np.concatenate([c["Q"][:, 0, :] for c in codes])
        m = np.concatenate([c["m"][:, 0] for c in codes])
        t0 = time.perf_counter()
        O.encode_batch(Xs, P, Q, m, w.s, w.seed_encode)
    out["encode"] = {"entries_per_s": entries / (time.perf_counter() - t0), "cores": threads}
    t0 = time.perf_counter()
    if w.mode == "budget":
        ra = O.solve_approx_budget_batch(Xs, P, w.s, w.b, w.steps)
        n_ap = int(sum(1 if ra["lam_hi"][i] == 0 else 2 + w.steps for i in range(done_rows)))
    else:
        O.solve_approx_batch(Xs, P, w.s, w.lambdas()[:done_rows])
        n_ap = done_rows * w.lambdas().shape[1]
    t_ap = time.perf_counter() - t0
    out["approx"] = {"relaxations_per_s": n_ap * relaxations_per_solve(w.p, w.s) / t_ap, "solves": n_ap,
                     "cores": threads}
    res["stages"] = out
    return res


def run_reference(args, w: W.Workload, rank: int, world: int):
    from oracle import oracle as O

    if rank != 0:
        return None
    per_step = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_sample(w, per_step / 4, stages=False)
    vals = []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        vals.append(oracle_sample(w, per_step, stages=False))
    wall = time.perf_counter() - t0
    v = float(np.mean([x["value"] for x in vals]))
    cb = dict(vals[-1])
    cb["value"] = v
    return {"impl": "reference", "metric": METRIC,
            "value": v, "unit": "triples/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": wall * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": describe(w), "n": w.n, "d": w.d, "p": w.p, "s": w.s,
                       "step": "fp64 CPU oracle on a row sample: grid + bucketing + DP solves"},
            "cpu_baseline": cb,
            "e2e": {"value": v, "unit": "triples/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="weights", choices=sorted(W.WORKLOADS))
    ap.add_argument("--fp64", action="store_true", help="fp64 DP layers (parity mode)")
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-other-workloads", action="store_true",
                    help="skip the exact-solver figures of the gradients, sweep and mixture workloads and the "
                         "grid/bucketing/encoding figures on the 1 GiB gradients input")
    ap.add_argument("--no-large-alphabet", action="store_true",
                    help="skip the approximation on a 4097-value BF16 alphabet")
    ap.add_argument("--rows", type=int, default=0, help="first rows only (profiling runs; not a bench line)")
    args = ap.parse_args()
    w = W.WORKLOADS[args.workload]
    if args.rows:
        import dataclasses

        w = dataclasses.replace(w, n=min(args.rows, w.n))

    from entropy_constrained_unbiased_b200 import dist as D

    rank, world = D.world()
    if world > 1 and args.impl == "ours":
        D.setup("nccl")
    if args.impl == "reference":
        line = run_reference(args, w, rank, world)
    else:
        # the oracle's thread pool starts before the first CUDA call
        cpu = None
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            cpu = oracle_sample(w, args.cpu_seconds)
        line = run_ours(args, w, rank, world)
        if cpu is not None:
            line["cpu_baseline"] = cpu
    if rank == 0 and line is not None:
        print(json.dumps(line))
    if world > 1 and args.impl == "ours":
        D.teardown()


if __name__ == "__main__":
    main()
