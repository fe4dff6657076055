"""Mutation sampling of the fp64 CPU oracle against its CPU pins (test tooling).

Usage:  python tests/oracle_mutants.py --n 200 --seed 7 [--jobs 8] [--out FILE]

Each mutant changes one operator or constant on one code line of the oracle's
C++ sources (+ <-> -, < <-> <=, > <-> >=, == <-> !=, && -> ||, * -> /, x + 1 or
x - 1 -> x, 1.0 -> 2.0) in a copy under a temporary folder, builds it as a
shared library and runs every oracle pin file against it; the oracle under
oracle/ is not touched. A mutant is "killed" when a pin fails (or the run
times out), "survived" when every pin passes, "nocompile" when the change does
not build. Survivors are either equivalent (a buffer sized larger, an initial
value that is always overwritten, a comparison at a value that clamps to the
same result) or a gap in the pins; the report lists them with their lines.
One JSON object per mutant goes to --out (default: stdout), then a summary.
"""
import argparse
import json
import os
import random
import re
import shutil
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRCS = ["ecasq_oracle.cpp", "ecasq_approx_oracle.cpp", "ecasq_rans_oracle.cpp"]
PINS = ["tests/test_oracle_pins.py", "tests/test_oracle_approx_pins.py", "tests/test_oracle_alphabet_pins.py",
        "tests/test_oracle_dequantize_pins.py", "tests/test_oracle_rans_pins.py", "tests/test_oracle_edge_pins.py"]
OPS = [(r"(?<![+\-<>=!&|*/])\+(?![+=])", "-"), (r"(?<![+\-<>=!&|*/])-(?![\-=>])", "+"),
       (r"<(?![<=])", "<="), (r"<=", "<"), (r">(?![>=])", ">="), (r">=", ">"),
       (r"\+ 1\b", ""), (r"- 1\b", ""), (r"\b1\.0\b", "2.0"), (r"\*", "/"), (r"==", "!="), (r"&&", "||")]
SIGNATURE = re.compile(r"^(static |inline |double |int |void |uint|int64_t |size_t |bool |struct |template)")


def code_lines(src):
    """Indices of the lines that hold code (no comments, preprocessor lines,
    namespace or linkage lines, or function signatures)."""
    out, in_block = [], False
    for i, ln in enumerate(src.splitlines()):
        s = ln.strip()
        if in_block:
            in_block = "*/" not in s
            continue
        if s.startswith("/*"):
            in_block = "*/" not in s
            continue
        if not s or s.startswith(("//", "#", "extern", "namespace")):
            continue
        if SIGNATURE.match(s) and s.endswith("{") and "(" in s and "=" not in s:
            continue
        out.append(i)
    return out


def candidates():
    cands = []
    for f in SRCS:
        lines = open(os.path.join(ROOT, "oracle", f)).read().splitlines()
        for i in code_lines("\n".join(lines)):
            code = lines[i].split("//")[0]
            for pat, rep in OPS:
                for m in re.finditer(pat, code):
                    cands.append((f, i, m.start(), m.end(), rep))
    return cands


def run_one(cand, timeout):
    f, i, a, b, rep = cand
    d = tempfile.mkdtemp(prefix="oracle_mutant_")
    try:
        for g in SRCS:
            shutil.copy(os.path.join(ROOT, "oracle", g), d)
        path = os.path.join(d, f)
        lines = open(path).read().splitlines()
        orig = lines[i]
        lines[i] = orig[:a] + rep + orig[b:]
        open(path, "w").write("\n".join(lines) + "\n")
        lib = os.path.join(d, "liboracle_mutant.so")
        r = subprocess.run(["g++", "-O1", "-std=c++17", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-fPIC",
                            "-shared", "-w", "-o", lib] + [os.path.join(d, g) for g in SRCS],
                           capture_output=True, text=True)
        res = {"file": f, "line": i + 1, "orig": orig.strip(), "mutant": lines[i].strip()}
        if r.returncode != 0:
            return dict(res, status="nocompile")
        # the pins load the oracle through oracle.build.build(): point it at the mutant
        code = ("import sys; sys.path.insert(0, %r); import oracle.build as ob; "
                "ob.build = lambda force=False: %r; import pytest; "
                "sys.exit(pytest.main(['-q', '-x', '-p', 'no:cacheprovider'] + %r))"
                % (ROOT, lib, [os.path.join(ROOT, t) for t in PINS]))
        try:
            t = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=timeout,
                               cwd=ROOT, env=dict(os.environ, OMP_NUM_THREADS="1"))
            return dict(res, status="killed" if t.returncode != 0 else "survived")
        except subprocess.TimeoutExpired:
            return dict(res, status="killed")
    finally:
        shutil.rmtree(d, ignore_errors=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--n", type=int, default=200)
    ap.add_argument("--seed", type=int, default=7)
    ap.add_argument("--jobs", type=int, default=os.cpu_count() or 4)
    ap.add_argument("--timeout", type=int, default=240)
    ap.add_argument("--out", default=None)
    args = ap.parse_args()
    cands = candidates()
    random.Random(args.seed).shuffle(cands)
    sel = cands[:args.n]
    out = open(args.out, "w") if args.out else sys.stdout
    counts = {}
    survivors = []
    with ThreadPoolExecutor(args.jobs) as ex:
        for res in ex.map(lambda c: run_one(c, args.timeout), sel):
            print(json.dumps(res), file=out, flush=True)
            counts[res["status"]] = counts.get(res["status"], 0) + 1
            if res["status"] == "survived":
                survivors.append(res)
    print(json.dumps({"candidates": len(cands), "sampled": len(sel), "seed": args.seed, **counts}), file=sys.stderr)
    for r in survivors:
        print("survived %s:%d  %s  ->  %s" % (r["file"], r["line"], r["orig"], r["mutant"]), file=sys.stderr)


if __name__ == "__main__":
    main()
