"""Build libecasq.so (sm_100a) in-tree with nvcc."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libecasq.so")
PEAKS_LIB = os.path.join(HERE, "libecasq_peaks.so")
SOURCES = ["api.cu", "dp.cu", "approx.cu", "grid_bucket.cu", "encode.cu", "rans.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(ROOT, "include", "ecasq.h")]
    return any(os.path.getmtime(f) > t for f in deps)


def build_peaks(force: bool = False) -> str:
    """Microbenchmarks of the MUFU lg2 and FFMA rates (measurement tooling)."""
    if not force and not _stale(PEAKS_LIB):
        return PEAKS_LIB
    subprocess.run(["nvcc", *ARCH, "-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "-o", PEAKS_LIB,
                    os.path.join(CSRC, "peaks.cu")], check=True)
    return PEAKS_LIB


def build(force: bool = False, verbose: bool = False) -> str:
    build_peaks(force)
    if not force and not _stale():
        return LIB
    cmd = ["nvcc", *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-shared",
           "-I", os.path.join(ROOT, "include"), "-o", LIB]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, f) for f in SOURCES]
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    import sys
    print(build(force=True, verbose="-v" in sys.argv))
