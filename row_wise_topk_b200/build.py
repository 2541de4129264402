"""Builds the in-tree CUDA library ``libdsel.so`` for sm_100a with nvcc.

Run ``python row_wise_topk_b200/build.py [--force] [--stats] [-v]`` (or call :func:`build`).  The library is
written next to this file so it travels with the source tree.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libdsel.so")
STATS_LIB = os.path.join(HERE, "libdsel_stats.so")   # same library, with per-CTA counters
SOURCES = ["dsel_api.cu", "dsel_plan.cpp", "dsel_shard.cu"]
HEADERS = ["dsel_device.cuh", "dsel_kernels.cuh", "dsel_plan.h", "dsel_resident.cuh", "dsel_slice.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc():
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    path = os.path.join(cuda, "bin", "nvcc")
    return path if os.path.exists(path) else "nvcc"


def _stale(lib):
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(HERE, "..", "include", "dsel.h"))
    deps.append(os.path.abspath(__file__))
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


def build(force=False, verbose=False, extra=(), stats=False):
    lib = STATS_LIB if stats else LIB
    if not force and not _stale(lib):
        return lib
    extra = list(extra) + (["-DDSEL_STATS"] if stats else [])
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
           "-o", lib + ".tmp", *[os.path.join(CSRC, f) for f in SOURCES], *extra]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building libdsel.so")
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    out = build(force="--force" in sys.argv, verbose="-v" in sys.argv, stats="--stats" in sys.argv)
    print(out)
