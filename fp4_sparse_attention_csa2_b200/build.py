"""Build ``libcsa2.so`` (the CUDA library behind the C ABI in include/csa2.h)
in-tree with nvcc for sm_100a, and its debug variant ``libcsa2_debug.so``
(NVTX ranges per C-ABI call, device-side bounds checks on every position and
page: -DCSA2_NVTX -DCSA2_DEBUG_BOUNDS).

    python -m fp4_sparse_attention_csa2_b200.build [--force] [--debug]

No fast-math: the quantiser relies on IEEE binary32 division.  The binding
loads the debug variant when CSA2_LIBRARY=debug is set.
"""
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libcsa2.so")
LIB_DEBUG = os.path.join(HERE, "libcsa2_debug.so")
DEBUG_FLAGS = ["-DCSA2_NVTX", "-DCSA2_DEBUG_BOUNDS", "-ldl"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
    "-I", os.path.join(ROOT, "include"),
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib=LIB):
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
    deps.append(os.path.join(ROOT, "include", "csa2.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    if not force and not _stale(lib):
        return lib
    tmp = lib + ".tmp%d" % os.getpid()
    extra = ["-Xptxas", "-v"] if verbose else []
    cmd = [NVCC, *FLAGS, *(DEBUG_FLAGS if debug else []), *extra, *sources(), "-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
