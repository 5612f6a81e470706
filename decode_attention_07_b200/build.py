"""Build libfdecode.so (the C-ABI library) for sm_100a with nvcc, in-tree."""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIBRARY = os.path.join(PKG, "libfdecode.so")
DEBUG_LIBRARY = os.path.join(PKG, "libfdecode_debug.so")   # -DFD_DEBUG: device-side bounds checks
HOST_BENCH = os.path.join(PKG, "fd_host_bench")   # host time per call through the C ABI (bench.py runs it)
SOURCES = [os.path.join(CSRC, "fd_api.cu"), os.path.join(CSRC, "fd_probe.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")] + \
    [os.path.join(INCLUDE, "fd.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "-shared", "-Xcompiler", "-fPIC,-fvisibility=hidden",
    "-cudart", "static",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    raise RuntimeError("nvcc not found")


def up_to_date(out: str) -> bool:
    if not os.path.exists(out):
        return False
    t = os.path.getmtime(out)
    return all(os.path.getmtime(d) <= t for d in DEPS)


def build_host_bench(force: bool = False) -> str:
    """The C++ program that times fd_decode's host side; linked against the
    in-tree libfdecode.so (found next to it at run time)."""
    src = os.path.join(CSRC, "fd_host_bench.cu")
    if not force and os.path.exists(HOST_BENCH) and os.path.getmtime(HOST_BENCH) >= max(
            os.path.getmtime(src), os.path.getmtime(LIBRARY)):
        return HOST_BENCH
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-std=c++17", "-I", INCLUDE, "-o",
           HOST_BENCH, src, "-L", PKG, "-lfdecode", "-Xlinker", "-rpath,$ORIGIN"]
    subprocess.run(cmd, check=True)
    return HOST_BENCH


def build(force: bool = False, verbose_ptxas: bool = False, out: str = None, debug: bool = False) -> str:
    out = out or (DEBUG_LIBRARY if debug else LIBRARY)
    if not force and up_to_date(out):
        return out
    cmd = [nvcc(), *NVCC_FLAGS, *(["-DFD_DEBUG"] if debug else []), "-I", INCLUDE, "-I", CSRC, "-o", out, *SOURCES]
    if verbose_ptxas:
        cmd[1:1] = ["-Xptxas", "-v"]
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    print(build(force=True, verbose_ptxas="-v" in sys.argv, debug="--debug" in sys.argv))
