"""Build libplora.so (the C-ABI library with its sm_100a kernels) in-tree with nvcc, and its
PLORA_DEBUG variant libplora_debug.so (device-side bounds checks in every kernel)."""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libplora.so")
DEBUG_LIB = os.path.join(HERE, "libplora_debug.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

SOURCES = ["plora.cu"]
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-shared",
         "-cudart", "static", "--expt-relaxed-constexpr"]


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(ROOT, "include", "plora.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(lib: str, defines=(), verbose: bool = False, extra=()) -> None:
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [NVCC, *FLAGS, *defines, *extra, *[os.path.join(CSRC, s) for s in SOURCES], "-o", tmp, "-ldl"]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)


def build(force: bool = False, verbose: bool = False, extra=(), debug: bool = True) -> str:
    """Build the release library (and, with debug=True, the PLORA_DEBUG one) if a source is newer."""
    if force or _stale(LIB):
        _compile(LIB, verbose=verbose, extra=extra)
    if debug and (force or _stale(DEBUG_LIB)):
        _compile(DEBUG_LIB, defines=["-DPLORA_DEBUG"], verbose=verbose, extra=extra)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True, debug="--no-debug" not in sys.argv,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [])
