"""Build libidx.so (CUDA for sm_100a behind the C ABI of include/idx.h).

Run ``python -m page_scoring_top_b200.build`` (or call :func:`build`).  The
library is built in-tree, next to this file, with static cudart, so it needs
nothing from the CUDA toolkit at run time beyond the driver.
"""

from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libidx.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")))


def _deps():
    return sources() + glob.glob(os.path.join(HERE, "csrc", "*.cuh")) + \
        glob.glob(os.path.join(HERE, "csrc", "*.h")) + [os.path.join(ROOT, "include", "idx.h")]


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in _deps())


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    """Compile every csrc/*.cu to an object (in parallel), then link libidx.so."""
    if not force and not stale():
        return LIB
    import concurrent.futures
    import tempfile
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    flags = ["-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC",
             "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
             "-I", os.path.join(ROOT, "include"), *extra]
    with tempfile.TemporaryDirectory(prefix="idx_build_") as tmpdir:
        def compile_one(src):
            obj = os.path.join(tmpdir, os.path.basename(src) + ".o")
            cmd = [nvcc, *flags, "-c", src, "-o", obj]
            if verbose:
                print(" ".join(cmd), file=sys.stderr)
            subprocess.check_call(cmd)
            return obj
        srcs = sources()
        with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
            objs = list(ex.map(compile_one, srcs))
        tmp = LIB + ".tmp%d" % os.getpid()
        subprocess.check_call([nvcc, "-shared", *ARCH, *objs, "-o", tmp])
        os.replace(tmp, LIB)
    return LIB

if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [])
