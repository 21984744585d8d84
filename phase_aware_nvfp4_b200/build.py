"""Build libmixquant.so (the CUDA library behind include/mixquant.h) for sm_100a.

    python -m phase_aware_nvfp4_b200.build [--verbose]

Compiles every ``csrc/*.cu`` with nvcc for ``sm_100a`` only (tcgen05 / TMA
instructions need the architecture-specific target) and links them into
``phase_aware_nvfp4_b200/libmixquant.so``, in the source tree, so the library
travels with the package.  Object files go to ``_build/``.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OUT = os.path.join(PKG, "libmixquant.so")
BUILD_DIR = os.path.join(ROOT, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
              "--expt-relaxed-constexpr", "-I" + os.path.join(ROOT, "include")]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libmixquant")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) +
                  glob.glob(os.path.join(ROOT, "include", "*.h")))


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(verbose: bool = False, force: bool = False) -> str:
    """Compile changed sources and link libmixquant.so; returns its path."""
    os.makedirs(BUILD_DIR, exist_ok=True)
    cc = nvcc()
    objs = []
    hdrs = headers()
    for src in sources():
        obj = os.path.join(BUILD_DIR, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if force or _stale(obj, [src] + hdrs):
            cmd = [cc, *ARCH, *NVCC_FLAGS, "-c", src, "-o", obj]
            if verbose:
                cmd += ["-Xptxas", "-v"]
                print(" ".join(cmd), flush=True)
            subprocess.check_call(cmd)
    if force or _stale(OUT, objs):
        # Exported symbols: the extern "C" mq_* functions (default visibility
        # is hidden for everything else).
        # The CUDA runtime is linked statically; the driver API (tensor-map
        # encoding) is reached through cudaGetDriverEntryPoint, so no -lcuda.
        cmd = [cc, *ARCH, "-shared", "-o", OUT + ".tmp", *objs]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.check_call(cmd)
        os.replace(OUT + ".tmp", OUT)
    return OUT


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--force", action="store_true")
    a = ap.parse_args(argv)
    path = build(verbose=a.verbose, force=a.force)
    print(path)


if __name__ == "__main__":
    sys.exit(main())
