"""Build libgradsolve.so in-tree with nvcc for sm_100a.

The forward replay relies on the floating-point contract (explicit fused
multiply-adds only), so every translation unit is compiled with -fmad=false.
"""
from __future__ import annotations

import glob
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libgradsolve.so")
SOURCES = sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")))
HEADERS = sorted(glob.glob(os.path.join(HERE, "csrc", "*.cuh")) + glob.glob(os.path.join(ROOT, "include", "*.h")))

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-fmad=false", "-std=c++17",
              "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-I", os.path.join(ROOT, "include")]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in SOURCES + HEADERS + [__file__])


def build(force: bool = False, verbose: bool = False, extra_flags: list[str] | None = None) -> str:
    """Compile every csrc/*.cu and link libgradsolve.so (skipped when fresh).
    extra_flags: additional nvcc flags (e.g. -D tuning macros) for a forced
    rebuild."""
    if not force and not extra_flags and not stale():
        return LIB
    from concurrent.futures import ThreadPoolExecutor

    objdir = os.path.join(ROOT, "_build")
    os.makedirs(objdir, exist_ok=True)
    cmds, objs = [], []
    for src in SOURCES:
        obj = os.path.join(objdir, os.path.basename(src)[:-3] + ".o")
        cmds.append([_nvcc(), *NVCC_FLAGS, *(extra_flags or []), "-c", src, "-o", obj])
        objs.append(obj)
        if verbose:
            print(" ".join(cmds[-1]))
    # one nvcc per translation unit, in parallel; any failure raises
    with ThreadPoolExecutor(max_workers=max(1, min(len(cmds), os.cpu_count() or 1))) as pool:
        for fut in [pool.submit(subprocess.run, c, check=True) for c in cmds]:
            fut.result()
    tmp = LIB + ".tmp"
    subprocess.run([_nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-cudart", "static",
                    "-o", tmp, *objs], check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    import sys
    print(build(force=True, verbose=True, extra_flags=sys.argv[1:]))
