"""Build the CUDA library libep_b200.so in-tree for B200 (sm_100a).

    python -m combine_ep_layout_10_b200.build [--force]

nvcc compiles every csrc/*.cu for sm_100a only (no PTX for other targets,
no fast-math: the FP8 scale and the combine's fma chain rely on IEEE
rounding) and links one shared library with the CUDA runtime linked
statically.  Cross-compiles without a GPU.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIBDIR = os.path.join(PKG, "lib")
LIB = os.path.join(LIBDIR, "libep_b200.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
    "-Xptxas", "-warn-spills",
    "-cudart", "static",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None,
          out: str | None = None) -> str:
    """Compile and link libep_b200.so (or `out`, e.g. a variant built with
    extra -D flags) if missing or stale; return its path."""
    target = out or LIB
    if not force and out is None and not _stale():
        return LIB
    os.makedirs(os.path.dirname(target), exist_ok=True)
    tmp = target + ".tmp.%d" % os.getpid()
    cmd = [nvcc(), *NVCC_FLAGS, *(extra or []), "-I", INCLUDE, "-I", CSRC, "-shared",
           *sources(), "-o", tmp]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("CUDA library build failed:\n%s\n%s%s" % (" ".join(cmd), res.stdout, res.stderr))
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(tmp, target)
    return target


if __name__ == "__main__":
    extra = ["-Xptxas", "-v"] if "-v" in sys.argv else []
    print(build(force="--force" in sys.argv or bool(extra), verbose=True, extra=extra))
