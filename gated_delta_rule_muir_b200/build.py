"""Build libmuir.so in-tree for B200 (sm_100a) with nvcc (cross-compiles without a GPU)."""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libmuir.so")
# the checking build: the same library with device-side index checks (-DMUIR_CHECK)
CHECK_LIB = os.path.join(PKG, "libmuir_check.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC,-O2",
    "--expt-relaxed-constexpr",
]


def sources() -> list[str]:
    out = []
    for d in (CSRC, os.path.join(ROOT, "include")):
        for f in sorted(os.listdir(d)):
            if f.endswith((".cu", ".cuh", ".h", ".inc")):
                out.append(os.path.join(d, f))
    return out


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in sources())


def _start(lib: str, extra: list[str], verbose: bool):
    nvcc = os.environ.get("NVCC", "nvcc")
    cmd = [nvcc, *NVCC_FLAGS, *extra, "-o", lib + ".tmp", os.path.join(CSRC, "muir.cu")]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    return subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)


def _finish(proc, lib: str, verbose: bool) -> None:
    out, err = proc.communicate()
    if proc.returncode != 0:
        raise RuntimeError(f"nvcc failed ({proc.returncode}):\n{out}\n{err}")
    if verbose and (out or err):
        print(out + err, file=sys.stderr)  # e.g. the -Xptxas -v report
    os.replace(lib + ".tmp", lib)


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None, check: bool = False) -> str:
    """Build libmuir.so (and, with check=True, libmuir_check.so at the same time)."""
    jobs = []
    if force or needs_build(LIB):
        jobs.append((LIB, _start(LIB, list(extra or []), verbose)))
    if check and (force or needs_build(CHECK_LIB)):
        jobs.append((CHECK_LIB, _start(CHECK_LIB, [*(extra or []), "-DMUIR_CHECK"], verbose)))
    for lib, proc in jobs:
        _finish(proc, lib, verbose)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None, check="--check" in sys.argv)
    print(LIB)
