"""Build of the CUDA library (sm_100a) into the package directory: libfmoe.so."""
from __future__ import annotations

import os
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libfmoe.so")
SOURCES = ["engine.cu", "pack.cu", "api.cu"]
HEADERS = ["engine.h", "ptx.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _inputs():
    return ([os.path.join(CSRC, s) for s in SOURCES + HEADERS] + [os.path.join(INCLUDE, "fmoe.h")])


def stale(out: str = LIB) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(p) > t for p in _inputs())


def build(force: bool = False, nvcc: str = "nvcc", extra: list[str] | None = None,
          out: str = LIB, ptxas_log: str | None = None) -> str:
    """Compile every source for sm_100a with -lineinfo into one shared library."""
    if not force and not stale(out) and not extra:
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = [nvcc, "-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC", "-shared",
           "-I", INCLUDE, "-I", CSRC, *(extra or [])]
    if ptxas_log:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, s) for s in SOURCES] + ["-o", tmp, "-lcudart"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if ptxas_log:
        with open(ptxas_log, "w") as f:
            f.write(res.stdout + res.stderr)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    import sys
    print(build(force="--force" in sys.argv, ptxas_log="/dev/stdout" if "-v" in sys.argv else None))
