"""Build libfa.so (the C-ABI attention library) in-tree for sm_100a.

    python exact_attention_149_b200/build.py [--force] [-v]

(run it as a script: importing the package would first bind the existing
library, which may be stale).

The library is one translation unit (csrc/fa_api.cu includes every kernel
header), compiled with nvcc for sm_100a only and linked against the static
CUDA runtime, so the .so loads on a machine without a GPU (host-only checks
and symbol inspection work there) and needs only the driver on a B200.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libfa.so")
ROOT = os.path.dirname(HERE)


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    out = []
    for fn in sorted(os.listdir(CSRC)):
        if fn.endswith((".cu", ".cuh", ".inc", ".h")):
            out.append(os.path.join(CSRC, fn))
    out.append(os.path.join(ROOT, "include", "fa.h"))
    return out


def is_stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(s) > t for s in sources())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not is_stale():
        return LIB
    cmd = [
        nvcc_path(),
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-lineinfo", "-O3", "-std=c++17",
        "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
        "-cudart", "static",
        "-I", os.path.join(ROOT, "include"),
        "-o", LIB + ".tmp",
        os.path.join(CSRC, "fa_api.cu"),
    ]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
