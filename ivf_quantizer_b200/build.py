"""Build the in-tree CUDA library ``_fgmm.so`` for sm_100a with nvcc.

Usage: ``python ivf_quantizer_b200/build.py`` (or ``__graft_entry__.build()``); run it
as a file, not through the package, whose import loads the library it builds.
Cross-compiles without a GPU; the result is loaded by ``ivf_quantizer_b200._lib``.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
OUT = os.path.join(HERE, "_fgmm.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC,-O3",
         "--expt-relaxed-constexpr", "-Xptxas", "-v"]


def nvcc_path() -> str:
    p = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(p):
        raise RuntimeError("nvcc not found")
    return p


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def build(verbose: bool = False, out: str = OUT) -> str:
    cmd = [nvcc_path(), *ARCH, *FLAGS, "-I", os.path.join(HERE, "..", "include"),
           *sources(), "-o", out + ".tmp"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    log = r.stdout + r.stderr
    with open(os.path.join(HERE, "_build_ptxas.log"), "w") as f:
        f.write(log)
    if r.returncode != 0:
        sys.stderr.write(log)
        raise RuntimeError("nvcc failed")
    if verbose:
        sys.stderr.write(log)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv))
