"""Build the sm_100a shared library ``libsvdq.so`` in-tree with nvcc.

    python -m bit_quantized_diffusion_b200.build

The library is one translation unit (csrc/svdq.cu) exporting the C ABI of
include/svdq.h. The CUDA runtime is linked statically; the driver's
cuTensorMapEncodeTiled is looked up at run time, so no libcuda is needed at
link time.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libsvdq.so")
SOURCES = [os.path.join(PKG, "csrc", "svdq.cu")]
DEPS = SOURCES + [os.path.join(PKG, "csrc", f) for f in os.listdir(os.path.join(PKG, "csrc"))
                  if f.endswith(".cuh")] + [os.path.join(ROOT, "include", "svdq.h")]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def command(out: str = LIB, verbose_ptxas: bool = False) -> list[str]:
    cmd = [nvcc(), "-shared", "-Xcompiler", "-fPIC", "-O3", "-std=c++17",
           "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
           "-I", os.path.join(ROOT, "include"), "-o", out, *SOURCES]
    if verbose_ptxas:
        cmd[1:1] = ["-Xptxas", "-v"]
    return cmd


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in DEPS)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if force or not up_to_date():
        tmp = LIB + ".tmp"
        subprocess.run(command(tmp, verbose_ptxas), check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv)
    print(LIB)
