"""Build the sm_100a shared library ``libmla_decode_b200.so`` in this directory.

    python -m decode_attention_latent_b200.build [--verbose-ptxas]

nvcc cross-compiles for sm_100a without a GPU.  The CUDA runtime is linked
statically, so the library depends only on the driver at run time.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SOURCES = [os.path.join(HERE, "csrc", "mla_decode.cu"), os.path.join(HERE, "csrc", "mla_merge.cu"),
           os.path.join(HERE, "csrc", "mla_naive.cu")]
HEADERS = [os.path.join(HERE, "csrc", "sm100_ptx.cuh"), os.path.join(ROOT, "include", "mla_decode.h")]
LIBRARY = os.path.join(HERE, "libmla_decode_b200.so")


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def command(output: str = LIBRARY, ptxas_verbose: bool = False) -> list:
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
           "-I", os.path.join(ROOT, "include"), "-o", output] + SOURCES
    if ptxas_verbose:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def up_to_date(output: str = LIBRARY) -> bool:
    if not os.path.exists(output):
        return False
    t = os.path.getmtime(output)
    return all(os.path.getmtime(s) <= t for s in SOURCES + HEADERS)


def build(force: bool = False, ptxas_verbose: bool = False, output: str = LIBRARY) -> str:
    if force or ptxas_verbose or not up_to_date(output):
        subprocess.run(command(output, ptxas_verbose), check=True)
    return output


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--force", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, ptxas_verbose=a.verbose_ptxas))
    sys.exit(0)
