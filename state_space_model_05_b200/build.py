"""Build the SSD C-ABI library (libssd.so) in-tree for sm_100a with nvcc.

    python -m state_space_model_05_b200.build [--force] [--verbose-ptxas]
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libssd.so")
GEN_LIB = os.path.join(HERE, "libssd_inputs.so")
GEN_SRC = os.path.join(CSRC, "gen", "gen_inputs.cu")

SOURCES = ["api.cu", "decode.cu", "gdn_decode.cu", "prefill_simt.cu", "prefill_tc.cu", "prefill_fused.cu",
           "prefill_noalloc.cu", "selftest.cu"]
HEADERS = ["common.cuh", "ptx.cuh", "prefill_tc.h"]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _inputs():
    files = [os.path.join(CSRC, s) for s in SOURCES + HEADERS]
    files.append(os.path.join(INCLUDE, "ssd.h"))
    return files


def stale(target: str = LIB) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(f) > t for f in _inputs())


def build_inputs(force: bool = False) -> str:
    """The seeded device input generator (random draws only), a library of its own."""
    deps = [GEN_SRC, os.path.join(INCLUDE, "ssd_inputs.h")]
    if force or not os.path.exists(GEN_LIB) or any(os.path.getmtime(f) > os.path.getmtime(GEN_LIB) for f in deps):
        subprocess.check_call([nvcc(), *ARCH, "-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-shared",
                               "-I", INCLUDE, "-o", GEN_LIB + ".tmp", GEN_SRC])
        os.replace(GEN_LIB + ".tmp", GEN_LIB)
    return GEN_LIB


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    build_inputs(force)
    if not force and not stale():
        return LIB
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-shared",
           "-I", INCLUDE, "-I", CSRC, "-o", LIB + ".tmp"]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    subprocess.check_call(cmd)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, ptxas_verbose="--verbose-ptxas" in sys.argv)
    print(LIB)
