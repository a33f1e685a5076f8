"""Builds libfavor.so in this package directory (sm_100a only).

    python -m linear_attention_positive_b200.build

The CUDA translation unit (csrc/favor_api.cu, which includes the kernel files) is compiled by
nvcc for sm_100a; the host feature draw (csrc/features.cpp) by g++ without FMA contraction or
fast-math, so its floating-point steps stay exactly as written.
"""

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB = os.path.join(HERE, "libfavor.so")
BUILD = os.path.join(HERE, "_build")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-Xptxas", "-v",
]
GXX_FLAGS = ["-O2", "-fPIC", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-fvisibility=hidden"]


def _nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _run(cmd, log):
    proc = subprocess.run(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)
    log.append(" ".join(cmd) + "\n" + proc.stdout)
    if proc.returncode != 0:
        sys.stderr.write(proc.stdout)
        raise RuntimeError(f"build step failed: {' '.join(cmd[:3])} ...")


def build(verbose=False):
    """Compile csrc/ into libfavor.so; returns the library path. Writes _build/ptxas.log."""
    os.makedirs(BUILD, exist_ok=True)
    log = []
    feat_o = os.path.join(BUILD, "features.o")
    _run(["g++", *GXX_FLAGS, "-I", INCLUDE, "-c", os.path.join(CSRC, "features.cpp"), "-o", feat_o], log)
    api_o = os.path.join(BUILD, "favor_api.o")
    _run([_nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-c", os.path.join(CSRC, "favor_api.cu"), "-o", api_o], log)
    tmp = LIB + ".tmp"
    _run([_nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-Xcompiler", "-fPIC",
          api_o, feat_o, "-o", tmp], log)
    os.replace(tmp, LIB)
    with open(os.path.join(BUILD, "ptxas.log"), "w") as f:
        f.write("\n".join(log))
    if verbose:
        print("\n".join(log))
    return LIB


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv))
