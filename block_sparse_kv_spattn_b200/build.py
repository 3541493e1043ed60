"""Build libspattn.so (the CUDA library) in-tree for sm_100a.

    python -m block_sparse_kv_spattn_b200.build [--verbose]

One translation unit (csrc/spattn.cu) compiled by nvcc into a shared
library with the CUDA runtime linked statically; only the spattn_* C ABI
symbols declared in include/spattn.h are exported.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libspattn.so")
SOURCES = ["spattn.cu"]
DEPS = ["common.cuh", "compress.cuh", "scores.cuh", "select.cuh", "attention.cuh", "tcgen05.cuh",
        "attention_tc.cuh", "attention_tcw.cuh", "merge.cuh", "hca.cuh", "exports.map"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    files = [os.path.join(CSRC, f) for f in SOURCES + DEPS] + [os.path.join(INCLUDE, "spattn.h")]
    return any(os.path.getmtime(f) > t for f in files)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    cmd = [_nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-Xlinker", "--version-script=" + os.path.join(CSRC, "exports.map"),
           "-I", INCLUDE, "-o", LIB + ".tmp", *[os.path.join(CSRC, f) for f in SOURCES]]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv))
