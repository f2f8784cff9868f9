"""Builds libtq.so in-tree with nvcc for sm_100a (no GPU needed to compile).

Each source compiles to an object under _build/ in parallel; one nvcc call then
links the shared library.
"""

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJ = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libtq.so")
SOURCES = ["tq_codec.cpp", "tq_pack.cu", "tq_pack_mma.cu", "tq_decode.cu", "tq_decode_mma.cu", "tq_decode_static.cu"]
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC"]


def nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    raise RuntimeError("nvcc not found")


def build(verbose: bool = False, ptxas_info: bool = False) -> str:
    os.makedirs(OBJ, exist_ok=True)
    nv = nvcc()
    objs = [os.path.join(OBJ, os.path.splitext(s)[0] + ".o") for s in SOURCES]

    def compile_one(i):
        cmd = [nv, *FLAGS, "-I", INCLUDE, "-I", CSRC, "-c", os.path.join(CSRC, SOURCES[i]), "-o", objs[i]]
        if ptxas_info:
            cmd += ["-Xptxas", "-v"]
        if verbose:
            print(" ".join(cmd))
        return subprocess.run(cmd, capture_output=True, text=True)

    with ThreadPoolExecutor(max_workers=len(SOURCES)) as pool:
        results = list(pool.map(compile_one, range(len(SOURCES))))
    for src, res in zip(SOURCES, results):
        sys.stdout.write(res.stdout)
        sys.stderr.write(res.stderr)
        if res.returncode != 0:
            raise subprocess.CalledProcessError(res.returncode, f"nvcc {src}")
    link = [nv, *FLAGS, "-shared", "-o", LIB, *objs]
    if verbose:
        print(" ".join(link))
    subprocess.run(link, check=True)
    return LIB


if __name__ == "__main__":
    build(verbose=True, ptxas_info="-v" in sys.argv)
