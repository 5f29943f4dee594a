"""Build libadmmq.so (sm_100a) in-tree with nvcc.

    python -m post_weight_quantization_10_b200.build [--verbose]

The library is compiled for sm_100a only and links cuSOLVER (the one-time
eigendecomposition) from the CUDA toolkit.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libadmmq.so")
SOURCES = ["admmq.cu"]
HEADERS = ["ptx.cuh", "gemm.cuh", "kernels.cuh", "admm_loop.cuh", "gptq.cuh"]
INCLUDE = os.path.join(os.path.dirname(HERE), "include", "admmq.h")


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [INCLUDE]
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> str:
    if not force and not _stale():
        return LIB
    nvcc = _nvcc()
    cuda_home = os.path.dirname(os.path.dirname(nvcc))
    libdir = os.path.join(cuda_home, "lib64")
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "-Xcompiler", "-fPIC,-O2", "-shared", "--expt-relaxed-constexpr",
           "-o", LIB + ".tmp"] + [os.path.join(CSRC, s) for s in SOURCES] + [
           "-L" + libdir, "-lcusolver", "-lcublas", "-Xlinker", "-rpath," + libdir]
    if ptxas_info:
        cmd += ["-Xptxas", "-v"]
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or res.returncode != 0:
        sys.stdout.write(res.stdout)
        sys.stderr.write(res.stderr)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed with exit code {res.returncode}")
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="--verbose" in sys.argv,
          ptxas_info="--ptxas" in sys.argv)
    print(LIB)
