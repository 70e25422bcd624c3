"""Build the sm_100a shared library ``libw4a4.so`` in-tree with nvcc.

    python -m bit_diffusion_transformer_nvfp4_b200.build [-v]

The library links the CUDA runtime dynamically (soname libcudart.so.12) so
that it shares the runtime instance, and with it the current device, with
PyTorch when both live in one process.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libw4a4.so")
SOURCES = ["w4a4_api.cu"]
DEPS = ["w4a4_api.cu", "attention.cuh", "gemm.cuh", "gemm2.cuh", "mma_rate.cuh", "quant.cuh", "sm100.cuh"]

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def command(out: str = LIB, extra=()) -> list[str]:
    cuda_home = os.path.dirname(os.path.dirname(nvcc_path()))
    return [nvcc_path(), *ARCH_FLAGS, "-lineinfo", "-O3", "-std=c++17", "--expt-relaxed-constexpr",
            "-shared", "-Xcompiler", "-fPIC", "-cudart", "shared",
            f"-I{os.path.join(ROOT, 'include')}",
            "-Xlinker", f"-rpath,{os.path.join(cuda_home, 'lib64')}",
            *extra, "-o", out, *[os.path.join(CSRC, s) for s in SOURCES]]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, d) for d in DEPS] + [os.path.join(ROOT, "include", "w4a4.h")]
    # every source in csrc/ counts, listed or not
    deps += [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh", ".h"))]
    return all(os.path.getmtime(d) <= t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    tmp = LIB + ".tmp.so"
    cmd = command(out=tmp)
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
    if verbose and (res.stdout or res.stderr):
        print(res.stdout, res.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="-v" in sys.argv)
    print(LIB)
