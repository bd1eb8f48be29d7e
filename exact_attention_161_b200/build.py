"""Build the CUDA library ``libattn_b200.so`` in-tree for sm_100a with nvcc.

The library is one translation unit (``csrc/attn_api.cu``) exporting the C ABI of
``include/attn.h``. The CUDA runtime is linked statically, so the library only needs the
NVIDIA driver at run time.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB = os.path.join(HERE, "libattn_b200.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh"))) + [
        os.path.join(INCLUDE, "attn.h")]


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile if the library is missing or older than any source; returns its path."""
    if not force and os.path.exists(LIB):
        newest = max(os.path.getmtime(s) for s in sources())
        if os.path.getmtime(LIB) >= newest:
            return LIB
    cmd = [NVCC, *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-shared",
           "-I", INCLUDE, os.path.join(CSRC, "attn_api.cu"), "-o", LIB + ".tmp"]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
