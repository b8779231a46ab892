"""Build ``libattn_b200.so`` (the C-ABI CUDA library) in-tree with nvcc.

sm_100a only: ``-gencode arch=compute_100a,code=sm_100a``.  The runtime is
linked statically, so the library needs only the NVIDIA driver at run time.
"""
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libattn_b200.so")
SOURCES = [os.path.join(CSRC, "attn_api.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [
    os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE)]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def flags(verbose: bool = False):
    f = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
         "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "-I", INCLUDE, "-I",
         CSRC, "-cudart", "static"]
    if verbose:
        f += ["-Xptxas", "-v"]
    return f


def build(force: bool = False, verbose: bool = False) -> str:
    if (not force and os.path.exists(LIB) and
            os.path.getmtime(LIB) >= max(os.path.getmtime(p) for p in DEPS)):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc()] + flags(verbose) + SOURCES + ["-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
