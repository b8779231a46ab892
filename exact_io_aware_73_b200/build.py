"""Build ``libattn_b200.so`` (the C-ABI CUDA library) in-tree with nvcc.

sm_100a only: ``-gencode arch=compute_100a,code=sm_100a``.  The runtime is
linked statically, so the library needs only the NVIDIA driver at run time.
``--debug`` builds ``libattn_b200_debug.so`` instead: the same library with
the kernels' index checks compiled in (ATTN_DEBUG_BOUNDS), which report a
failed check through the device status word instead of making the access.
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
DEBUG_LIB = os.path.join(PKG, "libattn_b200_debug.so")
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


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    out = DEBUG_LIB if debug else LIB
    if (not force and os.path.exists(out) and
            os.path.getmtime(out) >= max(os.path.getmtime(p) for p in DEPS)):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = [nvcc()] + flags(verbose) + (["-DATTN_DEBUG_BOUNDS"] if debug else [])
    subprocess.run(cmd + SOURCES + ["-o", tmp], check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                debug="--debug" in sys.argv))
