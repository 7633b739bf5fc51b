"""Build libtbq4.so (sm_100a) in-tree with nvcc.

    python long_context_attention_tbq4_b200/build.py [--force] [-v] [--debug]

(run it as a script, or load it by path: importing it through the package
would load the library it is about to rebuild).

The library is one translation unit (csrc/tbq4.cu) compiled for sm_100a only,
with -lineinfo for profiling and no fast-math (the quantiser must be
bit-exact).  The CUDA runtime is linked statically so the library does not
depend on which libcudart the host process carries.

--debug builds libtbq4_debug.so from the same sources with -DTBQ4_DEBUG: the
kernels then check every global access they derive from lengths, positions,
page ids or the split plan against its buffer's extent, and report a failed
check as TBQ4_ERR_BOUNDS.  The package loads it instead of libtbq4.so when
TBQ4_DEBUG=1 is set in the environment.
"""
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libtbq4.so")
LIB_DEBUG = os.path.join(PKG, "libtbq4_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-shared", "-Xcompiler", "-fPIC",
              "-Xcompiler", "-fvisibility=hidden", "--cudart", "static",
              "-Xptxas", "-warn-spills"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the TBQ4 library needs the CUDA toolkit to build")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + [os.path.join(INCLUDE, "tbq4.h")])


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    if not force and up_to_date(lib):
        return lib
    tmp = lib + ".tmp%d" % os.getpid()
    cmd = [nvcc(), *ARCH, *NVCC_FLAGS, *(["-DTBQ4_DEBUG"] if debug else []), "-I", INCLUDE,
           "-I", CSRC, os.path.join(CSRC, "tbq4.cu"), "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                debug="--debug" in sys.argv))
