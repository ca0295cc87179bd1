"""Build the CUDA library libvsa.so in-tree for sm_100a (B200).

    python -m block_sparse_attention_30_b200.build [--force] [--debug-checks]

--debug-checks builds libvsa_debug.so instead: the same kernels compiled with
-DVSA_DEBUG_CHECKS, which also record non-finite outputs and TMA boxes outside
the grid in the workspace status word (reported as VSA_ERR_DEVICE_CHECK).

nvcc cross-compiles without a GPU; the shared library sits next to this
file so that it ships with the source tree.
"""
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libvsa.so")
DEBUG_LIB = os.path.join(HERE, "libvsa_debug.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return (sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
            + [os.path.join(ROOT, "include", "vsa.h")])


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _deps())


def build(force: bool = False, verbose: bool = False, debug_checks: bool = False) -> str:
    lib = DEBUG_LIB if debug_checks else LIB
    if not force and up_to_date(lib):
        return lib
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = lib + f".tmp{os.getpid()}"
    extra = ["-DVSA_DEBUG_CHECKS"] if debug_checks else []
    cmd = [nvcc, *ARCH, *FLAGS, *extra, "-shared", "-o", tmp, *sources(), "-I", os.path.join(ROOT, "include")]
    if verbose:
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, debug_checks="--debug-checks" in sys.argv))
