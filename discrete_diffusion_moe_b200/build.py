"""Build of the in-tree CUDA library libdg.so (sm_100a) with nvcc.

nvcc cross-compiles for sm_100a without a GPU.  The library is rebuilt only
when a source or header is newer than the built file.
"""

import glob
import os
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libdg.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-shared"]


def sources():
    return [os.path.join(PKG, "csrc", "dg_api.cu"), os.path.join(ROOT, "synth", "synth_device.cu")]


def deps():
    return (sources() + glob.glob(os.path.join(PKG, "csrc", "*.cuh"))
            + glob.glob(os.path.join(ROOT, "include", "*.h")) + [os.path.join(ROOT, "synth", "synth.h")])


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in deps())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [NVCC, *ARCH_FLAGS, *CFLAGS, "-o", tmp, *sources()]
    if verbose:
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose=True))
