"""Build ``libsv.so`` (the C-ABI CUDA library) in-tree for sm_100a.

    python -m speculative_decoding_verification_93_b200.build [--force]

nvcc cross-compiles without a GPU.  The CUDA runtime is linked statically so
the library does not depend on which libcudart the host process loaded.
"""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libsv.so")
SOURCES = [os.path.join(CSRC, f) for f in ("sv_api.cu", "sv_verify.cu", "sv_admit.cu",
                                           "sv_sts.cu", "sv_vocab.cu", "sv_hostio.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in ("sv_device.cuh", "sv_host.h")] + \
    [os.path.join(INCLUDE, "sv.h")]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-shared", "-cudart", "static", "-I" + INCLUDE, "-I" + CSRC]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in DEPS)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    cmd = [NVCC] + FLAGS + (["-Xptxas", "-v"] if verbose else []) + SOURCES + ["-o", LIB + ".tmp"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
