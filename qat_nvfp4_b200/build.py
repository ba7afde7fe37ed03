"""Build libnvfp4.so in-tree with nvcc for sm_100a.

    python -m qat_nvfp4_b200.build [--force]

The library is the C ABI of include/nvfp4.h; the CUDA runtime is linked statically, so
the .so depends only on the driver (libcuda) and the C/C++ runtime.
"""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libnvfp4.so")
SOURCES = [os.path.join(CSRC, "nvfp4_kernels.cu"), os.path.join(CSRC, "nvfp4_w4a16.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in ("nvfp4_device.cuh", "nvfp4_runtime.h", "nvfp4_stream.cuh",
                                                  "nvfp4_reduce.cuh", "nvfp4_encode.cuh", "nvfp4_ragged.cuh",
                                                  "nvfp4_strided.cuh", "nvfp4_f32scale.cuh")]
DEPS += [os.path.join(INCLUDE, "nvfp4.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-fvisibility=hidden",
    "-Xptxas", "-warn-spills",
    "--cudart", "static",
    "-shared",
]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def build_library(force: bool = False, verbose: bool = False) -> str:
    """Compile libnvfp4.so if it is missing or older than a source; return its path."""
    if not force and os.path.exists(LIB):
        newest = max(os.path.getmtime(p) for p in DEPS)
        if os.path.getmtime(LIB) >= newest:
            return LIB
    cmd = [nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, *SOURCES, "-o", LIB + ".tmp"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build_library(force="--force" in sys.argv, verbose="-v" in sys.argv))
