"""Build the two third-party Philox references the Philox pins call:
libtorch_philox.so (PyTorch's host engine, g++) and libcurand_philox.so
(cuRAND's device API, nvcc for sm_100a).  Test infrastructure only.

    python tests/philox_ref/build.py
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")
TORCH_LIB = os.path.join(HERE, "libtorch_philox.so")
CURAND_LIB = os.path.join(HERE, "libcurand_philox.so")


def _stale(target, src):
    return not os.path.exists(target) or os.path.getmtime(src) > os.path.getmtime(target)


def build_torch_ref():
    import torch
    src = os.path.join(HERE, "torch_philox.cpp")
    if _stale(TORCH_LIB, src):
        inc = os.path.join(os.path.dirname(torch.__file__), "include")
        tmp = TORCH_LIB + ".tmp.%d" % os.getpid()
        subprocess.run(["g++", "-std=c++17", "-O1", "-fPIC", "-shared", "-I", inc, "-I",
                        os.path.join(CUDA, "include"), src, "-o", tmp], check=True)
        os.replace(tmp, TORCH_LIB)
    return TORCH_LIB


def build_curand_ref():
    src = os.path.join(HERE, "curand_philox.cu")
    if _stale(CURAND_LIB, src):
        tmp = CURAND_LIB + ".tmp.%d" % os.getpid()
        subprocess.run([os.path.join(CUDA, "bin", "nvcc"), "-gencode",
                        "arch=compute_100a,code=sm_100a", "-O2", "-Xcompiler", "-fPIC", "-shared",
                        src, "-o", tmp], check=True)
        os.replace(tmp, CURAND_LIB)
    return CURAND_LIB


def build():
    return build_torch_ref(), build_curand_ref()


if __name__ == "__main__":
    print(build())
    sys.exit(0)
