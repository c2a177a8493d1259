"""Builds the synthetic-input generator libraries in place.

libbeam_synth_host.so: host generator (gcc, OpenMP); needs no GPU.
libbeam_synth_cuda.so: device fill kernels (nvcc, sm_100a).
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
HOST_LIB = os.path.join(HERE, "libbeam_synth_host.so")
CUDA_LIB = os.path.join(HERE, "libbeam_synth_cuda.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def _stale(target, sources):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def build_host(force=False):
    srcs = [os.path.join(HERE, "synth_host.c"), os.path.join(HERE, "synth.h")]
    if force or _stale(HOST_LIB, srcs):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               srcs[0], "-o", HOST_LIB + ".tmp", "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(HOST_LIB + ".tmp", HOST_LIB)
    return HOST_LIB


def build_cuda(force=False):
    srcs = [os.path.join(HERE, "synth_cuda.cu"), os.path.join(HERE, "synth.h")]
    if force or _stale(CUDA_LIB, srcs):
        cmd = [NVCC, "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
               "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
               srcs[0], "-o", CUDA_LIB + ".tmp"]
        subprocess.run(cmd, check=True)
        os.replace(CUDA_LIB + ".tmp", CUDA_LIB)
    return CUDA_LIB


if __name__ == "__main__":
    print(build_host(force=True))
    print(build_cuda(force=True))
