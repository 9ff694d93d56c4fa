"""Build the CUDA library libssmscan.so in-tree for sm_100a (nvcc, no JIT cache).

    python -m selective_state_space_47_b200.build [--force]
"""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
SOURCES = [os.path.join(CSRC, "ssm_scan.cu"), os.path.join(CSRC, "ssm_host.cu"), os.path.join(CSRC, "ssm_scan_bwd.cu"),
           os.path.join(CSRC, "ssm_ssd.cu")]
DEPS = SOURCES + [os.path.join(CSRC, "ssm_device.cuh"), os.path.join(CSRC, "ssm_scan_kernel.cuh"), os.path.join(ROOT, "include", "ssm_scan.h")]
LIB = os.path.join(PKG, "libssmscan.so")
NVCC_FLAGS = ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
              "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall", "-cudart", "static",
              "-I", os.path.join(ROOT, "include")]


def nvcc():
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def build(force=False, verbose=False):
    if not force and os.path.exists(LIB):
        newest = max(os.path.getmtime(p) for p in DEPS)
        if os.path.getmtime(LIB) >= newest:
            return LIB
    tmp = LIB + ".tmp"
    cmd = [nvcc()] + NVCC_FLAGS + ["-o", tmp] + SOURCES
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
