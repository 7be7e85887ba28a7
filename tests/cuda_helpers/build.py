"""Build the test-only device-check library (tests/cuda_helpers/libnvfp4_checks.so)."""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
SRC = os.path.join(HERE, "device_checks.cu")
DEV_HDR = os.path.join(ROOT, "nvfp4_bit_quantized_02_b200", "csrc", "nvfp4_device.cuh")
LIB = os.path.join(HERE, "libnvfp4_checks.so")


def build(force: bool = False) -> str:
    newest = max(os.path.getmtime(SRC), os.path.getmtime(DEV_HDR))
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= newest:
        return LIB
    cmd = [os.environ.get("NVCC", "nvcc"), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
           "-fmad=false", "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
           "-I" + os.path.dirname(DEV_HDR), "-o", LIB + ".tmp", SRC]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
