"""Build libnvfp4.so in-tree for sm_100a (B200) with nvcc.

Each .cu is compiled to an object under _build/, then linked into
nvfp4_bit_quantized_02_b200/libnvfp4.so.  The quantization and API translation units are
compiled with -fmad=false: codes and scales must come from single IEEE operations.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
PKG = os.path.dirname(HERE)
ROOT = os.path.dirname(PKG)
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libnvfp4.so")
NVCC = os.environ.get("NVCC", "nvcc")

SOURCES = {
    "quantize.cu": ["-fmad=false"],
    "api.cu": ["-fmad=false"],
    "gemm_sm100.cu": [],
    "glue.cu": [],
    "noalloc.cu": [],
}
HEADERS = ["nvfp4_device.cuh", "nvfp4_internal.h"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-I" + os.path.join(ROOT, "include"), "-I" + HERE]


def _newest(paths):
    return max(os.path.getmtime(p) for p in paths)


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    deps = [os.path.join(HERE, h) for h in HEADERS] + [os.path.join(ROOT, "include", "nvfp4.h")]
    objs = []
    for src, extra in SOURCES.items():
        s = os.path.join(HERE, src)
        o = os.path.join(BUILD, src.replace(".cu", ".o"))
        objs.append(o)
        if force or not os.path.exists(o) or os.path.getmtime(o) < _newest([s] + deps):
            cmd = [NVCC] + ARCH + COMMON + extra + ["-c", s, "-o", o]
            if verbose:
                cmd += ["-Xptxas", "-v"]
            subprocess.run(cmd, check=True)
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < _newest(objs):
        cmd = [NVCC] + ARCH + ["-shared", "-cudart", "static", "-o", LIB + ".tmp"] + objs
        subprocess.run(cmd, check=True)
        os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
