"""Build the CUDA library ``liblpar.so`` in-tree with nvcc for sm_100a.

The library is a plain shared object with a C ABI (``include/lpar.h``); the
CUDA runtime is linked statically, so it loads without a GPU and shares the
device's primary context with PyTorch at run time.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
SOURCES = [os.path.join(CSRC, "lpar_kernels.cu"), os.path.join(CSRC, "lpar_collectives.cu"),
           os.path.join(CSRC, "lpar_f32.cu"), os.path.join(CSRC, "lpar_static_ws.cu"),
           os.path.join(CSRC, "lpar_host.cu"), os.path.join(CSRC, "lpar_peer.cu")]
HEADERS = [os.path.join(CSRC, "lpar_codec.cuh"), os.path.join(CSRC, "lpar_tiles.cuh"), os.path.join(ROOT, "include", "lpar.h")]
LIB = os.path.join(HERE, "liblpar.so")
PTXAS_LOG = os.path.join(HERE, "liblpar.ptxas.txt")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-fmad=false",                  # no contraction: every FMA in the codecs is written out
    "-Xptxas", "-v",
    "-Xcompiler", "-fPIC,-fvisibility=hidden",
    "-shared",
    "-I", os.path.join(ROOT, "include"),
    "-I", CSRC,
]


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in SOURCES + HEADERS + [__file__])


def build(force: bool = False) -> str:
    if force or needs_build():
        tmp = LIB + ".tmp.%d" % os.getpid()
        res = subprocess.run([NVCC, *FLAGS, *SOURCES, "-o", tmp], capture_output=True, text=True)
        with open(PTXAS_LOG, "w") as f:
            f.write(res.stdout + res.stderr)
        if res.returncode != 0:
            raise RuntimeError("nvcc failed:\n" + res.stderr[-4000:])
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
