"""Build liboq.so (the C-ABI library) in-tree for sm_100a.

    python -m rotation_bit_quantization_rpbh_b200.build [--force]

nvcc cross-compiles for sm_100a without a GPU.  The CUDA runtime is linked
statically; the driver's tensor-map encoder is fetched at run time, so the
library links against nothing but libc/libstdc++.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
OUT = os.path.join(HERE, "liboq.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
SOURCES = ["liboq.cu", "host.cpp"]
DEPS = ["liboq.cu", "host.cpp", "api.cu", "rpbh_quant.cu", "rpbh_groups.cu", "rht_big.cu", "qgemm.cu", "device_util.cuh", "oq_internal.h",
        "rpbh_quant.cuh", "qgemm.cuh"]


def _stale() -> bool:
    if not os.path.exists(OUT):
        return True
    t = os.path.getmtime(OUT)
    hdr = os.path.join(HERE, "..", "include", "oq.h")
    return any(os.path.getmtime(os.path.join(CSRC, f)) > t for f in DEPS) or os.path.getmtime(hdr) > t


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return OUT
    tmp = OUT + ".tmp%d" % os.getpid()
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
           "-Xcompiler", "-fPIC,-O2", "-shared", "-o", tmp]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    subprocess.run(cmd, check=True, cwd=CSRC)
    os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
