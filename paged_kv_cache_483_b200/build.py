"""Build libpagedattn.so in-tree with nvcc for sm_100a.

Usage: python -m paged_kv_cache_483_b200.build [--verbose-ptxas]
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libpagedattn.so")
SOURCES = ["block_manager.cpp", "pa_api.cu", "kv_write.cu", "attention_generic.cu",
           "decode_mma.cu", "decode_q8.cu", "decode_q8tc.cu", "prefill_tc.cu",
           "decode_static.cu", "batch_upload.cu"]
HEADERS = ["block_manager.hpp", "common.cuh", "device_once.hpp", "launch.hpp", "tcgen05.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or cand == "nvcc"):
            return cand
    return "nvcc"


def stale():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(HERE, "..", "include", "pa.h"))
    deps.append(os.path.abspath(__file__))
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


def build(force=False, ptxas_verbose=False):
    if not force and not stale():
        return LIB
    cmd = [nvcc(), "-O3", "-std=c++17", *ARCH, "-lineinfo", "-shared",
           "-Xcompiler", "-fPIC,-O3", "--expt-relaxed-constexpr",
           "-o", LIB + ".tmp"]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, f) for f in SOURCES]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv)
    print(LIB)
