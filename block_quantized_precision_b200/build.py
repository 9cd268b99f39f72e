"""Builds libqattn.so (the C-ABI library) in place with nvcc for sm_100a.

Run as `python -m block_quantized_precision_b200.build` or call build().
The library statically links the CUDA runtime and resolves the one driver
entry point it needs (tensor-map encoding) at run time, so it depends on
nothing beyond libc/libstdc++ and the NVIDIA driver.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libqattn.so")
SOURCES = ["qattn_abi.cu", "rotate_quant.cu", "prefill.cu", "prefill_bf16.cu", "decode.cu", "decode_noalloc.cu", "kv_append.cu",
           "path_host.cu", "widen_int4.cu"]
HEADERS = ["qattn_device.cuh", "qattn_internal.h", "prefill_common.cuh"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=default",
    "--shared", "-cudart", "static",
    "-diag-suppress", "20044",
]


def _nvcc():
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(os.path.dirname(HERE), "include", "qattn.h"))
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = [_nvcc()] + NVCC_FLAGS + ["-o", tmp] + [os.path.join(CSRC, f) for f in SOURCES]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
