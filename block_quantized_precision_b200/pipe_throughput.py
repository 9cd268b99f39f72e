"""Builds and runs csrc/pipe_throughput.cu: the issue throughput, per SM and
clock, of the instructions the kernels rely on (FP32 FMA -- the peak of the
rotation's roofline --, exponentials, e4m3 conversions, integer maxima, byte
permutes). Needs a GPU.

    python -m block_quantized_precision_b200.pipe_throughput [SM clock MHz]
"""
import os
import subprocess
import sys
import tempfile

from .build import _nvcc

HERE = os.path.dirname(os.path.abspath(__file__))


def main(argv):
    src = os.path.join(HERE, "csrc", "pipe_throughput.cu")
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "pipe_throughput")
        subprocess.check_call([_nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-o", exe, src])
        return subprocess.call([exe] + argv)


if __name__ == "__main__":
    sys.exit(main(sys.argv[1:]))
