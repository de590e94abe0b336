"""Builds and runs the UMMA-rate microbenchmark (umma_rate.cu) on cuda:0.

    python -m long_context_sparse_apb_b200.microbench.run
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))


def main() -> int:
    exe = os.path.join(ROOT, "_build", "umma_rate")
    os.makedirs(os.path.dirname(exe), exist_ok=True)
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                    "-I", os.path.join(ROOT, "include"), os.path.join(HERE, "umma_rate.cu"), "-o",
                    exe], check=True)
    return subprocess.run([exe]).returncode


if __name__ == "__main__":
    sys.exit(main())
