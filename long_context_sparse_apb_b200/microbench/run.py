"""Builds and runs the UMMA microbenchmarks on cuda:0: issue rate
(umma_rate.cu, single SM; umma_pair_rate.cu, cta_group::2 pairs) and the
cost of shared-memory accesses between UMMA runs (umma_sync.cu).

    python -m long_context_sparse_apb_b200.microbench.run
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))


def main() -> int:
    rc = 0
    for name in ("umma_rate", "umma_pair_rate", "umma_sync"):
        exe = os.path.join(ROOT, "_build", name)
        os.makedirs(os.path.dirname(exe), exist_ok=True)
        subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                        "-I", os.path.join(ROOT, "include"), os.path.join(HERE, name + ".cu"),
                        "-o", exe], check=True)
        rc |= subprocess.run([exe]).returncode
    return rc


if __name__ == "__main__":
    sys.exit(main())
