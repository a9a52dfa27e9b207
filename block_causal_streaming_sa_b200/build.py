"""Build libsa.so in-tree with nvcc for sm_100a (B200), and its checked twin
libsa_checked.so (the same sources with SA_DEVICE_CHECKS: device-side bounds
checks on every direct global access of the attention path's kernels).

Usage: python -m block_causal_streaming_sa_b200.build [--verbose]
"""

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libsa.so")
LIB_CHECKED = os.path.join(HERE, "libsa_checked.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "-Xcompiler", "-fPIC,-fvisibility=hidden",
    "-shared",
]


def sources():
    out = []
    for d, _, files in os.walk(CSRC):
        out += [os.path.join(d, f) for f in files if f.endswith((".cu", ".cuh", ".h"))]
    return out + [os.path.join(ROOT, "include", "sa.h")]


def up_to_date(lib):
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(s) <= t for s in sources())


def _compile(lib, extra, verbose):
    nvcc = os.environ.get("NVCC", "nvcc")
    cmd = [nvcc] + NVCC_FLAGS + extra + (["-Xptxas", "-v"] if verbose else []) + [
        os.path.join(CSRC, "sa_api.cu"), "-o", lib + ".tmp"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed building {os.path.basename(lib)}")
    os.replace(lib + ".tmp", lib)


def build(force=False, verbose=False, checked=True):
    """Compile csrc/sa_api.cu (which includes every kernel) into libsa.so and,
    with checked, into libsa_checked.so as well."""
    if force or not up_to_date(LIB):
        _compile(LIB, [], verbose)
    if checked and (force or not up_to_date(LIB_CHECKED)):
        _compile(LIB_CHECKED, ["-DSA_DEVICE_CHECKS"], verbose)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
    print(LIB_CHECKED)
