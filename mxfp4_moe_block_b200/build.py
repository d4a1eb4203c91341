"""Build the CUDA library in-tree: libmxfp4_moe.so next to this file.

    python -m mxfp4_moe_block_b200.build            # libmxfp4_moe.so
    python -m mxfp4_moe_block_b200.build --checks   # libmxfp4_moe_checks.so

Compiles csrc/mxfp4_moe.cu (which includes every kernel) for sm_100a only.
The checked build (-DMOE_CHECKS) tests every index read from a caller's
array before it addresses memory and reports a bad one in the device status
word (MOE_DEV_BAD_INDEX); the package loads it when MXFP4_MOE_CHECKS=1.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc", "mxfp4_moe.cu")
OUT = os.path.join(HERE, "libmxfp4_moe.so")
OUT_CHECKS = os.path.join(HERE, "libmxfp4_moe_checks.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
    "-Xptxas", "-warn-spills",
]


def sources():
    d = os.path.join(HERE, "csrc")
    return [os.path.join(d, f) for f in sorted(os.listdir(d))] + [
        os.path.join(os.path.dirname(HERE), "include", "mxfp4_moe.h")]


def up_to_date(out=OUT):
    if not os.path.exists(out):
        return False
    t = os.path.getmtime(out)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(force=False, verbose=False, checks=False):
    out = OUT_CHECKS if checks else OUT
    if not force and up_to_date(out):
        return out
    cmd = [NVCC, *FLAGS, *(["-DMOE_CHECKS"] if checks else []), "-o", out + ".tmp", SRC]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(force=True, verbose="-v" in sys.argv, checks="--checks" in sys.argv))
