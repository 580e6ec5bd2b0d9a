"""Build libmoe.so (sm_100a) in-tree with nvcc.

    python -m sparse_moe_layer_top_b200.build [--force] [--verbose-ptxas] [--checks]

--checks builds the bounds-checking variant libmoe_checks.so instead
(-DMOE_CHECKS: device checks of the kernels' computed and read indices,
reported through the device status word); the binding loads it when the
environment sets MOE_CHECKS=1.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmoe.so")
LIB_CHECKS = os.path.join(HERE, "libmoe_checks.so")
SOURCES = [os.path.join(CSRC, "api.cu")]
DEPS = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(ROOT, "include", "moe.h")]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
    "-Xcompiler", "-fPIC,-O2,-fvisibility=hidden",
    "-shared", "-cudart", "static",
]


def stale(lib=LIB):
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(f) > t for f in DEPS if os.path.isfile(f))


def build(force=False, ptxas_verbose=False, checks=False):
    lib = LIB_CHECKS if checks else LIB
    if not force and not stale(lib):
        return lib
    tmp = lib + ".tmp.%d" % os.getpid()
    cmd = ([NVCC] + FLAGS + (["-DMOE_CHECKS"] if checks else []) + (["-Xptxas", "-v"] if ptxas_verbose else []) +
           ["-o", tmp] + SOURCES)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, ptxas_verbose="--verbose-ptxas" in sys.argv,
                checks="--checks" in sys.argv))
