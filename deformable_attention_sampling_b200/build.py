"""Build libdcn_b200.so in-tree with nvcc for sm_100a (B200).

    python -m deformable_attention_sampling_b200.build [--verbose]

The shared library lands in deformable_attention_sampling_b200/_lib/ next to
the binding that loads it, so that it travels with the source tree.  nvcc
cross-compiles without a GPU.
"""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_DIR = os.path.join(PKG, "_lib")
LIB = os.path.join(LIB_DIR, "libdcn_b200.so")
SOURCES = [os.path.join(CSRC, "dcn_abi.cu")]
DEPENDS = SOURCES + [os.path.join(CSRC, f) for f in ("common.cuh", "dcn_fwd.cuh", "msda_fwd.cuh", "dcn_bwd.cuh", "msda_bwd.cuh",
                                                   "dynconv_fwd.cuh")]
DEPENDS.append(os.path.join(INCLUDE, "dcn.h"))

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-Xcompiler", "-fvisibility=hidden",
]


def nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def _stale():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in DEPENDS)


def build(force=False, verbose=False):
    """Compile the library if it is missing or older than a source; return its path."""
    if not force and not _stale():
        return LIB
    os.makedirs(LIB_DIR, exist_ok=True)
    cmd = [nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, *SOURCES, "-o", LIB]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    return LIB


PROBE_SRC = os.path.join(CSRC, "l1_gather_probe.cu")
PROBE = os.path.join(LIB_DIR, "l1_gather_probe")


def build_probe():
    """Compile the gather-rate probe (a standalone program) next to the library."""
    os.makedirs(LIB_DIR, exist_ok=True)
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
           PROBE_SRC, "-o", PROBE]
    subprocess.run(cmd, check=True)
    return PROBE


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv))
    if "--probe" in sys.argv:
        print(build_probe())
