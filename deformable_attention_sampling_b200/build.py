"""Build libdcn_b200.so in-tree with nvcc for sm_100a (B200).

    python -m deformable_attention_sampling_b200.build [--verbose]

Each translation unit of the C interface (csrc/abi_*.cu) is compiled to an
object file in parallel, and the objects are linked into one shared library
in deformable_attention_sampling_b200/_lib/, next to the binding that loads
it, so that it travels with the source tree.  nvcc cross-compiles without a
GPU.  `--verbose` passes -Xptxas -v (registers, spills, shared memory per
kernel).
"""
import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_DIR = os.path.join(PKG, "_lib")
OBJ_DIR = os.path.join(LIB_DIR, "obj")
LIB = os.path.join(LIB_DIR, "libdcn_b200.so")
SOURCES = sorted(glob.glob(os.path.join(CSRC, "abi_*.cu")))
HEADERS = sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + [os.path.join(INCLUDE, "dcn.h")]
DEPENDS = SOURCES + HEADERS

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + [
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC",
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


def _object(src):
    return os.path.join(OBJ_DIR, os.path.splitext(os.path.basename(src))[0] + ".o")


def build(force=False, verbose=False, jobs=None):
    """Compile the library if it is missing or older than a source; return its path."""
    if not force and not _stale():
        return LIB
    os.makedirs(OBJ_DIR, exist_ok=True)
    extra = ["-Xptxas=-v"] if verbose else []

    def compile_one(src):
        cmd = [nvcc(), *NVCC_FLAGS, *extra, "-I", INCLUDE, "-I", CSRC, "-c", src,
               "-o", _object(src)]
        return subprocess.run(cmd, capture_output=True, text=True)

    jobs = jobs or min(len(SOURCES), os.cpu_count() or 1)
    with ThreadPoolExecutor(max_workers=jobs) as pool:
        results = list(pool.map(compile_one, SOURCES))
    failed = False
    for src, r in zip(SOURCES, results):
        if r.stdout or r.stderr:
            sys.stderr.write(r.stdout + r.stderr)
        if r.returncode != 0:
            sys.stderr.write(f"nvcc failed on {os.path.basename(src)}\n")
            failed = True
    if failed:
        raise subprocess.CalledProcessError(1, "nvcc")
    cmd = [nvcc(), *ARCH, "-shared", "-o", LIB, *[_object(s) for s in SOURCES]]
    subprocess.run(cmd, check=True)
    # the objects are not kept: every build compiles all units, and the
    # library alone travels with the source tree
    for s in SOURCES:
        os.remove(_object(s))
    os.rmdir(OBJ_DIR)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv))
