"""Build libdcn_b200.so in-tree with nvcc for sm_100a (B200).

    python -m deformable_attention_sampling_b200.build [--verbose]

It also builds the debug library, libdcn_b200_debug.so. That one holds the
forward entry points and the status calls, compiled with DCN_DEBUG: every
gather, shared-memory and store address, and the MSDA level table, is checked
on the device. A violation is reported in the status word (dcn_device_flags)
and the access is skipped.

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
DEBUG_LIB = os.path.join(LIB_DIR, "libdcn_b200_debug.so")
DEBUG_UNITS = ("abi_common.cu", "abi_dcn_fwd.cu", "abi_fused.cu", "abi_msda.cu")
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


def _stale(lib):
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in DEPENDS)


def _object(src, tag):
    return os.path.join(OBJ_DIR, os.path.splitext(os.path.basename(src))[0] + tag + ".o")


def _link(jobs, verbose):
    """Compile the release units and the debug units in parallel, link both
    libraries, and remove the objects (only the libraries travel with the
    source tree)."""
    os.makedirs(OBJ_DIR, exist_ok=True)
    extra = ["-Xptxas=-v"] if verbose else []
    debug_sources = [s for s in SOURCES if os.path.basename(s) in DEBUG_UNITS]
    work = [(s, "", []) for s in SOURCES] + [(s, "_debug", ["-DDCN_DEBUG"]) for s in debug_sources]

    def compile_one(item):
        src, tag, defs = item
        cmd = [nvcc(), *NVCC_FLAGS, *extra, *defs, "-I", INCLUDE, "-I", CSRC, "-c", src,
               "-o", _object(src, tag)]
        return subprocess.run(cmd, capture_output=True, text=True)

    jobs = jobs or min(len(work), os.cpu_count() or 1)
    with ThreadPoolExecutor(max_workers=jobs) as pool:
        results = list(pool.map(compile_one, work))
    failed = False
    for (src, tag, _), r in zip(work, results):
        if r.stdout or r.stderr:
            sys.stderr.write(r.stdout + r.stderr)
        if r.returncode != 0:
            sys.stderr.write(f"nvcc failed on {os.path.basename(src)}{tag}\n")
            failed = True
    if failed:
        raise subprocess.CalledProcessError(1, "nvcc")
    subprocess.run([nvcc(), *ARCH, "-shared", "-o", LIB,
                    *[_object(s, "") for s in SOURCES]], check=True)
    subprocess.run([nvcc(), *ARCH, "-shared", "-o", DEBUG_LIB,
                    *[_object(s, "_debug") for s in debug_sources]], check=True)
    for src, tag, _ in work:
        os.remove(_object(src, tag))
    os.rmdir(OBJ_DIR)


def build(force=False, verbose=False, jobs=None):
    """Compile both libraries if either is missing or older than a source;
    return the release library's path."""
    if force or _stale(LIB) or _stale(DEBUG_LIB):
        _link(jobs, verbose)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv))
