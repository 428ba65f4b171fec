"""Builds libfmoe.so in-tree: every CUDA source of the package for sm_100a, one shared library."""
import glob
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SO = os.path.join(HERE, "libfmoe.so")
# the debug build: the same sources with FMOE_DEBUG_BOUNDS (device-side bounds checks)
DEBUG_SO = os.path.join(HERE, "libfmoe_debug.so")
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
              "-Xptxas", "-warn-spills"]


def sources():
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")))


def _deps():
    return sources() + glob.glob(os.path.join(HERE, "csrc", "*.h")) + glob.glob(os.path.join(HERE, "csrc", "*.cuh")) + \
        glob.glob(os.path.join(ROOT, "include", "*.h"))


def build(force=False, verbose=False, extra_flags=(), debug_bounds=False):
    so = DEBUG_SO if debug_bounds else SO
    if debug_bounds:
        extra_flags = (*extra_flags, "-DFMOE_DEBUG_BOUNDS")
    if not force and os.path.exists(so):
        t = os.path.getmtime(so)
        if all(os.path.getmtime(d) <= t for d in _deps()):
            return so
    objdir = os.path.join(HERE, "_build_debug" if debug_bounds else "_build")
    os.makedirs(objdir, exist_ok=True)
    objs = []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        cmd = ["nvcc", *NVCC_FLAGS, *extra_flags, "-I", os.path.join(ROOT, "include"), "-I", os.path.join(HERE, "csrc"),
               "-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd))
        subprocess.check_call(cmd)
        objs.append(obj)
    cmd = ["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-shared", *objs, "-o", so]
    if verbose:
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    return so


if __name__ == "__main__":
    import sys
    build(force=True, verbose=True, debug_bounds="--debug-bounds" in sys.argv)
