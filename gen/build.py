"""Builds the seeded input generator: a host library (gcc) and a device library (nvcc, sm_100a)."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
HOST_SO = os.path.join(HERE, "libfmoegen_host.so")
CUDA_SO = os.path.join(HERE, "libfmoegen_cuda.so")


def _stale(target, sources):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def build(force=False, verbose=False):
    hdr = os.path.join(HERE, "fmoe_gen.h")
    src_h = os.path.join(HERE, "gen_host.c")
    src_c = os.path.join(HERE, "gen_cuda.cu")
    if force or _stale(HOST_SO, [hdr, src_h]):
        cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-std=c11", src_h, "-o", HOST_SO, "-lm"]
        if verbose:
            print(" ".join(cmd))
        subprocess.check_call(cmd)
    if force or _stale(CUDA_SO, [hdr, src_c]):
        cmd = ["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-fmad=false",
               "-prec-div=true", "-prec-sqrt=true", "-shared", "-Xcompiler", "-fPIC", src_c, "-o", CUDA_SO]
        if verbose:
            print(" ".join(cmd))
        subprocess.check_call(cmd)
    return HOST_SO, CUDA_SO


if __name__ == "__main__":
    build(force=True, verbose=True)
