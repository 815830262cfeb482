"""Build the seeded input generator: a host library (gcc) and a device library (nvcc, sm_100a).

Both compile gen_core.h with fused multiply-add contraction off, so the host
and the device produce the same bits.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
HOST_SO = os.path.join(HERE, "libseeded_inputs_host.so")
CUDA_SO = os.path.join(HERE, "libseeded_inputs_cuda.so")


def _stale(target, sources):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def build(force=False, cuda=True):
    core = os.path.join(HERE, "gen_core.h")
    host_src = os.path.join(HERE, "gen_host.c")
    if force or _stale(HOST_SO, [core, host_src]):
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-ffp-contract=off",
             "-fno-fast-math", "-fno-math-errno", host_src, "-o", HOST_SO])
    cuda_src = os.path.join(HERE, "gen_cuda.cu")
    if cuda and (force or _stale(CUDA_SO, [core, cuda_src])):
        subprocess.check_call(
            ["nvcc", "-O2", "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "-fmad=false",
             "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", cuda_src, "-o", CUDA_SO])


if __name__ == "__main__":
    build(force="--force" in sys.argv)
