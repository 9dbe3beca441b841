"""Build libpkv.so in-tree: the CUDA kernels for sm_100a plus the host block manager.

    python -m paged_kv_cache_392_b200.build [--force] [--verbose-ptxas]
"""
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libpkv.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _inputs():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(CSRC, "*.h")) + [os.path.join(ROOT, "include", "pkv.h"),
                                               os.path.abspath(__file__)]


def up_to_date():
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force=False, verbose_ptxas=False, out=None, defines=()):
    """Compile libpkv.so unless it is newer than every source; return its path.
    ``out``/``defines`` build a variant elsewhere (e.g. -DPKV_DECODE_WARPS=8)."""
    target = out or LIB
    if not force and out is None and up_to_date():
        return LIB
    tmp = target + ".tmp.%d" % os.getpid()
    cmd = [NVCC] + ARCH + ["-lineinfo", "-O3", "-std=c++17", "-shared",
                           "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
                           "-I", os.path.join(ROOT, "include")]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    cmd += list(defines) + sources() + ["-o", tmp]
    subprocess.check_call(cmd)
    os.replace(tmp, target)
    return target


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="--verbose-ptxas" in sys.argv))
