"""Build libpkv.so in-tree: the CUDA kernels for sm_100a plus the host block manager.

    python -m paged_kv_cache_392_b200.build [--force] [--verbose-ptxas]
                                            [--out PATH -DNAME[=VALUE] ...]

With --out, a variant of the same sources is compiled to PATH with the given macros (the
build-time tuning macros of the kernels, e.g. -DPKV_DECODE_FORCE_SIMT); load it by setting
PKV_LIB=PATH before the binding is imported.
"""
import glob
import hashlib
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
    return up_to_date_at(LIB)


def up_to_date_at(path):
    if not os.path.exists(path):
        return False
    t = os.path.getmtime(path)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def variant_path(defines):
    """In-tree path of the variant built with these macros (one file per set of macros)."""
    tag = hashlib.sha256(" ".join(sorted(defines)).encode()).hexdigest()[:10]
    return os.path.join(HERE, "libpkv_variant_%s.so" % tag)


def build(force=False, verbose_ptxas=False, out=None, defines=()):
    """Compile libpkv.so unless it is newer than every source; return its path.
    ``out``/``defines`` build a variant elsewhere (e.g. -DPKV_DECODE_WARPS=8); a variant at
    ``variant_path(defines)`` is rebuilt only when a source is newer than it, like the
    library itself, one at any other path always."""
    target = out or LIB
    reusable = out is None or out == variant_path(defines)
    if not force and not verbose_ptxas and reusable and up_to_date_at(target):
        return target
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


def main(argv):
    defines = [a for a in argv if a.startswith("-D")]
    out = None
    if "--out" in argv:
        out = os.path.abspath(argv[argv.index("--out") + 1])
    elif defines:
        out = variant_path(defines)
    print(build(force="--force" in argv, verbose_ptxas="--verbose-ptxas" in argv, out=out,
                defines=defines))


if __name__ == "__main__":
    main(sys.argv[1:])
