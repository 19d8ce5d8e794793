"""Build libmoe_mxfp4.so (the C-ABI library) in-tree with nvcc for sm_100a."""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmoe_mxfp4.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

SOURCES = [os.path.join(CSRC, "moe_mxfp4.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")] + [
    os.path.join(ROOT, "include", "moe_mxfp4.h")]


DEBUG_LIB = os.path.join(HERE, "libmoe_mxfp4_debug.so")


def nvcc_cmd(out, extra=()):
    return [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
            "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr",
            "-I", os.path.join(ROOT, "include"), "-o", out, *SOURCES, *extra]


def _build_one(lib: str, force: bool, extra) -> str:
    if (not force and os.path.exists(lib)
            and os.path.getmtime(lib) >= max(os.path.getmtime(p) for p in DEPS)):
        return lib
    tmp = lib + ".tmp%d" % os.getpid()
    subprocess.check_call(nvcc_cmd(tmp, extra))
    os.replace(tmp, lib)
    return lib


def build(force: bool = False, verbose: bool = False) -> str:
    """The release library (the product path)."""
    return _build_one(LIB, force, ("-Xptxas", "-v") if verbose else ())


def build_debug(force: bool = False) -> str:
    """The same sources with device index checks and guard regions (MOE_DEBUG_CHECKS)."""
    return _build_one(DEBUG_LIB, force, ("-DMOE_DEBUG_CHECKS",))


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
    print(build_debug(force="--force" in sys.argv))
