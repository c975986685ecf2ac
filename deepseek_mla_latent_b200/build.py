"""Build the in-tree shared library ``libmla_b200.so`` with nvcc for sm_100a.

One translation unit (csrc/mla_lib.cu) includes every kernel header; the CUDA
runtime is linked statically and the driver entry point needed for TMA
descriptors is fetched at run time, so the library loads on machines without
a GPU driver (symbols can be listed there; compute calls need a B200).
"""
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libmla_b200.so")
SOURCES = [os.path.join(HERE, "csrc", "mla_lib.cu")]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _newest_source_mtime() -> float:
    paths = [__file__]
    for d in (os.path.join(ROOT, "include"), os.path.join(HERE, "csrc")):
        for dd, _, files in os.walk(d):
            paths += [os.path.join(dd, f) for f in files if f.endswith((".cu", ".cuh", ".h"))]
    return max(os.path.getmtime(p) for p in paths)


# Library variants: the product library, and a fault-injection build used only by the tests of
# the bounded device waits (short wait limits and a host-set fault plan; see mla_fault_inject.h).
VARIANTS = {"": ([], LIB),
            "fault_inject": (["-DMLA_FAULT_INJECT"], os.path.join(HERE, "libmla_b200_fault_inject.so"))}


def build(force: bool = False, verbose: bool = False, extra=(), variant: str = "") -> str:
    flags, lib = VARIANTS[variant]
    if not force and os.path.exists(lib) and os.path.getmtime(lib) >= _newest_source_mtime():
        return lib
    tmp = lib + ".tmp"
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "--shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "-cudart", "static", "--expt-relaxed-constexpr",
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(HERE, "csrc"),
           *flags, *extra, *SOURCES, "-o", tmp]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    variant = "fault_inject" if "--fault-inject" in sys.argv else ""
    print(build(force="--force" in sys.argv, verbose=True,
                extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [], variant=variant))
