"""Builds libdcn4.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m deformable_convolution_dcn4_b200.build [--force] [--verbose]

No fast-math: sample positions rely on IEEE fp32 rounding of each multiply
and add (the kernels use __fmul_rn/__fadd_rn where it matters).
"""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIBRARY = os.path.join(PKG, "libdcn4.so")
SOURCES = ["dcn4_api.cu", "dcn4_kernels.cu", "dcn4_kernels_fwd.cu", "dcn4_kernels_bwd.cu",
           "dcn4_noalloc.cu"]
OBJDIR = os.path.join(PKG, "_build")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "-DDCN4_BUILDING_LIBRARY", "-I", INCLUDE, "-I", CSRC]


def _inputs():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    files.append(os.path.join(INCLUDE, "dcn4.h"))
    return files


def up_to_date():
    if not os.path.exists(LIBRARY):
        return False
    t = os.path.getmtime(LIBRARY)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force=False, verbose=False):
    """Compiles each translation unit to an object (in parallel), then links
    the shared library."""
    if not force and up_to_date():
        return LIBRARY
    os.makedirs(OBJDIR, exist_ok=True)
    procs, objs = [], []
    for src in SOURCES:
        obj = os.path.join(OBJDIR, src[:-3] + ".o")
        cmd = [NVCC, *FLAGS, "-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            cmd += ["-Xptxas", "-v"]
        procs.append((src, subprocess.Popen(cmd)))
        objs.append(obj)
    failed = [src for src, p in procs if p.wait() != 0]
    if failed:
        raise subprocess.CalledProcessError(1, f"nvcc ({', '.join(failed)})")
    subprocess.run([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", *objs,
                    "-o", LIBRARY], check=True)
    return LIBRARY


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
