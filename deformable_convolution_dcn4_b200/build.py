"""Builds libdcn4.so (the C-ABI library) in-tree with nvcc for sm_100a, and
its bounds-checked twin libdcn4_checked.so (-DDCN4_CHECKED: every shared- and
global-memory access of the kernels is range-checked; a violation skips the
access and is reported as DCN4_ERR_INTERNAL by dcn4_last_device_error).

    python -m deformable_convolution_dcn4_b200.build [--force] [--verbose] [--checked]

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
CHECKED_LIBRARY = os.path.join(PKG, "libdcn4_checked.so")
SOURCES = ["dcn4_api.cu", "dcn4_kernels.cu", "dcn4_kernels_fwd.cu", "dcn4_kernels_bwd.cu",
           "dcn4_kernels_fused.cu", "dcn4_noalloc.cu"]
OBJDIR = os.path.join(PKG, "_build")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "-DDCN4_BUILDING_LIBRARY", "-I", INCLUDE, "-I", CSRC]


def _inputs():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    files.append(os.path.join(INCLUDE, "dcn4.h"))
    return files


def up_to_date(library=LIBRARY):
    if not os.path.exists(library):
        return False
    t = os.path.getmtime(library)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force=False, verbose=False, checked=False):
    """Compiles each translation unit to an object (in parallel), then links
    the shared library; checked=True builds libdcn4_checked.so."""
    library = CHECKED_LIBRARY if checked else LIBRARY
    if not force and up_to_date(library):
        return library
    objdir = OBJDIR + ("_checked" if checked else "")
    os.makedirs(objdir, exist_ok=True)
    procs, objs = [], []
    for src in SOURCES:
        obj = os.path.join(objdir, src[:-3] + ".o")
        cmd = [NVCC, *FLAGS, *(["-DDCN4_CHECKED"] if checked else []), "-c",
               os.path.join(CSRC, src), "-o", obj]
        if verbose:
            cmd += ["-Xptxas", "-v"]
        procs.append((src, subprocess.Popen(cmd)))
        objs.append(obj)
    failed = [src for src, p in procs if p.wait() != 0]
    if failed:
        raise subprocess.CalledProcessError(1, f"nvcc ({', '.join(failed)})")
    subprocess.run([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", *objs,
                    "-o", library], check=True)
    return library


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv,
                checked="--checked" in sys.argv))
