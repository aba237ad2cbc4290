"""Build libvimscan.so in-tree with nvcc for sm_100a (no GPU needed to build).

    python -m vision_mamba_selective_b200.build [--verbose]

The library links the CUDA runtime statically, so it loads wherever the NVIDIA
driver is present; it is placed next to this file, where the binding looks for it.
"""
import glob
import os
import subprocess
import sys
import tempfile

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libvimscan.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    return sorted(glob.glob(os.path.join(PKG, "csrc", "*.cu")))


def deps():
    return sources() + sorted(glob.glob(os.path.join(PKG, "csrc", "*.cuh"))) + [
        os.path.join(ROOT, "include", "vimscan.h")]


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every csrc/*.cu to an object in parallel (the kernel variants are
    spread over several units for that), then link the shared library."""
    if not force and os.path.exists(LIB):
        t = os.path.getmtime(LIB)
        if all(os.path.getmtime(f) <= t for f in deps()):
            return LIB
    flags = [*ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-I", os.path.join(ROOT, "include")]
    if verbose:
        flags.insert(0, "-Xptxas=-v")
    with tempfile.TemporaryDirectory(prefix="vimscan_build_") as tmp:
        objs, procs = [], []
        for src in sources():
            obj = os.path.join(tmp, os.path.basename(src) + ".o")
            objs.append(obj)
            procs.append((src, subprocess.Popen([NVCC, *flags, "-c", "-o", obj, src])))
        failed = [src for src, p in procs if p.wait() != 0]
        if failed:
            raise subprocess.CalledProcessError(1, f"nvcc ({', '.join(map(os.path.basename, failed))})")
        subprocess.run([NVCC, *ARCH, "--cudart", "static", "-shared", "-o", LIB, *objs], check=True)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv))
