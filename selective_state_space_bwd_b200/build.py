"""Build libssm_scan.so (all CUDA sources under csrc/) for sm_100a with nvcc, in-tree."""

from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libssm_scan.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")))


def deps():
    return sources() + sorted(glob.glob(os.path.join(HERE, "csrc", "*.h*"))) + [
        os.path.join(ROOT, "include", "ssm_scan.h")]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in deps())


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every source whose object is stale to an object, in parallel (one nvcc process
    each; no device code crosses files), then link the shared library."""
    if not force and up_to_date():
        return LIB
    nvcc = os.environ.get("NVCC", "nvcc")
    obj_dir = os.path.join(HERE, "_build")
    os.makedirs(obj_dir, exist_ok=True)
    flags = [*ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
             "-I", os.path.join(ROOT, "include")]
    if verbose:
        flags.append("-Xptxas=-v")
    objs = [os.path.join(obj_dir, os.path.basename(src)[:-3] + ".o") for src in sources()]
    headers = [p for p in deps() if not p.endswith(".cu")]

    def stale(src, obj):
        return force or not os.path.exists(obj) or any(
            os.path.getmtime(p) > os.path.getmtime(obj) for p in [src, *headers])

    procs = [subprocess.Popen([nvcc, *flags, "-c", src, "-o", obj])
             for src, obj in zip(sources(), objs) if stale(src, obj)]
    failed = [p.args for p in procs if p.wait() != 0]
    if failed:
        raise subprocess.CalledProcessError(1, failed[0])
    subprocess.run([nvcc, *ARCH, "-shared", "-o", LIB + ".tmp", *objs], check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="-v" in sys.argv)
    print(LIB)
