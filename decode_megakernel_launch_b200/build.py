"""Builds libamk.so in-tree with nvcc for sm_100a (no JIT cache, so the library travels with the repo)."""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libamk.so")
SOURCES = ["csrc/amk_device.cu", "csrc/amk_api.cu", "csrc/amk_plan.cpp", "csrc/amk_noalloc.cu"]
NVCC = os.environ.get("NVCC", "nvcc")


def _newest_source_mtime() -> float:
    paths = [os.path.join(PKG, s) for s in SOURCES]
    paths += [os.path.join(PKG, "csrc", f) for f in os.listdir(os.path.join(PKG, "csrc")) if f.endswith(".h")]
    paths.append(os.path.join(ROOT, "include", "amk.h"))
    return max(os.path.getmtime(p) for p in paths)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile libamk.so unless it is newer than every source. Returns its path."""
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= _newest_source_mtime():
        return LIB
    cmd = [NVCC, "-O3", "-lineinfo", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
           "-Xcompiler", "-fPIC", "-shared", "-I" + os.path.join(ROOT, "include"),
           *[os.path.join(PKG, s) for s in SOURCES], "-o", LIB + ".tmp"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
