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


# Compile-time knobs of the kernel (macros of csrc/amk_internal.h) that a variant build may set,
# with the values the kernel's static checks and the planner accept.
TUNABLE = {
    "AMK_SLOT_BYTES": (32768, 49152, 65536),   # ring slot size (3 slots of 64 KB fill shared memory)
    "AMK_SLOTS": (2, 3, 4, 5, 6),             # ring depth (static_assert bounds the total)
    "AMK_INFLIGHT": (1, 2, 3, 4),             # outstanding bulk copies (<= slots)
    "AMK_PF_ITEMS": tuple(range(0, 17)),      # L2 warm-up items while the compute warps stall
    "AMK_PF_GAP_NS": (200, 400, 600, 800, 1000, 1200, 1600),
    "AMK_PF_STALL_NS": (100, 200, 400, 800),
    "AMK_PF_CONTINUOUS": (0, 1),              # warm-up between stalls too
    "AMK_NB32": (2, 4),                       # rows per register batch, 32-byte groups
    "AMK_I4_NOSHIFT": (0, 1),                 # int4 high nibbles in place (1) or shifted (0)
    "AMK_CONSUMER_WARPS": (12, 15, 16),       # compute warps per CTA (16 caps registers at 96)
    "AMK_INLINE_HOT": (0, 1),                 # the hot int8 GEMV instance inlined into the task loop
    "AMK_INLINE_HOT4": (0, 1),                # the same for the hot int4 instance
}


def _nvcc_cmd(out: str, defines: dict, verbose: bool) -> list:
    cmd = [NVCC, "-O3", "-lineinfo", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
           "-Xcompiler", "-fPIC", "-shared", "-I" + os.path.join(ROOT, "include"),
           *[f"-D{k}={int(v)}" for k, v in sorted(defines.items())],
           *[os.path.join(PKG, s) for s in SOURCES], "-o", out]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def check_defines(defines: dict) -> None:
    """Raises ValueError unless every define is a known kernel knob set to an accepted value."""
    for k, v in defines.items():
        if k not in TUNABLE:
            raise ValueError(f"{k} is not a kernel knob (known: {', '.join(sorted(TUNABLE))})")
        if int(v) not in TUNABLE[k]:
            raise ValueError(f"{k}={v} is outside the accepted values {TUNABLE[k]}")


def variant_tag(defines: dict) -> str:
    """File-name tag of a variant build ("default" for none)."""
    return "_".join(f"{k[4:].lower()}-{int(v)}" for k, v in sorted(defines.items())) or "default"


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile libamk.so unless it is newer than every source. Returns its path."""
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= _newest_source_mtime():
        return LIB
    subprocess.run(_nvcc_cmd(LIB + ".tmp", {}, verbose), check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


def build_variant(defines: dict, force: bool = False) -> str:
    """Compile a variant of the library with compile-time knobs overridden (`{"AMK_PF_ITEMS": 6}`)
    into variants/libamk_<tag>.so beside the package; returns its path. Load it by setting
    AMK_LIB to that path before importing `decode_megakernel_launch_b200.amk`."""
    check_defines(defines)
    if not defines:
        return build(force)
    out_dir = os.path.join(PKG, "variants")
    os.makedirs(out_dir, exist_ok=True)
    out = os.path.join(out_dir, f"libamk_{variant_tag(defines)}.so")
    if not force and os.path.exists(out) and os.path.getmtime(out) >= _newest_source_mtime():
        return out
    subprocess.run(_nvcc_cmd(out + ".tmp", defines, False), check=True)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
