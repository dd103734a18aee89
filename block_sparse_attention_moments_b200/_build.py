"""Compile the CUDA library (libsol_attn.so) for sm_100a, in-tree, with nvcc."""
from __future__ import annotations

import os
import shutil
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libsol_attn.so")
PROFILE_LIB = os.path.join(PKG, "libsol_attn_profile.so")
SOURCES = [os.path.join(PKG, "csrc", "sol_attn.cu")]
DEPS = [os.path.join(PKG, "csrc", f) for f in ("fused.cuh", "moments.cuh", "pool.cuh", "sm100_ptx.cuh",
                                                "topk_router.cuh")] + [
    os.path.join(ROOT, "include", "sol_attn.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
    "--expt-relaxed-constexpr",
]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libsol_attn.so")


def is_stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(f) > t for f in SOURCES + DEPS)


def build(force: bool = False, verbose: bool = False, extra_flags=(), profile: bool = False) -> str:
    """Build libsol_attn.so (or, with profile=True, libsol_attn_profile.so with the
    fused kernel's cycle accounting compiled in)."""
    lib = PROFILE_LIB if profile else LIB
    if not force and not is_stale(lib):
        return lib
    flags = [*NVCC_FLAGS, *extra_flags] + (["-DSOL_ATTN_PROFILE"] if profile else [])
    cmd = [nvcc_path(), *flags, "-I", os.path.join(ROOT, "include"), "-o", lib, *SOURCES]
    if verbose:
        print(" ".join(cmd))
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed ({r.returncode}):\n{r.stdout}\n{r.stderr}")
    if verbose and (r.stdout or r.stderr):
        print(r.stdout, r.stderr)
    return lib


if __name__ == "__main__":
    import sys
    print(build(force="--force" in sys.argv, verbose=True, profile="--profile" in sys.argv,
                extra_flags=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else []))
