"""Build the CUDA library (libssd_mixer.so) in-tree for sm_100a with nvcc.

Usage: ``python -m hybrid_mamba_ssm_causal_b200.build [--force] [--verbose-ptxas] [--debug-bounds]``.
The shared library lands next to this file, so it travels with the source tree.
``--debug-bounds`` builds libssd_mixer_debug.so instead: the same kernels compiled with
-DSSD_DEBUG_BOUNDS, so that an index outside its buffer is recorded in the call's status word
(SSD_ERR_DEVICE) and its access skipped instead of faulting. The binding opens it when the
environment variable SSD_MIXER_LIBRARY names it.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB = os.path.join(HERE, "libssd_mixer.so")
DEBUG_LIB = os.path.join(HERE, "libssd_mixer_debug.so")
BUILD_DIR = os.path.join(HERE, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
              "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA library cannot be built")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str | None = None) -> bool:
    lib = lib or LIB
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
    deps += glob.glob(os.path.join(INCLUDE, "*.h")) + [os.path.abspath(__file__)]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, ptxas_verbose: bool = False, jobs: int | None = None, debug_bounds: bool = False) -> str:
    """Compile every csrc/*.cu for sm_100a and link libssd_mixer.so (cudart static), or the
    bounds-checked libssd_mixer_debug.so."""
    lib = DEBUG_LIB if debug_bounds else LIB
    if not force and not _stale(lib):
        return lib
    bdir = os.path.join(BUILD_DIR, "debug_bounds") if debug_bounds else BUILD_DIR
    os.makedirs(bdir, exist_ok=True)
    cc = nvcc()
    objs, procs = [], []
    extra = ["-Xptxas", "-v"] if ptxas_verbose else []
    if debug_bounds:
        extra.append("-DSSD_DEBUG_BOUNDS")
    for src in sources():
        obj = os.path.join(bdir, os.path.basename(src) + ".o")
        objs.append(obj)
        cmd = [cc, *ARCH, *NVCC_FLAGS, *extra, "-c", src, "-o", obj]
        procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)))
    failed = []
    for src, pr in procs:
        out, _ = pr.communicate()
        if out and (pr.returncode != 0 or ptxas_verbose):
            sys.stderr.write(out.decode(errors="replace"))
        if pr.returncode != 0:
            failed.append(src)
    if failed:
        raise RuntimeError(f"nvcc failed for: {failed}")
    tmp = lib + ".tmp"
    subprocess.run([cc, *ARCH, "-shared", "-o", tmp, *objs, "-lcuda"], check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--debug-bounds", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, ptxas_verbose=a.verbose_ptxas, debug_bounds=a.debug_bounds))
