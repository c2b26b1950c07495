"""Builds the kdkl CUDA library in-tree: ``output_head_kl_b200/_lib/libkdkl.so``.

Every kernel is compiled for sm_100a only.  Run ``python -m output_head_kl_b200.build``
(or ``__graft_entry__.build()``); the result travels with the source tree.

A second library, ``_lib/libkdkl_debug.so``, is the same sources compiled with
``-DKDKL_DEBUG``: every list walk, partial-result slot, shared-memory list write,
TMA coordinate and lockstep slot is range-checked in the kernels, and a failed
check sets ``KDKL_DEV_BOUNDS`` in the device flag word and skips (or clamps) the
access instead of making it.  It stands in for a memory checker, which this
hardware pool does not offer; the tests run the ragged parity cases through it.

A third, ``_lib/libkdkl_prof.so``, is compiled with ``-DKDKL_PROFILE``: the same
kernels, which also count the SM cycles their TMA producer, MMA issuer and
epilogue spend at their barrier waits (``include/kdkl_profile.h``;
``python -m output_head_kl_b200.profile_roles`` reports them).
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
OUT_DIR = os.path.join(HERE, "_lib")
LIB = os.path.join(OUT_DIR, "libkdkl.so")
DEBUG_LIB = os.path.join(OUT_DIR, "libkdkl_debug.so")
PROFILE_LIB = os.path.join(OUT_DIR, "libkdkl_prof.so")
SOURCES = ("kernels.cu", "api.cu", "noalloc.cu")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-Xptxas", "-v"]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found")
    return path


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    deps.append(os.path.join(os.path.dirname(HERE), "include", "kdkl.h"))
    deps.append(os.path.join(os.path.dirname(HERE), "include", "kdkl_profile.h"))
    deps.append(os.path.abspath(__file__))
    return any(os.path.getmtime(p) > t for p in deps)


def _build_one(lib: str, prefix: str, defines, log_name: str):
    objs = []
    logs = []
    for src in SOURCES:
        obj = os.path.join(OUT_DIR, prefix + src.replace(".cu", ".o"))
        cmd = [nvcc(), *ARCH, *FLAGS, *defines, "-I", os.path.join(os.path.dirname(HERE), "include"), "-c",
               os.path.join(CSRC, src), "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        logs.append(r.stdout + r.stderr)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
        objs.append(obj)
    tmp = lib + ".tmp"
    cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    with open(os.path.join(OUT_DIR, log_name), "w") as f:
        f.write("\n".join(logs))
    return logs


def build(force: bool = False, verbose: bool = False, debug: bool = True, profile: bool = True) -> str:
    """Builds libkdkl.so (and, when asked, the bounds-checking libkdkl_debug.so and the
    cycle-counting libkdkl_prof.so)."""
    os.makedirs(OUT_DIR, exist_ok=True)
    if force or _stale(LIB):
        logs = _build_one(LIB, "", [], "ptxas.log")
        if verbose:
            print("\n".join(logs))
    if debug and (force or _stale(DEBUG_LIB)):
        _build_one(DEBUG_LIB, "dbg_", ["-DKDKL_DEBUG"], "ptxas_debug.log")
    if profile and (force or _stale(PROFILE_LIB)):
        _build_one(PROFILE_LIB, "prof_", ["-DKDKL_PROFILE"], "ptxas_prof.log")
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
