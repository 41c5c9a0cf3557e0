"""Builds libmoba.so in-tree from csrc/*.cu for sm_100a (nvcc cross-compiles without a GPU), and
its MOBA_CHECKS variant libmoba_checks.so (every device-side index derived from data on the device
checked against its buffer; see csrc/common.cuh).

    python -m block_sparse_long_moba_b200.build [--force] [--verbose] [--checks]
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmoba.so")
LIB_CHECKS = os.path.join(HERE, "libmoba_checks.so")
OBJ_DIR = os.path.join(HERE, "_build")
OBJ_DIR_CHECKS = os.path.join(HERE, "_build_checks")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-O3",
         "--expt-relaxed-constexpr", "-Xptxas", "-O3"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the MoBA CUDA library cannot be built")


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(
        os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(INCLUDE, "*.h")))


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in _deps())


def build(force: bool = False, verbose: bool = False, extra_flags=(), checks: bool = False) -> str:
    """Compile every csrc/*.cu to an object and link libmoba.so (libmoba_checks.so with
    checks=True, compiled with -DMOBA_CHECKS=1). Returns the library path."""
    lib = LIB_CHECKS if checks else LIB
    obj_dir = OBJ_DIR_CHECKS if checks else OBJ_DIR
    flags = [*extra_flags, "-DMOBA_CHECKS=1"] if checks else list(extra_flags)
    if not force and not needs_build(lib):
        return lib
    os.makedirs(obj_dir, exist_ok=True)
    cc = nvcc()
    objs = []
    procs = []
    for src in _sources():
        obj = os.path.join(obj_dir, os.path.basename(src)[:-3] + ".o")
        cmd = [cc, *ARCH, *FLAGS, *flags, "-I", INCLUDE, "-c", src, "-o", obj]
        if verbose:
            cmd += ["-Xptxas", "-v"]
            print(" ".join(cmd), flush=True)
        procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)))
        objs.append(obj)
    failed = []
    for src, p in procs:
        out, _ = p.communicate()
        text = out.decode(errors="replace")
        if p.returncode != 0:
            failed.append((src, text))
        elif verbose and text.strip():
            print(text, flush=True)
    if failed:
        msg = "\n".join(f"--- {s}\n{t}" for s, t in failed)
        raise RuntimeError(f"nvcc failed:\n{msg}")
    tmp = lib + ".tmp"
    link = [cc, *ARCH, "-shared", "-o", tmp, *objs]
    r = subprocess.run(link, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)
    if r.returncode != 0:
        raise RuntimeError("link failed:\n" + r.stdout.decode(errors="replace"))
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv,
                checks="--checks" in sys.argv))
