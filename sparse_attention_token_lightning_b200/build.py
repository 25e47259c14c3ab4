"""Build the CUDA library ``libli.so`` in-tree for sm_100a with nvcc.

``python -m sparse_attention_token_lightning_b200.build`` (or ``build()``) compiles every
``csrc/*.cu`` into the package directory. No GPU is needed to build.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
CSRC = PKG / "csrc"
INCLUDE = ROOT / "include"
LIB = PKG / "libli.so"
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and Path(cand).exists():
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(CSRC.glob("*.cu"))


def headers():
    return sorted(CSRC.glob("*.cuh")) + sorted(INCLUDE.glob("*.h"))


# Test build: every bounded device wait gives up after 1 ms, and the score kernel's TMA producer
# issues no load (so no bulk copy is ever in flight and the MMA warp's first wait runs out). The
# tests load it beside libli.so to drive the timeout exit; nothing else uses it.
WAIT_TEST_LIB = PKG / "libli_waittest.so"
WAIT_TEST_FLAGS = ("-DLI_WAIT_LIMIT_NS=1000000ull", "-DLI_TEST_NO_LOADS=1")


# Bounds-checked build: every computed shared- or global-memory index the kernels form passes a
# check first; a failing check sets LI_DEVERR_BOUNDS in the status word and the access is
# skipped (see in_bounds() in csrc/li_internal.cuh). Same C ABI; loaded by the tests beside
# libli.so, whose release kernels it must match bit for bit.
DEBUG_LIB = PKG / "libli_debug.so"
DEBUG_FLAGS = ("-DLI_DEBUG=1",)


def up_to_date(lib: Path = LIB) -> bool:
    if not lib.exists():
        return False
    t = lib.stat().st_mtime
    return all(f.stat().st_mtime <= t for f in sources() + headers())


def build_wait_test(force: bool = False, verbose: bool = False) -> Path:
    """libli_waittest.so (see WAIT_TEST_FLAGS)."""
    return build(force, verbose, WAIT_TEST_FLAGS, lib=WAIT_TEST_LIB, obj_sub="waittest")


def build_debug(force: bool = False, verbose: bool = False) -> Path:
    """libli_debug.so (see DEBUG_FLAGS)."""
    return build(force, verbose, DEBUG_FLAGS, lib=DEBUG_LIB, obj_sub="debug")


def build(force: bool = False, verbose: bool = False, extra=(), lib: Path = LIB,
          obj_sub: str = "") -> Path:
    if not force and up_to_date(lib):
        return lib
    obj_dir = PKG / "_build" / obj_sub if obj_sub else PKG / "_build"
    obj_dir.mkdir(parents=True, exist_ok=True)
    objs = []
    procs = []
    common = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
              "-I", str(INCLUDE), "-I", str(CSRC), *extra]
    for src in sources():
        obj = obj_dir / (src.stem + ".o")
        objs.append(obj)
        cmd = common + ["-c", str(src), "-o", str(obj)]
        if verbose:
            print(" ".join(cmd), flush=True)
        procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)))
    failed = []
    for src, pr in procs:
        out, _ = pr.communicate()
        if pr.returncode != 0 or verbose:
            sys.stdout.write(out.decode(errors="replace"))
        if pr.returncode != 0:
            failed.append(src.name)
    if failed:
        raise RuntimeError(f"nvcc failed for {failed}")
    tmp = lib.with_suffix(".so.tmp")
    link = [nvcc(), *ARCH, "-shared", "-o", str(tmp), *map(str, objs)]
    subprocess.run(link, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    build_wait_test(force="--force" in sys.argv, verbose="-v" in sys.argv)
    build_debug(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
