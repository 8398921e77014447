"""Build libgoldwkv.so in-tree for sm_100a with nvcc.

    python -m linear_attention_rnn_finch_b200.build [-v] [--ptxas-info] [--debug]

Each ``csrc/*.cu`` is compiled to an object under ``_build/`` and the objects are linked
into ``linear_attention_rnn_finch_b200/libgoldwkv.so`` (CUDA runtime linked statically, so
the library does not depend on a particular libcudart.so being on the loader path).

``--debug`` builds ``libgoldwkv_debug.so`` instead (objects under ``_build_debug/``), with
``-DGW_DEBUG``: the chunked kernels check the coordinates of every copy and store and the
index ranges of their threads on the device; a failed check sets bit 1 of the call's
status word and skips the access.  Same ABI, slower; for tests and debugging.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import shutil
import subprocess
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
CSRC = PKG / "csrc"
BUILD = PKG / "_build"
LIB = PKG / "libgoldwkv.so"
BUILD_DEBUG = PKG / "_build_debug"
LIB_DEBUG = PKG / "libgoldwkv_debug.so"
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
          f"-I{ROOT / 'include'}", f"-I{CSRC}"]


def nvcc() -> str:
    exe = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not Path(exe).exists():
        raise RuntimeError("nvcc not found; the CUDA 12.9 toolkit is required to build libgoldwkv")
    return exe


def sources():
    return sorted(CSRC.glob("*.cu"))


def _deps_mtime():
    return max(p.stat().st_mtime for p in list(CSRC.glob("*")) + [ROOT / "include" / "goldwkv.h"])


def _compile(src: Path, ptxas_info: bool, verbose: bool, debug: bool = False) -> Path:
    obj = (BUILD_DEBUG if debug else BUILD) / (src.stem + ".o")
    cmd = [nvcc(), *ARCH, *CFLAGS, *(["-DGW_DEBUG"] if debug else []), "-c", str(src), "-o",
           str(obj)]
    if ptxas_info:
        cmd.insert(1, "-Xptxas=-v")
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src.name}:\n{res.stdout}\n{res.stderr}")
    if ptxas_info or verbose:
        print(res.stderr, flush=True)
    return obj


def up_to_date(debug: bool = False) -> bool:
    lib = LIB_DEBUG if debug else LIB
    return lib.exists() and lib.stat().st_mtime >= _deps_mtime()


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False,
          debug: bool = False) -> Path:
    lib = LIB_DEBUG if debug else LIB
    if not force and not ptxas_info and up_to_date(debug):
        return lib
    (BUILD_DEBUG if debug else BUILD).mkdir(exist_ok=True)
    srcs = sources()
    with cf.ThreadPoolExecutor(max_workers=min(len(srcs), os.cpu_count() or 1)) as ex:
        objs = list(ex.map(lambda s: _compile(s, ptxas_info, verbose, debug), srcs))
    tmp = lib.with_suffix(".so.tmp")
    cmd = [nvcc(), *ARCH, "-shared", "-o", str(tmp), *map(str, objs)]
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"link failed:\n{res.stdout}\n{res.stderr}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true")
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--debug", action="store_true", help="build libgoldwkv_debug.so (-DGW_DEBUG)")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, ptxas_info=a.ptxas_info, debug=a.debug))
