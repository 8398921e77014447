"""Build libgoldwkv.so in-tree for sm_100a with nvcc.

    python -m linear_attention_rnn_finch_b200.build [-v] [--ptxas-info]

Each ``csrc/*.cu`` is compiled to an object under ``_build/`` and the objects are linked
into ``linear_attention_rnn_finch_b200/libgoldwkv.so`` (CUDA runtime linked statically, so
the library does not depend on a particular libcudart.so being on the loader path).
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


def _compile(src: Path, ptxas_info: bool, verbose: bool) -> Path:
    obj = BUILD / (src.stem + ".o")
    cmd = [nvcc(), *ARCH, *CFLAGS, "-c", str(src), "-o", str(obj)]
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


def up_to_date() -> bool:
    return LIB.exists() and LIB.stat().st_mtime >= _deps_mtime()


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> Path:
    if not force and not ptxas_info and up_to_date():
        return LIB
    BUILD.mkdir(exist_ok=True)
    srcs = sources()
    with cf.ThreadPoolExecutor(max_workers=min(len(srcs), os.cpu_count() or 1)) as ex:
        objs = list(ex.map(lambda s: _compile(s, ptxas_info, verbose), srcs))
    tmp = LIB.with_suffix(".so.tmp")
    # cuBLASLt serves the plain GEMMs of the GOLD compression entry points
    cmd = [nvcc(), *ARCH, "-shared", "-o", str(tmp), *map(str, objs), "-lcublasLt"]
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"link failed:\n{res.stdout}\n{res.stderr}")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true")
    ap.add_argument("--force", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, ptxas_info=a.ptxas_info))
