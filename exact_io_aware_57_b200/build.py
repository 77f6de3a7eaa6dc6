"""Build libattn.so in-tree for sm_100a with nvcc (no JIT cache, no torch).

Usage: python -m exact_io_aware_57_b200.build [--force] [-j N]
"""
from __future__ import annotations

import argparse
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor
from pathlib import Path

PKG = Path(__file__).resolve().parent
CSRC = PKG / "csrc"
OBJ = PKG / "_build"
LIB = PKG / "libattn.so"
SOURCES = ["attn_api.cu", "kernels_f32.cu", "fwd_launch.cu", "fwd_pp_sm100.cu", "fwd_db_sm100.cu", "bwd_sm100.cu", "naive.cu", "bwd_noalloc.cu", "merge.cu", "selftest.cu", "quant_fp8.cu"]
HEADERS = ["common.cuh", "kernels.h"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-std=c++17", "-O3", "-lineinfo", "-Xcompiler", "-fPIC", "-gencode", "arch=compute_100a,code=sm_100a",
         "--expt-relaxed-constexpr", "-Xptxas", "-warn-spills"]


def _stale(obj: Path, src: Path) -> bool:
    if not obj.exists():
        return True
    deps = [src, *(CSRC / h for h in HEADERS), PKG.parent / "include" / "attn.h"]
    return any(d.stat().st_mtime > obj.stat().st_mtime for d in deps)


def _compile(src: str, force: bool, verbose: bool) -> Path:
    s = CSRC / src
    o = OBJ / (Path(src).stem + ".o")
    if force or _stale(o, s):
        cmd = [NVCC, *FLAGS, *(["-Xptxas", "-v"] if verbose else []), "-c", str(s), "-o", str(o)]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stderr}")
        if verbose:
            sys.stderr.write(r.stderr)
    return o


def build(force: bool = False, jobs: int = 4, verbose: bool = False) -> Path:
    OBJ.mkdir(exist_ok=True)
    with ThreadPoolExecutor(max_workers=jobs) as ex:
        objs = list(ex.map(lambda s: _compile(s, force, verbose), SOURCES))
    if force or not LIB.exists() or any(o.stat().st_mtime > LIB.stat().st_mtime for o in objs):
        cmd = [NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", *map(str, objs), "-o", str(LIB)]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stderr}")
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("-j", type=int, default=4)
    a = ap.parse_args()
    print(build(a.force, a.j, a.verbose))
