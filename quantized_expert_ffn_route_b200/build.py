"""Builds libmoe.so for sm_100a with nvcc (in-tree, under _build/).

Usage: python -m quantized_expert_ffn_route_b200.build [--force] [--debug]

--debug builds the MOE_DEBUG variant into _build_debug/ (every index read from
a caller's buffer is also reported in the device error word when out of
range); the package loads it when MOE_LIBRARY=debug is set.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import subprocess
import sys
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
CSRC = PKG / "csrc"
OUT_DIR = PKG / "_build"
LIB = OUT_DIR / "libmoe.so"
DEBUG_DIR = PKG / "_build_debug"          # the MOE_DEBUG variant (reports out-of-range indices)
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
         "--expt-relaxed-constexpr", f"-I{ROOT / 'include'}", f"-I{CSRC}"]


def sources():
    return sorted(CSRC.glob("*.cu"))


def _headers_mtime():
    hs = list(CSRC.glob("*.cuh")) + list(CSRC.glob("*.h")) + list((ROOT / "include").glob("*.h"))
    return max((h.stat().st_mtime for h in hs), default=0.0)


def _compile(src: Path, extra, out_dir: Path) -> Path:
    obj = out_dir / (src.stem + ".o")
    if obj.exists() and obj.stat().st_mtime >= max(src.stat().st_mtime, _headers_mtime()):
        return obj
    cmd = [NVCC, *ARCH, *FLAGS, *extra, "-c", str(src), "-o", str(obj)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src.name}:\n{r.stderr}")
    if r.stderr.strip():
        sys.stderr.write(r.stderr)
    return obj


def build(force: bool = False, verbose_ptxas: bool = False, debug: bool = False) -> Path:
    """Compiles every source and links libmoe.so (debug: the MOE_DEBUG variant
    under _build_debug/); returns the library's path."""
    out_dir = DEBUG_DIR if debug else OUT_DIR
    lib_path = out_dir / "libmoe.so"
    out_dir.mkdir(parents=True, exist_ok=True)
    srcs = sources()
    extra = (["-Xptxas", "-v"] if verbose_ptxas else []) + (["-DMOE_DEBUG"] if debug else [])
    if force:
        for o in out_dir.glob("*.o"):
            o.unlink()
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(lambda s: _compile(s, extra, out_dir), srcs))
    newest = max(o.stat().st_mtime for o in objs)
    if force or not lib_path.exists() or lib_path.stat().st_mtime < newest:
        tmp = lib_path.with_suffix(f".{os.getpid()}.tmp")
        cmd = [NVCC, *ARCH, "-shared", "-o", str(tmp), *map(str, objs), "-lcudart",
               "-Xlinker", "-rpath=/usr/local/cuda/lib64"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stderr}")
        os.replace(tmp, lib_path)
    return lib_path


if __name__ == "__main__":
    p = build(force="--force" in sys.argv, verbose_ptxas="--ptxas-v" in sys.argv, debug="--debug" in sys.argv)
    print(p)
