"""Builds libsdm_b200.so in-tree with nvcc for sm_100a.

    python -m sparse_memory_linear_pkm_b200.build [--force] [--ptxas-verbose]
"""

from __future__ import annotations

import argparse
import os
import shutil
import subprocess
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
CSRC = PKG / "csrc"
INCLUDE = ROOT / "include"
LIBRARY = PKG / "libsdm_b200.so"
ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and Path(cand).exists():
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    return sorted(CSRC.glob("*.cu")) + sorted(CSRC.glob("*.cuh")) + sorted(CSRC.glob("*.h")) + [INCLUDE / "sdm.h"]


def up_to_date(out: Path = LIBRARY) -> bool:
    if not out.exists():
        return False
    t = out.stat().st_mtime
    return all(p.stat().st_mtime <= t for p in _sources())


def build(force: bool = False, ptxas_verbose: bool = False, out: Path = LIBRARY) -> Path:
    """Compiles every translation unit (csrc/*.cu) to an object in parallel,
    then links them into the shared library."""
    if not force and up_to_date(out):
        return out
    from concurrent.futures import ThreadPoolExecutor

    nvcc = nvcc_path()
    objdir = PKG / "_build"
    objdir.mkdir(exist_ok=True)
    common = [*ARCH_FLAGS, "-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC,-O2,-fvisibility=hidden",
              "-I", str(INCLUDE), "-I", str(CSRC)]
    if ptxas_verbose:
        common = ["-Xptxas", "-v", *common]
    units = sorted(CSRC.glob("*.cu"))
    objs = [objdir / (u.stem + f".{os.getpid()}.o") for u in units]

    def compile_one(pair):
        src, obj = pair
        return subprocess.run([nvcc, *common, "-c", str(src), "-o", str(obj)], capture_output=True, text=True)

    with ThreadPoolExecutor(max_workers=max(1, min(len(units), os.cpu_count() or 1))) as pool:
        results = list(pool.map(compile_one, zip(units, objs)))
    failed = False
    for src, res in zip(units, results):
        if res.stdout or res.stderr:
            print(res.stdout + res.stderr, end="")
        if res.returncode != 0:
            failed = True
            print(f"compiling {src.name} failed")
    if failed:
        raise subprocess.CalledProcessError(1, "nvcc")
    tmp = out.with_name(out.name + f".tmp{os.getpid()}")
    subprocess.run([nvcc, *ARCH_FLAGS, "-shared", "-Xcompiler", "-fPIC,-fvisibility=hidden", *map(str, objs),
                    "-o", str(tmp)], check=True)
    for obj in objs:
        obj.unlink()
    os.replace(tmp, out)
    return out


def main():
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true")
    args = ap.parse_args()
    print(build(force=args.force, ptxas_verbose=args.ptxas_verbose))


if __name__ == "__main__":
    main()
