"""Builds libdsa.so (the C ABI of include/dsa.h) from csrc/*.cu for sm_100a, in-tree.

    python -m sparse_attention_17_b200.build          # incremental
    python -m sparse_attention_17_b200.build --force  # rebuild
    python -m sparse_attention_17_b200.build --force --nvtx  # with NVTX ranges (tracing)
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor
from pathlib import Path

PKG = Path(__file__).resolve().parent
CSRC = PKG / "csrc"
INCLUDE = PKG.parent / "include"
LIB = PKG / "libdsa.so"
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and Path(cand).exists():
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list[Path]:
    return sorted(CSRC.glob("*.cu"))


def _stale() -> bool:
    if not LIB.exists():
        return True
    t = LIB.stat().st_mtime
    deps = sources() + sorted(CSRC.glob("*.cuh")) + sorted(CSRC.glob("*.h")) + [INCLUDE / "dsa.h"]
    return any(p.stat().st_mtime > t for p in deps)


def build(force: bool = False, verbose: bool = False, nvtx: bool = False) -> Path:
    """Compiles every kernel file into libdsa.so next to this module (sm_100a only).  With
    nvtx, the host side marks layers and index windows as NVTX ranges for timelines."""
    if not force and not _stale():
        return LIB
    build_dir = PKG / "_build"
    build_dir.mkdir(exist_ok=True)
    objs, cmds = [], []
    for src in sources():
        obj = build_dir / (src.stem + ".o")
        cmds.append([nvcc(), *ARCH, "-std=c++17", "-O3", "-lineinfo", "-Xcompiler", "-fPIC",
                     "-Xptxas", "-v" if verbose else "-O3", f"-I{INCLUDE}",
                     *(["-DDSA_NVTX=1"] if nvtx else []), "-c", str(src), "-o", str(obj)])
        objs.append(str(obj))
    # the kernel files compile independently: one nvcc per file, in parallel
    with ThreadPoolExecutor(max_workers=min(len(cmds), os.cpu_count() or 1)) as pool:
        for fut in [pool.submit(subprocess.run, c, check=True) for c in cmds]:
            fut.result()
    tmp = LIB.with_suffix(f".so.{os.getpid()}.tmp")
    subprocess.run([nvcc(), *ARCH, "-shared", "-o", str(tmp), *objs], check=True)
    os.replace(tmp, LIB)
    return LIB


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true", help="print ptxas register/smem usage")
    ap.add_argument("--nvtx", action="store_true", help="NVTX ranges per layer and window")
    a = ap.parse_args(argv)
    print(build(force=a.force, verbose=a.verbose, nvtx=a.nvtx))
    return 0


if __name__ == "__main__":
    sys.exit(main())
