"""Build libfa.so in-tree with nvcc for sm_100a (no GPU needed to build).

    python -m exact_attention_146_b200.build            # build if sources changed
    python -m exact_attention_146_b200.build --force    # always rebuild
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
CSRC = PKG / "csrc"
INCLUDE = ROOT / "include"
LIB = PKG / "libfa.so"
SOURCES = [CSRC / "fa_fwd.cu", CSRC / "fa_bwd.cu"]
DEPS = SOURCES + sorted(CSRC.glob("*.cuh")) + sorted(CSRC.glob("*.h")) + sorted(INCLUDE.glob("*.h"))

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC",
    "-Xptxas", "-v",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and Path(cand).exists():
            return cand
    raise RuntimeError("nvcc not found")


def up_to_date() -> bool:
    if not LIB.exists():
        return False
    t = LIB.stat().st_mtime
    return all(p.stat().st_mtime <= t for p in DEPS)


def build(force: bool = False, verbose: bool = False) -> Path:
    if not force and up_to_date():
        return LIB
    tmp = LIB.with_name(LIB.name + f".tmp{os.getpid()}")
    # translation units compile in parallel to objects, then link into the shared library
    objs = [LIB.with_name(f"{src.stem}.{os.getpid()}.o") for src in SOURCES]
    procs = [subprocess.Popen([nvcc(), *NVCC_FLAGS, f"-I{INCLUDE}", f"-I{CSRC}", "-c", str(src), "-o", str(o)],
                              stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)
             for src, o in zip(SOURCES, objs)]
    try:
        failed = False
        for pr in procs:
            out, err = pr.communicate()
            if pr.returncode != 0:
                sys.stderr.write(out + err)
                failed = True
            elif verbose:
                sys.stderr.write(err)
        if failed:
            raise RuntimeError("nvcc failed building libfa.so")
        link = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", *map(str, objs),
                "-o", str(tmp)]
        res = subprocess.run(link, capture_output=True, text=True)
        if res.returncode != 0:
            sys.stderr.write(res.stdout + res.stderr)
            raise RuntimeError("nvcc failed linking libfa.so")
    finally:
        for o in objs:
            if o.exists():
                o.unlink()
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))
