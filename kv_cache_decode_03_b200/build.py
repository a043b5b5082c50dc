"""Build libkvc.so in-tree for sm_100a with nvcc.

    python -m kv_cache_decode_03_b200.build [-v]

The shared library is written next to this file, so it travels with the
source tree; the package's loader refuses to run without it.
"""
from __future__ import annotations

import os
import subprocess
import sys
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
CSRC = PKG / "csrc"
INCLUDE = ROOT / "include"
LIB = PKG / "libkvc.so"
SOURCES = [CSRC / "kvc_api.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    cand = Path(os.environ.get("CUDA_HOME", "/usr/local/cuda")) / "bin" / "nvcc"
    return str(cand) if cand.exists() else "nvcc"


def build(verbose: bool = False, out: Path = LIB, extra: list[str] | None = None) -> Path:
    # compile beside the target and rename over it, so that a process that has the old
    # library loaded keeps an intact file
    tmp = out.with_name(f".{out.name}.{os.getpid()}.tmp")
    cmd = [nvcc(), "-O3", "-std=c++17", *ARCH, "-lineinfo", "--expt-relaxed-constexpr",
           "-Xcompiler", "-fPIC", "-shared", f"-I{INCLUDE}", f"-I{CSRC}",
           *(["-Xptxas", "-v"] if verbose else []), *(extra or []),
           *[str(s) for s in SOURCES], "-o", str(tmp)]
    try:
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            sys.stderr.write(res.stdout + res.stderr)
            raise RuntimeError("nvcc failed building libkvc.so")
        os.replace(tmp, out)
    finally:
        if tmp.exists():
            tmp.unlink()
    if verbose:
        sys.stderr.write(res.stderr)
    return out


def up_to_date() -> bool:
    if not LIB.exists():
        return False
    t = LIB.stat().st_mtime
    srcs = list(CSRC.glob("*")) + list(INCLUDE.glob("*.h"))
    return all(s.stat().st_mtime <= t for s in srcs)


if __name__ == "__main__":
    build(verbose="-v" in sys.argv)
    print(LIB)
