"""Build the CUDA library (sm_100a) in-tree: quantized_int8_gemm_q4_b200/_build/libdllm_qgemm.so."""
from __future__ import annotations

import os
import subprocess
import sys
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
CSRC = PKG / "csrc"
OUT = PKG / "_build" / "libdllm_qgemm.so"
SOURCES = [CSRC / "dllm.cu"]
DEPS = sorted(CSRC.glob("*.cu*")) + [ROOT / "include" / "dllm_qgemm.h"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.isabs(c) and os.path.exists(c) or not os.path.isabs(c)):
            return c
    return "nvcc"


def build(force: bool = False, verbose: bool = False) -> Path:
    OUT.parent.mkdir(parents=True, exist_ok=True)
    newest = max(p.stat().st_mtime for p in DEPS)
    if not force and OUT.exists() and OUT.stat().st_mtime >= newest:
        return OUT
    tmp = str(OUT) + ".tmp"
    cmd = [nvcc(), *NVCC_FLAGS, *(["-Xptxas", "-v"] if verbose else []), "-I", str(ROOT / "include"),
           *map(str, SOURCES), "-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
