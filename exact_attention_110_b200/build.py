"""Builds libfa.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m exact_attention_110_b200.build [--force] [--verbose]
"""
from __future__ import annotations

import os
import subprocess
import sys
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
CSRC = PKG / "csrc"
LIB = PKG / "libfa.so"

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-cudart", "static",
    "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (cand == "nvcc" or Path(cand).exists()):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(CSRC.glob("*.cu")) + sorted(CSRC.glob("*.cuh")) + sorted(CSRC.glob("*.h")) + [ROOT / "include" / "fa.h"]


# Kernels that re-balance registers with setmaxnreg: the launch allocation ptxas reports must
# be exactly what their warpgroup split adds up to (see ptx.cuh, reg_alloc/reg_dealloc).
REG_SPLIT_KERNELS = {"fa_fwd_kernel": 168, "fa_bwd_kernel": 128}


def check_register_split(ptxas_log: str) -> None:
    cur = None
    for line in ptxas_log.splitlines():
        if "Compiling entry function" in line:
            cur = next((k for k in REG_SPLIT_KERNELS if k in line), None)
        elif cur and "Used" in line and "registers" in line:
            n = int(line.split("Used")[1].split("registers")[0])
            if n != REG_SPLIT_KERNELS[cur]:
                raise RuntimeError(f"{cur}: launch allocation {n} registers/thread, the setmaxnreg split "
                                   f"assumes {REG_SPLIT_KERNELS[cur]}; refusing to build")
            cur = None


def build(force: bool = False, verbose: bool = False) -> Path:
    newest = max(p.stat().st_mtime for p in sources())
    if not force and LIB.exists() and LIB.stat().st_mtime >= newest:
        return LIB
    tmp = LIB.with_suffix(f".so.tmp{os.getpid()}")
    cmd = [nvcc(), "-Xptxas=-v", *NVCC_FLAGS, "-I", str(ROOT / "include"), str(CSRC / "libfa.cu"), "-o", str(tmp)]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or res.returncode != 0:
        sys.stdout.write(res.stdout)
        sys.stderr.write(res.stderr)
    if res.returncode != 0:
        raise subprocess.CalledProcessError(res.returncode, cmd)
    try:
        check_register_split(res.stderr + res.stdout)
    except RuntimeError:
        tmp.unlink(missing_ok=True)
        raise
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="--verbose" in sys.argv)
    print(LIB)
