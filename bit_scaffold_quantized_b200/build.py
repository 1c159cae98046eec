"""Build libdfssm.so in-tree for sm_100a (B200) with nvcc.

    python -m bit_scaffold_quantized_b200.build [--force] [--variant phases]

nvcc cross-compiles without a GPU.  The library links the CUDA runtime statically
and exports only the C ABI declared in include/dfssm.h.  The "phases" variant
(libdfssm_phases.so) is the same library with the batch-1 token kernel's per-phase
cycle counters compiled in (-DDFSSM_PHASE_TIMERS), for bit_scaffold_quantized_b200.phases.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libdfssm.so")
VARIANTS = {"": ([], LIB), "phases": (["-DDFSSM_PHASE_TIMERS"], os.path.join(PKG, "libdfssm_phases.so"))}
SOURCES = ["dfssm_api.cu"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-fvisibility=hidden",
    "-shared", "-cudart", "static",
    "--expt-relaxed-constexpr",
]


def _inputs():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh"))]
    files.append(os.path.join(INCLUDE, "dfssm.h"))
    files.append(os.path.abspath(__file__))
    return files


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False, variant: str = "") -> str:
    defines, lib = VARIANTS[variant]
    if not force and up_to_date(lib):
        return lib
    cmd = [NVCC, *FLAGS, *defines, "-I", INCLUDE, "-I", CSRC, "-o", lib + ".tmp",
           *[os.path.join(CSRC, s) for s in SOURCES]]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    v = sys.argv[sys.argv.index("--variant") + 1] if "--variant" in sys.argv else ""
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, variant=v))
