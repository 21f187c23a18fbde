"""Build libqlora_nf4.so in place (nvcc, sm_100a only).

    python -m bit_nf4_quantized_15_b200.build [--verbose]

The library is a plain C-ABI shared object; it links the CUDA runtime
statically and reaches the driver's tensor-map encoder through
cudaGetDriverEntryPoint, so it needs nothing on the library path.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libqlora_nf4.so")
SOURCES = ["api.cu", "engine.cu", "engine_pair.cu", "gemv.cu", "gemv_bwd.cu", "quant.cu", "adapters.cu",
           "noalloc.cu", "nf4_tables.cpp"]
HEADERS = ["common.cuh", "engine_util.cuh", "internal.h"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(ROOT, "include", "qlora_nf4.h"))
    deps.append(os.path.abspath(__file__))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    cmd = [
        nvcc_path(), "-shared", "-o", LIB + ".tmp",
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-O3", "-lineinfo", "-std=c++17",
        "-Xcompiler", "-fPIC,-O2,-fvisibility=hidden",
        "-I", os.path.join(ROOT, "include"),
    ]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, f) for f in SOURCES]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed building libqlora_nf4.so")
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
