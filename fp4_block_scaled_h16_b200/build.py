"""Build libfp4.so in-tree for sm_100a with nvcc (no JIT cache, no torch extension).

    python -m fp4_block_scaled_h16_b200.build [--force]
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libfp4.so")
SOURCES = ["fp4_api.cu", "quantize.cu", "quantize_rows_f32.cu", "quantize_cols_bf16.cu", "quantize_cols_f32.cu",
           "requantize_cols.cu", "gemm.cu", "gemm_db.cu", "quantize_noalloc.cu", "rotate.cu", "mxnorm.cu", "ufp4_split.cu",
           "outctl.cu", "gemm_outctl.cu", "gemm_pair.cu", "quantize_dual.cu"]
HEADERS = ["fp4_device.cuh", "internal.h", "sm100.cuh", "quant_common.cuh", "quant_rows.cuh", "quant_cols.cuh"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
    "--expt-relaxed-constexpr",
    "-cudart", "static",
    "-I", os.path.join(ROOT, "include"),
]


def _inputs():
    files = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    files.append(os.path.join(ROOT, "include", "fp4.h"))
    files.append(os.path.abspath(__file__))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    objs = []
    build_dir = os.path.join(HERE, "_build")
    os.makedirs(build_dir, exist_ok=True)
    procs = []
    for src in SOURCES:
        obj = os.path.join(build_dir, src.replace(".cu", ".o"))
        cmd = [NVCC, *FLAGS, "-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
            print(" ".join(cmd))
        procs.append(subprocess.Popen(cmd))
        objs.append(obj)
    rc = [p.wait() for p in procs]
    if any(rc):
        raise RuntimeError("nvcc failed (%s)" % rc)
    tmp = LIB + ".tmp%d" % os.getpid()
    subprocess.check_call([NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-cudart", "static", "-o", tmp, *objs])
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
