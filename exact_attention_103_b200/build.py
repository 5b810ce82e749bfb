"""Builds libattn.so (the CUDA library) in-tree for sm_100a with nvcc.

Usage: ``python -m exact_attention_103_b200.build [--force]``.  Objects go to
``_build/`` beside this file; the shared library to ``libattn.so``; ptxas
register/spill reports to ``_build/ptxas.log``.
"""
from __future__ import annotations

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OBJ = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libattn.so")
SOURCES = ["attn_api.cu", "attn_fwd_sm100.cu", "attn_bwd_sm100.cu", "selftest_sm100.cu",
           "attn_noalloc.cu"]
HEADERS = ["attn_fwd_sm100.h", "attn_bwd_sm100.h", "attn_internal.h", "sm100_ptx.cuh", "softmax_math.cuh", "exp2_poly.h"]
PUBLIC_HEADERS = [os.path.join(ROOT, "include", h) for h in ("attn.h", "attn_selftest.h")]
NVCC = os.environ.get("NVCC", "nvcc")
# Extra nvcc flags (e.g. -DATTN_P_SPLIT=4 to change how P~ is handed to the PV product).
EXTRA = os.environ.get("ATTN_NVCC_EXTRA", "").split()
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-Xptxas", "-v",
         "-I", os.path.join(ROOT, "include")]


def _newest(paths):
    return max(os.path.getmtime(p) for p in paths)


def build(force: bool = False, verbose: bool = False) -> str:
    srcs = [os.path.join(CSRC, s) for s in SOURCES]
    deps = srcs + [os.path.join(CSRC, h) for h in HEADERS] + PUBLIC_HEADERS + [__file__]
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= _newest(deps):
        return LIB
    os.makedirs(OBJ, exist_ok=True)

    def compile_one(src):
        obj = os.path.join(OBJ, os.path.basename(src).replace(".cu", ".o"))
        cmd = [NVCC, *FLAGS, *EXTRA, "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
        return obj, r.stderr

    with ThreadPoolExecutor(max_workers=len(srcs)) as ex:
        results = list(ex.map(compile_one, srcs))
    with open(os.path.join(OBJ, "ptxas.log"), "w") as f:
        for _, log in results:
            f.write(log)
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", tmp,
           *[o for o, _ in results]]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    if verbose:
        print(open(os.path.join(OBJ, "ptxas.log")).read())
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
