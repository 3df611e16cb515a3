"""Builds the CUDA libraries in-tree for sm_100a.

  lib/libgpt2.so       bf16 product build (tcgen05 GEMMs, flash attention)
  lib/libgpt2_fp32.so  fp32 validation build (no tensor cores)

Usage: python -m transformer_lm_pretraining_b200.build [--force] [-j N]
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OUT = os.path.join(HERE, "lib")
OBJ = os.path.join(HERE, "_build")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "--expt-relaxed-constexpr",
         "-I", CSRC, "-I", os.path.join(ROOT, "include")]

COMMON = ["gpt2.cu", "kernel_abi.cu", "noalloc.cu", "encoder.cu", "layernorm.cu", "misc.cu",
          "attention.cu", "generate.cu"]
VARIANTS = {
    "libgpt2.so": (COMMON + ["gemm_tc.cu", "attention_tc.cu", "attention_bwd_tc.cu"], []),
    "libgpt2_fp32.so": (COMMON + ["gemm_simt.cu"], ["-DGPT2_FP32_VALIDATE"]),
}


def _headers():
    return [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))] + [
        os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))]


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src, obj, defs, verbose):
    cmd = [NVCC] + ARCH + FLAGS + defs + ["-c", os.path.join(CSRC, src), "-o", obj]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    return obj


def build(force: bool = False, jobs: int | None = None, verbose: bool = False) -> list[str]:
    os.makedirs(OUT, exist_ok=True)
    os.makedirs(OBJ, exist_ok=True)
    hdrs = _headers()
    built = []
    jobs = jobs or min(8, os.cpu_count() or 4)
    with cf.ThreadPoolExecutor(jobs) as ex:
        futs = {}
        plan = {}
        for lib, (srcs, defs) in VARIANTS.items():
            tag = "fp32" if defs else "bf16"
            objs = []
            for src in srcs:
                obj = os.path.join(OBJ, f"{tag}_{src[:-3]}.o")
                objs.append(obj)
                if force or _stale(obj, [os.path.join(CSRC, src)] + hdrs):
                    futs[ex.submit(_compile, src, obj, defs, verbose)] = obj
            plan[lib] = objs
        for f in cf.as_completed(futs):
            f.result()
    for lib, objs in plan.items():
        target = os.path.join(OUT, lib)
        if force or _stale(target, objs):
            cmd = [NVCC] + ARCH + ["-shared", "-o", target + ".tmp"] + objs
            r = subprocess.run(cmd, capture_output=True, text=True)
            if r.returncode != 0:
                raise RuntimeError(f"link failed for {lib}:\n{r.stdout}\n{r.stderr}")
            os.replace(target + ".tmp", target)
        built.append(target)
    return built


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-j", type=int, default=None)
    ap.add_argument("-v", action="store_true")
    a = ap.parse_args()
    for p in build(a.force, a.j, a.v):
        print(p)
    sys.exit(0)
