"""In-tree build of libmoe.so for sm_100a (nvcc for the kernels, g++ for the packer).

    python -m bit_routed_expert_fp32_b200.build [--force]
"""
from __future__ import annotations

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OUT = os.path.join(PKG, "libmoe.so")
OBJDIR = os.path.join(PKG, "_build")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-Xptxas", "-v", "-I", INCLUDE, "-I", CSRC]
CXX_FLAGS = ["-O2", "-std=c++17", "-fPIC", "-I", INCLUDE]

CU = ["route.cu", "decode_ffn.cu", "decode_fused.cu", "prefill_tc.cu", "ep.cu", "cache.cu", "api.cu", "static_ws.cu"]
CPP = ["pack.cpp"]
HEADERS = ["common.cuh", "kernels.h", "dequant.cuh", "operands.cuh", "iqmma.cuh"]


def _newer(src_list, target):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in src_list)


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(OBJDIR, exist_ok=True)
    deps = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(INCLUDE, "moe.h")]
    jobs = []
    objs = []
    for f in CU + CPP:
        src = os.path.join(CSRC, f)
        obj = os.path.join(OBJDIR, f + ".o")
        objs.append(obj)
        if force or _newer([src] + deps, obj):
            if f.endswith(".cu"):
                cmd = [NVCC, *NVCC_FLAGS, "-c", src, "-o", obj]
            else:
                cmd = ["g++", *CXX_FLAGS, "-c", src, "-o", obj]
            jobs.append((f, cmd))

    def run(job):
        name, cmd = job
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"compiling {name} failed:\n{r.stdout}\n{r.stderr}")
        return name, r.stderr

    with ThreadPoolExecutor(max(1, len(jobs))) as ex:
        for name, log in ex.map(run, jobs):
            if verbose:
                print(f"== {name}\n{log}")
    if force or jobs or _newer(objs, OUT):
        tmp = OUT + f".tmp{os.getpid()}"
        subprocess.check_call([NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-o", tmp, *objs])
        os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
