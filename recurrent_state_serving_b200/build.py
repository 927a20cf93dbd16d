"""Build libdeltalog.so (sm_100a) in-tree with nvcc.

    python -m recurrent_state_serving_b200.build [--force] [--verbose]

Objects go to _build/ at the repository root; the shared library is written next
to this file, where the Python binding loads it.  The CUDA runtime is linked
statically, so the library loads on a machine without a GPU driver (symbols can
be inspected there; compute calls need a B200).
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libdeltalog.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-fvisibility=hidden",
          "-I", INCLUDE, "-I", CSRC]
STEP_DKS = (16, 64, 128)


def _sources():
    units = [("api", os.path.join(CSRC, "api.cpp"), []),
             ("kernels_merge", os.path.join(CSRC, "kernels_merge.cu"), []),
             ("kernels_warp_head", os.path.join(CSRC, "kernels_warp_head.cu"), []),
             ("noalloc", os.path.join(CSRC, "noalloc.cu"), [])]
    for dk in STEP_DKS:
        units.append((f"kernels_step_dk{dk}", os.path.join(CSRC, "kernels_step.cu"),
                      [f"-DDL_STEP_DK={dk}"]))
    return units


def _deps():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    files.append(os.path.join(INCLUDE, "deltalog.h"))
    files.append(os.path.abspath(__file__))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _deps())


def build(force: bool = False, verbose: bool = False, extra_flags=()) -> str:
    if not force and not extra_flags and up_to_date():
        return LIB
    os.makedirs(BUILD, exist_ok=True)

    def compile_one(unit):
        name, src, defs = unit
        obj = os.path.join(BUILD, name + ".o")
        cmd = [NVCC, *ARCH, *COMMON, *defs, *extra_flags, "-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {name}:\n{r.stdout}\n{r.stderr}")
        if verbose and (r.stdout or r.stderr):
            print(r.stdout + r.stderr, flush=True)
        return obj

    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(compile_one, _sources()))
    tmp = LIB + ".tmp"
    cmd = [NVCC, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print registers/spills (-Xptxas -v)")
    a = ap.parse_args()
    extra = ["-Xptxas", "-v"] if a.ptxas_info else []
    print(build(force=a.force or a.ptxas_info, verbose=a.verbose or a.ptxas_info, extra_flags=extra))


if __name__ == "__main__":
    main()
