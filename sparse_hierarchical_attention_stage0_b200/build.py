"""Build libdash.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python sparse_hierarchical_attention_stage0_b200/build.py [--force] [--verbose] [--debug]

Each .cu under csrc/ is compiled to an object (-gencode arch=compute_100a,code=sm_100a,
-O3, -lineinfo, no fast-math: the routing needs IEEE division, expf and logf) and linked
with the static CUDA runtime into sparse_hierarchical_attention_stage0_b200/libdash.so.
--debug builds libdash_debug.so instead: the same sources with DASH_DEBUG defined, whose
kernels check their computed indices against the buffers' bounds and report a failed check
as DASH_ERR_BOUNDS through the device status word.
"""
from __future__ import annotations

import argparse
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libdash.so")
BUILD = os.path.join(HERE, "_build")
LIB_DEBUG = os.path.join(HERE, "libdash_debug.so")
BUILD_DEBUG = os.path.join(HERE, "_build_debug")
SOURCES = ["stage0.cu", "route.cu", "attend.cu", "attend_tc.cu", "attend_fa.cu", "attend_pair.cu", "vtranspose.cu",
           "decode.cu", "backward.cu", "dash_api.cu", "dash_static_ws.cu"]
HEADERS = ["dash_common.cuh", "kernels.cuh", "attn_warp.cuh", "tc_common.cuh"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-I", os.path.join(ROOT, "include")]


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False,
          debug: bool = False) -> str:
    lib, bdir = (LIB_DEBUG, BUILD_DEBUG) if debug else (LIB, BUILD)
    os.makedirs(bdir, exist_ok=True)
    headers = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(ROOT, "include", "dash.h")]
    objs, procs = [], []
    for src in SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(bdir, src.replace(".cu", ".o"))
        objs.append(o)
        if force or _stale(o, [s] + headers):
            cmd = [NVCC, *ARCH, *FLAGS, *(["-DDASH_DEBUG"] if debug else []), "-c", s, "-o", o]
            if ptxas_info:
                cmd += ["-Xptxas", "-v"]
            if verbose:
                print(" ".join(cmd), flush=True)
            procs.append((cmd, subprocess.Popen(cmd)))
            if len(procs) >= max(1, min(8, os.cpu_count() or 1)):
                c, pr = procs.pop(0)
                if pr.wait() != 0:
                    raise subprocess.CalledProcessError(pr.returncode, c)
    for c, pr in procs:
        if pr.wait() != 0:
            raise subprocess.CalledProcessError(pr.returncode, c)
    if force or _stale(lib, objs):
        cmd = [NVCC, *ARCH, "-shared", "-cudart", "static", "-o", lib, *objs]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.check_call(cmd)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true")
    ap.add_argument("--debug", action="store_true")
    a = ap.parse_args()
    print(build(a.force, a.verbose, a.ptxas_info, a.debug))
    sys.exit(0)
