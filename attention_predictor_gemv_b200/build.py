"""Builds the CUDA library in-tree: attention_predictor_gemv_b200/libdejavu.so.

    python -m attention_predictor_gemv_b200.build [--force] [--verbose]

nvcc cross-compiles for sm_100a on machines without a GPU.
"""

from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libdejavu.so")
# One translation unit per kernel family, compiled in parallel, then linked.
SOURCES = ["dv_api.cu", "dv_inst_legacy.cu", "dv_inst_legacy_attn.cu", "dv_inst_attn_in.cu", "dv_inst_attn_out.cu", "dv_inst_attn_out_f32.cu",
           "dv_inst_mlp.cu", "dv_inst_pred.cu", "dv_inst_tc.cu",
           "dv_inst_q8.cu"]
HEADERS = ["dv_common.cuh", "dv_kernels.cuh", "dv_fused.cuh", "dv_colowner.cuh", "dv_launch.cuh", "dv_launchers.cuh",
           "dv_api_kernels.cuh", "dv_stream.cuh", "dv_tc.cuh", "dv_tc_args.h",
           "dv_tc_launch.h"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr"]


def nvcc_path() -> str:
    for c in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libdejavu.so")


def _inputs():
    files = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    files.append(os.path.join(ROOT, "include", "dejavu.h"))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False, extra=(), csrc: str = CSRC, out: str = LIB) -> str:
    if not force and out == LIB and up_to_date():
        return out
    nvcc = nvcc_path()
    objdir = out + ".objs"
    os.makedirs(objdir, exist_ok=True)
    procs = []
    for src in SOURCES:
        obj = os.path.join(objdir, src.replace(".cu", ".o"))
        cmd = [nvcc, *ARCH, *FLAGS, *extra, "-I", os.path.join(ROOT, "include"), "-c", "-o", obj,
               os.path.join(csrc, src)]
        if verbose:
            print(" ".join(cmd), flush=True)
        procs.append((obj, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)))
    errors = []
    for obj, p in procs:
        log = p.communicate()[0]
        if p.returncode != 0:
            errors.append(log)
        elif verbose and log:
            print(log)
    if errors:
        raise RuntimeError("nvcc failed:\n" + "\n".join(errors))
    cmd = [nvcc, *ARCH, "-shared", "-o", out + ".tmp", *[o for o, _ in procs]]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc link failed:\n" + r.stdout + r.stderr)
    os.replace(out + ".tmp", out)
    shutil.rmtree(objdir, ignore_errors=True)
    return out


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-v", action="store_true", help="print register / shared memory use per kernel")
    a = ap.parse_args()
    extra = ["-Xptxas", "-v"] if a.ptxas_v else []
    print(build(force=a.force or a.ptxas_v, verbose=a.verbose or a.ptxas_v, extra=extra))
    sys.exit(0)
