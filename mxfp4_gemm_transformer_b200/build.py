"""Builds libmxgemm.so in-tree with nvcc for sm_100a.

    python -m mxfp4_gemm_transformer_b200.build [--verbose-ptxas] [--trace]

The objects go to ``_build/`` beside this file and the shared library to
``libmxgemm.so`` in this package directory.  ``--trace`` builds the tracing
variant instead (kernels compiled with MXG_TRACE=1, so that
mx_debug_set_timeline records per-CTA milestones) as ``libmxgemm_trace.so``
from objects in ``_build/trace/``; load it with ``load(TRACE_LIB)``.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libmxgemm.so")
TRACE_LIB = os.path.join(HERE, "libmxgemm_trace.so")
SOURCES = ["mx_api.cu", "mx_quant.cu", "mx_norm_quant.cu", "mx_gemm.cu", "mx_gemm_pair.cu", "mx_decode.cu",
           "mx_noalloc.cu"]
DEPS = ["mx_internal.h", "mx_ptx.cuh", "mx_kernel_common.cuh", "mx_quant_common.cuh", "mx_decode_common.cuh"]
INCLUDE = os.path.join(os.path.dirname(HERE), "include")


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


FLAGS = [
    "-O3", "-std=c++17", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC,-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def _stale(obj: str, src: str) -> bool:
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    deps = [src] + [os.path.join(CSRC, d) for d in DEPS] + [os.path.join(INCLUDE, "mxgemm.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(verbose_ptxas: bool = False, force: bool = False, trace: bool = False) -> str:
    build_dir = os.path.join(BUILD, "trace") if trace else BUILD
    lib = TRACE_LIB if trace else LIB
    os.makedirs(build_dir, exist_ok=True)
    jobs = []
    for s in SOURCES:
        src = os.path.join(CSRC, s)
        obj = os.path.join(build_dir, s.replace(".cu", ".o"))
        if force or _stale(obj, src):
            cmd = [nvcc()] + FLAGS + (["-DMXG_TRACE=1"] if trace else []) + ["-I", INCLUDE, "-c", src, "-o", obj]
            if verbose_ptxas:
                cmd += ["-Xptxas", "-v"]
            jobs.append(cmd)
    if jobs:
        with cf.ThreadPoolExecutor(max_workers=len(jobs)) as ex:
            results = list(ex.map(lambda c: subprocess.run(c, capture_output=True, text=True), jobs))
        for cmd, r in zip(jobs, results):
            if r.returncode != 0 or (verbose_ptxas and r.stderr):
                sys.stderr.write(r.stderr)
            if r.returncode != 0:
                raise RuntimeError("nvcc failed: " + " ".join(cmd))
    objs = [os.path.join(build_dir, s.replace(".cu", ".o")) for s in SOURCES]
    if force or jobs or not os.path.exists(lib):
        cmd = [nvcc(), "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-o", lib] + objs
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            sys.stderr.write(r.stderr)
            raise RuntimeError("link failed")
    return lib


if __name__ == "__main__":
    print(build(verbose_ptxas="--verbose-ptxas" in sys.argv, force="--force" in sys.argv,
                trace="--trace" in sys.argv))
