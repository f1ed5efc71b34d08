"""Build libmoe.so (the C-ABI CUDA library) in-tree for sm_100a with nvcc.

    python -m expert_dispatch_gemm_b200.build [--force] [--verbose-ptxas]

Objects go to expert_dispatch_gemm_b200/_build/, the shared library to
expert_dispatch_gemm_b200/libmoe.so. The checked build of the same sources
(-DMOE_DEBUG_CHECKS: every out-of-range index read from the routing outputs is
reported as kErrBadIndex in the error word) goes to libmoe_checked.so, its
objects to _build_checked/. The FP32 FFMA throughput probe that the benchmark
uses for the router's roof goes to libmoe_probe.so. No GPU is needed to
build.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libmoe.so")
INCLUDE = os.path.join(ROOT, "include")

SOURCES = ["api.cu", "router.cu", "assign.cu", "dispatch_combine.cu", "ffn_f32.cu",
           "gemm_tc.cu", "gemm_swap.cu", "route_noalloc.cu", "gemm_bwd.cu", "bwd.cu",
           "bwd_f32.cu"]
PROBE_SOURCES = ["probe.cu"]
PROBE_LIB = os.path.join(PKG, "libmoe_probe.so")
CHECKED_LIB = os.path.join(PKG, "libmoe_checked.so")
BUILD_CHECKED = os.path.join(PKG, "_build_checked")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _headers():
    hs = [os.path.join(INCLUDE, "moe.h")]
    hs += [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    return hs


def _flags(extra=()):
    return ["-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC",
            "-Xcompiler", "-fvisibility=hidden", "-I", INCLUDE, "-I", CSRC,
            "--expt-relaxed-constexpr", "-DMOE_BUILD", *extra]


def build(force: bool = False, ptxas_verbose: bool = False, checked: bool = True) -> str:
    lib = _build_lib(SOURCES, LIB, force, ptxas_verbose)
    _build_lib(PROBE_SOURCES, PROBE_LIB, force, ptxas_verbose)
    if checked:
        _build_lib(SOURCES, CHECKED_LIB, force, False, BUILD_CHECKED, ["-DMOE_DEBUG_CHECKS"])
    return lib


def _build_lib(sources, out_lib, force, ptxas_verbose, build_dir=BUILD, defines=()) -> str:
    os.makedirs(build_dir, exist_ok=True)
    hdr_t = max(os.path.getmtime(h) for h in _headers())
    jobs = []
    for src in sources:
        s = os.path.join(CSRC, src)
        o = os.path.join(build_dir, src.replace(".cu", ".o"))
        if force or ptxas_verbose or not os.path.exists(o) or \
                os.path.getmtime(o) < max(os.path.getmtime(s), hdr_t):
            extra = ["-Xptxas", "-v"] if ptxas_verbose else []
            jobs.append([nvcc(), *_flags([*extra, *defines]), "-c", s, "-o", o])
    if jobs:
        with cf.ThreadPoolExecutor(max_workers=min(8, len(jobs))) as ex:
            results = list(ex.map(lambda c: subprocess.run(c, capture_output=True, text=True),
                                  jobs))
        for cmd, r in zip(jobs, results):
            if ptxas_verbose or r.returncode != 0:
                sys.stderr.write(r.stdout + r.stderr)
            if r.returncode != 0:
                raise RuntimeError("nvcc failed: " + " ".join(cmd))
    objs = [os.path.join(build_dir, s.replace(".cu", ".o")) for s in sources]
    if force or jobs or not os.path.exists(out_lib) or \
            os.path.getmtime(out_lib) < max(os.path.getmtime(o) for o in objs):
        # --no-undefined: a symbol missing from the sources fails the build,
        # not the first dlopen on a GPU machine
        cmd = [nvcc(), *ARCH, "-shared", "-Xcompiler", "-fPIC", "-Xlinker", "--no-undefined",
               "-o", out_lib + ".tmp", *objs]
        subprocess.check_call(cmd)
        os.replace(out_lib + ".tmp", out_lib)
    return out_lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, ptxas_verbose="--verbose-ptxas" in sys.argv))
