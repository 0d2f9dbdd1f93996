"""Build the in-tree shared libraries with nvcc for sm_100a.

* libtsd.so          -- the attention library (C ABI in include/tsd.h)
* libtsd_workload.so -- the device side of the seeded workload generator

Usage: python -m top_sparse_decode_topk_b200.build [--verbose]
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-shared",
          "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]

LIBS = {
    "libtsd.so": ["tsd_api.cu", "tsd_decode.cu", "tsd_topk.cu", "tsd_label.cu", "tsd_stochastic.cu", "tsd_cp.cu", "tsd_static_ws.cu"],
    "libtsd_workload.so": ["workload_fill.cu"],
}
HEADERS = ["tsd_common.cuh", "tsd_plan.h", "tsd_args.h", "tsd_kvtile.cuh", "tsd_umma.cuh", "tsd_filter.cuh"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale(target: str, sources) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    deps = list(sources) + [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(INCLUDE, "tsd.h"), __file__]
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


def build(verbose: bool = False, force: bool = False) -> None:
    for lib, srcs in LIBS.items():
        target = os.path.join(PKG, lib)
        paths = [os.path.join(CSRC, s) for s in srcs]
        if not force and not _stale(target, paths):
            continue
        cmd = [nvcc()] + ARCH + COMMON + (["-Xptxas", "-v"] if verbose else []) + ["-o", target + ".tmp"] + paths
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError(f"nvcc failed for {lib}:\n{res.stdout}\n{res.stderr}")
        if verbose:
            sys.stdout.write(res.stdout + res.stderr)
        os.replace(target + ".tmp", target)


if __name__ == "__main__":
    build(verbose="--verbose" in sys.argv, force="--force" in sys.argv)
