"""Build the sm_100a shared libraries in-tree with nvcc.

* compressed_sparse_kv_b200/libdsv4kv.so   — the product (C ABI in include/dsv4kv.h)
* datagen/libdsv4kv_datagen.so             — the GPU twin of the input generator

Run ``python -m compressed_sparse_kv_b200.build`` (or call ``build()``).
Rebuilds only when a source is newer than its library.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-fvisibility=hidden", "-shared",
          "--expt-relaxed-constexpr"]

LIB = os.path.join(PKG, "libdsv4kv.so")
DATAGEN_LIB = os.path.join(ROOT, "datagen", "libdsv4kv_datagen.so")


def _stale(target: str, sources: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def _nvcc(sources: list[str], out: str, extra: list[str], verbose: bool) -> None:
    cmd = [NVCC, *ARCH, *COMMON, *extra, "-o", out, *sources]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError(f"nvcc failed building {out}")
    if verbose and (r.stdout or r.stderr):
        sys.stderr.write(r.stdout + r.stderr)


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> None:
    srcs = sorted(glob.glob(os.path.join(PKG, "csrc", "*.cu")))
    deps = srcs + glob.glob(os.path.join(PKG, "csrc", "*.h*")) + [os.path.join(ROOT, "include", "dsv4kv.h")]
    extra = ["-I", os.path.join(ROOT, "include")]
    if ptxas_info:
        extra += ["-Xptxas", "-v"]
    if force or _stale(LIB, deps):
        _nvcc(srcs, LIB, extra, verbose or ptxas_info)
    dsrc = [os.path.join(ROOT, "datagen", "csrc", "datagen.cu")]
    if force or _stale(DATAGEN_LIB, dsrc):
        _nvcc(dsrc, DATAGEN_LIB, [], verbose)


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True, ptxas_info="--ptxas" in sys.argv)
