"""Build the in-tree shared libraries with nvcc for sm_100a.

    python -m sparse_decode_attention_spkv_b200.build

produces ``libspkv.so`` (the SP-KV kernels behind the C ABI of include/spkv.h) and
``inputs/libspkv_inputs.so`` (the device side of the seeded input generator).
Objects are cached under ``_build/`` and rebuilt when a source is newer.
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
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-I", os.path.join(ROOT, "include")]

LIBS = {
    os.path.join(PKG, "libspkv.so"): sorted(glob.glob(os.path.join(PKG, "csrc", "*.cu"))),
    os.path.join(PKG, "inputs", "libspkv_inputs.so"): [os.path.join(PKG, "inputs", "inputs_gen.cu")],
}


def _headers(src_dir):
    return glob.glob(os.path.join(src_dir, "*.cuh")) + glob.glob(os.path.join(src_dir, "*.h")) + \
        glob.glob(os.path.join(ROOT, "include", "*.h"))


def _run(cmd, verbose):
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError(f"nvcc failed: {' '.join(cmd)}")
    if verbose and r.stderr:
        sys.stderr.write(r.stderr)


def build(verbose: bool = False, ptxas_info: bool = False) -> list:
    out_dir = os.path.join(ROOT, "_build")
    os.makedirs(out_dir, exist_ok=True)
    built = []
    for lib, sources in LIBS.items():
        objs = []
        for src in sources:
            obj = os.path.join(out_dir, os.path.basename(src) + ".o")
            deps = [src] + _headers(os.path.dirname(src))
            stale = not os.path.exists(obj) or any(os.path.getmtime(d) > os.path.getmtime(obj) for d in deps)
            if stale or ptxas_info:
                extra = ["-Xptxas", "-v"] if ptxas_info else []
                _run([NVCC, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj], verbose or ptxas_info)
            objs.append(obj)
        if not os.path.exists(lib) or any(os.path.getmtime(o) > os.path.getmtime(lib) for o in objs):
            _run([NVCC, *ARCH, "-shared", "-o", lib, *objs, "-lcudart"], verbose)
        built.append(lib)
    return built


if __name__ == "__main__":
    for lib in build(verbose="-v" in sys.argv, ptxas_info="--ptxas" in sys.argv):
        print(lib)
