"""Build the in-tree shared libraries with nvcc for sm_100a.

    python -m sparse_decode_attention_spkv_b200.build

produces ``libspkv.so`` (the SP-KV kernels behind the C ABI of include/spkv.h),
``libspkv_debug.so`` (the same kernels built with SPKV_DEBUG: device-side index checks)
and ``inputs/libspkv_inputs.so`` (the device side of the seeded input generator).
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
    # library: (sources, extra compiler flags, object directory)
    os.path.join(PKG, "libspkv.so"): (sorted(glob.glob(os.path.join(PKG, "csrc", "*.cu"))), [], ""),
    # the same kernels with device-side checks of page-table entries and positions
    # (SPKV_DEBUG: a failed check latches SPKV_FLAG_INDEX; nothing traps)
    os.path.join(PKG, "libspkv_debug.so"): (sorted(glob.glob(os.path.join(PKG, "csrc", "*.cu"))),
                                            ["-DSPKV_DEBUG"], "debug"),
    os.path.join(PKG, "inputs", "libspkv_inputs.so"): ([os.path.join(PKG, "inputs", "inputs_gen.cu")],
                                                      [], ""),
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
    from concurrent.futures import ThreadPoolExecutor
    built = []
    for lib, (sources, extra, sub) in LIBS.items():
        out_dir = os.path.join(ROOT, "_build", sub)
        os.makedirs(out_dir, exist_ok=True)
        jobs, objs = [], []
        for src in sources:
            obj = os.path.join(out_dir, os.path.basename(src) + ".o")
            deps = [src] + _headers(os.path.dirname(src))
            stale = not os.path.exists(obj) or any(os.path.getmtime(d) > os.path.getmtime(obj) for d in deps)
            if stale or ptxas_info:
                px = ["-Xptxas", "-v"] if ptxas_info else []
                jobs.append([NVCC, *ARCH, *FLAGS, *extra, *px, "-c", src, "-o", obj])
            objs.append(obj)
        with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
            list(ex.map(lambda c: _run(c, verbose or ptxas_info), jobs))
        if not os.path.exists(lib) or any(os.path.getmtime(o) > os.path.getmtime(lib) for o in objs):
            _run([NVCC, *ARCH, "-shared", "-o", lib, *objs, "-lcudart"], verbose)
        built.append(lib)
    return built


if __name__ == "__main__":
    for lib in build(verbose="-v" in sys.argv, ptxas_info="--ptxas" in sys.argv):
        print(lib)
