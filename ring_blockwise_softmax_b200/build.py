"""Build the in-tree C-ABI library ``libra_attn.so`` for sm_100a with nvcc.

    python -m ring_blockwise_softmax_b200.build [--force] [--verbose]

Each translation unit is compiled in parallel into ``_build/`` (the tensor-core kernel once per
padded head dim, and so are the tensor-core backward kernels), then linked with the static CUDA runtime into a shared library next to this
file.  Units are rebuilt only when a source or header is newer than their object.  The ptxas
resource report (registers, spills, shared memory) of the last build is kept in
``_build/ptxas.log``.
"""

from __future__ import annotations

import argparse
import concurrent.futures
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libra_attn.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ARCH + ["-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-Xptxas", "-v",
                "-I" + INCLUDE, "-I" + CSRC]

UNITS = [
    ("ra_attn.cu", "ra_attn.o", []),
    ("ra_noalloc.cu", "ra_noalloc.o", []),
    ("ra_fmha_launch.cu", "fmha_dp32.o", ["-DRA_FMHA_DP=32"]),
    ("ra_fmha_launch.cu", "fmha_dp64.o", ["-DRA_FMHA_DP=64"]),
    ("ra_fmha_launch.cu", "fmha_dp128.o", ["-DRA_FMHA_DP=128"]),
    ("ra_bwd_launch.cu", "bwd_dp32.o", ["-DRA_BWD_DP=32"]),
    ("ra_bwd_launch.cu", "bwd_dp64.o", ["-DRA_BWD_DP=64"]),
    ("ra_bwd_launch.cu", "bwd_dp128.o", ["-DRA_BWD_DP=128"]),
]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources_mtime() -> float:
    files = glob.glob(os.path.join(CSRC, "*")) + glob.glob(os.path.join(INCLUDE, "*.h")) + [__file__]
    return max(os.path.getmtime(f) for f in files)


def _compile(unit, verbose):
    src, obj, extra = unit
    out = os.path.join(BUILD, obj)
    cmd = [_nvcc(), *FLAGS, *extra, "-c", os.path.join(CSRC, src), "-o", out]
    if verbose:
        print(" ".join(cmd), flush=True)
    p = subprocess.run(cmd, capture_output=True, text=True)
    if p.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src} {extra}:\n{p.stdout}\n{p.stderr}")
    return obj, p.stderr


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile (if stale) and link the library; returns the path of the .so."""
    newest = _sources_mtime()
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= newest:
        return LIB
    os.makedirs(BUILD, exist_ok=True)
    stale = [u for u in UNITS
             if force or not os.path.exists(os.path.join(BUILD, u[1]))
             or os.path.getmtime(os.path.join(BUILD, u[1])) < newest]
    logs = []
    if stale:
        with concurrent.futures.ThreadPoolExecutor(max_workers=len(stale)) as ex:
            for obj, log in ex.map(lambda u: _compile(u, verbose), stale):
                logs.append(f"== {obj}\n{log}")
        with open(os.path.join(BUILD, "ptxas.log"), "w") as f:
            f.write("\n".join(logs))
    objs = [os.path.join(BUILD, u[1]) for u in UNITS]
    if force or stale or not os.path.exists(LIB) or os.path.getmtime(LIB) < max(map(os.path.getmtime, objs)):
        cmd = [_nvcc(), *ARCH, "-shared", "-o", LIB, *objs]
        if verbose:
            print(" ".join(cmd), flush=True)
        p = subprocess.run(cmd, capture_output=True, text=True)
        if p.returncode != 0:
            raise RuntimeError(f"link failed:\n{p.stdout}\n{p.stderr}")
    return LIB


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args(argv)
    print(build(force=a.force, verbose=a.verbose))
    return 0


if __name__ == "__main__":
    sys.exit(main())
