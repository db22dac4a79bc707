"""Build libgdn.so in-tree with nvcc for sm_100a (B200).

    python -m linear_attention_token_gdn_b200.build [--verbose]

The library is one translation unit (``csrc/gdn_lib.cu``) that includes every kernel;
the resulting ``libgdn.so`` sits next to this file and is what the ctypes binding
loads.  ``libgdn_debug.so`` is the same source compiled with ``-DGDN_BOUNDS_CHECK``: its
kernels test their computed global indices and flag an index outside its tensor in the
device error word instead of accessing it.  ``-Xptxas -v`` (register / shared-memory /
spill report) is printed with ``--verbose``.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
SO = os.path.join(HERE, "libgdn.so")
DEBUG_SO = os.path.join(HERE, "libgdn_debug.so")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2",
    "-shared",
    "--expt-relaxed-constexpr",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(INCLUDE, "*.h")))


def stale(so: str = SO) -> bool:
    if not os.path.exists(so):
        return True
    t = os.path.getmtime(so)
    return any(os.path.getmtime(s) > t for s in sources())


def _start(so: str, debug: bool, verbose: bool):
    tmp = so + f".tmp{os.getpid()}"
    cmd = [NVCC, *FLAGS, *(["-DGDN_BOUNDS_CHECK"] if debug else []), "-I", INCLUDE, "-o", tmp,
           os.path.join(CSRC, "gdn_lib.cu")]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    return so, tmp, cmd, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)


def _finish(job, verbose: bool) -> str:
    so, tmp, cmd, proc = job
    out, _ = proc.communicate()
    if verbose or proc.returncode != 0:
        sys.stderr.write(out)
    if proc.returncode != 0:
        raise RuntimeError(f"nvcc failed ({proc.returncode}): {' '.join(cmd)}")
    os.replace(tmp, so)
    return so


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """libgdn.so (debug=True: libgdn_debug.so, the bounds-checking build), rebuilt when a
    source is newer."""
    so = DEBUG_SO if debug else SO
    if not force and not stale(so):
        return so
    return _finish(_start(so, debug, verbose), verbose)


def build_all(force: bool = False, verbose: bool = False) -> None:
    """Both builds, compiled concurrently."""
    jobs = [_start(so, dbg, verbose) for so, dbg in ((SO, False), (DEBUG_SO, True)) if force or stale(so)]
    for job in jobs:
        _finish(job, verbose)


if __name__ == "__main__":
    build_all(force=True, verbose="--verbose" in sys.argv)
    print(SO)
    print(DEBUG_SO)
