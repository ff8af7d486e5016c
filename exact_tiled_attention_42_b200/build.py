"""Compile the CUDA sources under csrc/ into the in-tree shared library.

    python -m exact_tiled_attention_42_b200.build [-v] [--force]

Every translation unit is compiled for sm_100a only
(``-gencode arch=compute_100a,code=sm_100a``) and linked into
``libfa_b200.so`` next to this file, with the CUDA runtime linked statically,
and the same sources again into ``libfa_b200_debug.so`` for the test of the
abort path (a 1 ms bound on every wait and a switch that withholds one copy).
Objects go to ``_build/`` at the repository root; a unit is rebuilt when it or
any header under csrc/ or include/ is newer than its object.
"""

from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libfa_b200.so")
# Debug variant for the abort-path and bounds tests: every bounded wait gives
# up after 1 ms, fa_debug_withhold_first_v() can keep the forward's first V
# tile from being loaded, and every computed global index is checked against
# its buffer (FA_ERR_BOUNDS). Never loaded by the product path.
DEBUG_LIB = os.path.join(PKG, "libfa_b200_debug.so")
DEBUG_FLAGS = ["-DFA_WAIT_TIMEOUT_NS=1000000ull", "-DFA_DEBUG_WITHHOLD", "-DFA_DEBUG_BOUNDS"]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-I" + INCLUDE, "-I" + CSRC]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def _compile(src: str, obj: str, verbose: bool, extra=()) -> str:
    cmd = [_nvcc(), *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {os.path.basename(src)}:\n{r.stdout}\n{r.stderr}")
    return r.stdout + r.stderr


def _build_variant(lib: str, objdir: str, extra: list, verbose: bool, force: bool) -> str:
    os.makedirs(objdir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    hdr_mtime = max((os.path.getmtime(h) for h in _headers()), default=0.0)
    jobs = []
    objs = []
    for s in srcs:
        o = os.path.join(objdir, os.path.basename(s)[:-3] + ".o")
        objs.append(o)
        if force or not os.path.exists(o) or os.path.getmtime(o) < max(os.path.getmtime(s), hdr_mtime):
            jobs.append((s, o))
    with cf.ThreadPoolExecutor(max_workers=min(8, max(1, len(jobs)))) as ex:
        for (s, _), log in zip(jobs, ex.map(lambda so: _compile(so[0], so[1], verbose, extra), jobs)):
            if verbose and log.strip():
                print(f"--- {os.path.basename(s)}\n{log}", file=sys.stderr)
    newest = max(os.path.getmtime(o) for o in objs)
    if force or jobs or not os.path.exists(lib) or os.path.getmtime(lib) < newest:
        cmd = [_nvcc(), *ARCH, "-shared", "-o", lib, *objs]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    return lib


def build(verbose: bool = False, force: bool = False) -> str:
    """Build the release library and the debug library (the latter only for
    the test that makes a bounded wait run out: 1 ms wait bound and a switch
    that withholds one copy). Returns the release library's path."""
    _build_variant(LIB, BUILD, [], verbose, force)
    _build_variant(DEBUG_LIB, os.path.join(BUILD, "debug"), DEBUG_FLAGS, verbose, force)
    return LIB


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--force", action="store_true")
    a = ap.parse_args()
    print(build(a.verbose, a.force))


if __name__ == "__main__":
    main()
