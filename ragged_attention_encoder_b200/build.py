"""Builds the C-ABI library ``librae.so`` in the package directory with nvcc (sm_100a).

It also links ``librae_test.so``, the test build: the same objects except the decode kernel,
which is compiled once more with ``RAE_TEST_HOOKS`` defined (the fault-injection entry point
of include/rae_test_hooks.h).  Only the failure-detection tests load it.

Objects go to ``ragged_attention_encoder_b200/_build/``; a source is recompiled only when it
or a header is newer than its object.  Usage: ``python -m ragged_attention_encoder_b200.build``.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "librae.so")
TEST_LIB = os.path.join(PKG, "librae_test.so")
HOOKED_SOURCE = "decode_simt.cu"     # the source compiled again with RAE_TEST_HOOKS

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _headers():
    return glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(nvcc, src, obj, deps, extra, verbose):
    if not _stale(obj, deps):
        return
    if src.endswith(".cu"):
        cmd = [nvcc, *ARCH, "-lineinfo", *COMMON, "-Xptxas", "-v", *extra, "-c", src, "-o", obj]
    else:
        cmd = [nvcc, *COMMON, *extra, "-x", "c++", "-c", src, "-o", obj]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"compile failed: {' '.join(cmd)}\n{res.stdout}\n{res.stderr}")
    with open(obj + ".log", "w") as f:
        f.write(res.stderr)
    if verbose:
        print(res.stderr, file=sys.stderr)


def _link(nvcc, lib, objs):
    if not _stale(lib, objs):
        return
    cmd = [nvcc, *ARCH, "-shared", "-o", lib + ".tmp", *objs, "-lcudart_static", "-lrt", "-ldl",
           "-lpthread"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"link failed: {' '.join(cmd)}\n{res.stdout}\n{res.stderr}")
    os.replace(lib + ".tmp", lib)


def build(verbose: bool = False, extra_flags=None) -> str:
    """Compiles every source under csrc/, links librae.so and librae_test.so; returns the
    path of librae.so."""
    os.makedirs(BUILD, exist_ok=True)
    nvcc = _nvcc()
    headers = _headers()
    extra = list(extra_flags or [])
    objs, test_objs = [], []
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))
    for src in sources:
        obj = os.path.join(BUILD, os.path.basename(src) + ".o")
        _compile(nvcc, src, obj, [src] + headers + [__file__], extra, verbose)
        objs.append(obj)
        if os.path.basename(src) == HOOKED_SOURCE:
            hobj = os.path.join(BUILD, os.path.basename(src) + ".hooks.o")
            _compile(nvcc, src, hobj, [src] + headers + [__file__], extra + ["-DRAE_TEST_HOOKS"],
                     verbose)
            test_objs.append(hobj)
        else:
            test_objs.append(obj)
    _link(nvcc, LIB, objs)
    _link(nvcc, TEST_LIB, test_objs)
    return LIB


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv))
