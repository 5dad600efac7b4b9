"""Build libpf.so (the packed-KV-cache C-ABI library) in-tree with nvcc.

Every CUDA source is compiled for sm_100a only; the CUDA runtime is linked
statically so the library loads on a machine without a GPU (calls then fail
with PF_ERR_CUDA).  Usage:  python -m packed_kv_cache_b200.build [--verbose]
"""
from __future__ import annotations

import contextlib
import fcntl
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libpf.so")
LOCK = os.path.join(HERE, ".build.lock")

SOURCES = ["pf_cache.cpp", "rope_shift.cu", "append_copy.cu", "select.cu", "attend.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return "nvcc"


def _compile(src: str, verbose: bool) -> str:
    obj = os.path.join(BUILD, os.path.splitext(src)[0] + ".o")
    cmd = [nvcc(), "-c", os.path.join(CSRC, src), "-o", obj, "-std=c++17", "-O3", "-lineinfo",
           "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC] + ARCH
    if src.endswith(".cu"):
        cmd += ["--expt-relaxed-constexpr"]
        if verbose:
            cmd += ["-Xptxas", "-v"]
    else:
        cmd += ["-x", "cu"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose and (r.stdout or r.stderr):
        print(f"--- {src}\n{r.stdout}{r.stderr}", file=sys.stderr)
    return obj


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, "pf.h"), __file__]
    return any(os.path.getmtime(d) > t for d in deps)


@contextlib.contextmanager
def _exclusive():
    """One build at a time across processes: the ranks of one job, or parallel
    test workers, may all find the library stale and would otherwise write the
    same object files at once."""
    with open(LOCK, "a") as f:
        fcntl.flock(f, fcntl.LOCK_EX)
        try:
            yield
        finally:
            fcntl.flock(f, fcntl.LOCK_UN)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile and link libpf.so if any source is newer than it; return its path."""
    if not force and not _stale():
        return LIB
    with _exclusive():
        if not force and not _stale():   # built by another process while this one waited
            return LIB
        os.makedirs(BUILD, exist_ok=True)
        with ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
            objs = list(ex.map(lambda s: _compile(s, verbose), SOURCES))
        tmp = f"{LIB}.{os.getpid()}.tmp"
        cmd = [nvcc(), "-shared", "-o", tmp] + objs + ARCH + ["-cudart", "static", "-Xcompiler", "-fPIC"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv))
