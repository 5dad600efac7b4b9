"""The library's host-side validation under the undefined-behaviour sanitizer:
tests/host_fuzz.c drives pf_cache_bytes, pf_cache_create and
pf_select_mid_static with random sizes around the limits and the int extremes.
The host code (pf_cache.cpp, and select.cu's host part) is compiled with
-fsanitize=undefined, so any signed overflow in the checks fails the run.
CPU only: the calls that pass validation end at their first CUDA call, which
fails without a GPU.  With a GPU visible they would reach the device with
placeholder addresses, so the test (and the program itself) refuses to run."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "packed_kv_cache_b200")
CSRC = os.path.join(PKG, "csrc")
INC = ["-I", os.path.join(ROOT, "include"), "-I", CSRC]
UBSAN = ["-fsanitize=undefined", "-fno-sanitize-recover=all"]


def _run(cmd):
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, f"{' '.join(cmd)}\n{r.stdout}\n{r.stderr}"
    return r.stdout


@pytest.mark.skipif(not (shutil.which("gcc") and shutil.which("g++")), reason="needs gcc and g++")
def test_host_validation_has_no_undefined_behaviour(tmp_path):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is visible: the fuzzer's placeholder addresses must not reach it")
    from packed_kv_cache_b200 import build
    nvcc = build.nvcc()
    cuda_inc = os.path.join(os.path.dirname(os.path.dirname(os.path.realpath(nvcc))), "include")
    cuda_lib = os.path.join(os.path.dirname(os.path.dirname(os.path.realpath(nvcc))), "lib64")
    out = str(tmp_path)
    objs = []
    # host code under the sanitizer
    objs.append(os.path.join(out, "pf_cache.o"))
    _run(["g++", "-std=c++17", "-O1", "-g", "-fPIC", *UBSAN, "-c", os.path.join(CSRC, "pf_cache.cpp"),
          "-o", objs[-1], *INC, "-I", cuda_inc])
    objs.append(os.path.join(out, "select.o"))
    _run([nvcc, "-c", os.path.join(CSRC, "select.cu"), "-o", objs[-1], "-std=c++17", "-O1",
          "-Xcompiler", ",".join(["-fPIC", *UBSAN]), *INC, *build.ARCH])
    # the other kernels as built (only their launch wrappers are linked in)
    for src in ("rope_shift.cu", "append_copy.cu", "attend.cu"):
        objs.append(os.path.join(out, src.replace(".cu", ".o")))
        _run([nvcc, "-c", os.path.join(CSRC, src), "-o", objs[-1], "-std=c++17", "-O1",
              "-Xcompiler", "-fPIC", *INC, *build.ARCH])
    objs.append(os.path.join(out, "host_fuzz.o"))
    _run(["gcc", "-O1", "-g", *UBSAN, "-c", os.path.join(ROOT, "tests", "host_fuzz.c"), "-o", objs[-1], *INC,
          "-I", cuda_inc])
    exe = os.path.join(out, "host_fuzz")
    _run(["g++", *UBSAN, *objs, "-L", cuda_lib, "-lcudart_static", "-ldl", "-lpthread", "-lrt", "-o", exe])
    text = _run([exe, "200000"])
    if text.startswith("skipped"):
        pytest.skip(text.strip())
    assert "configs:" in text and "static selection:" in text, text
