"""The boundary is a plain C ABI: include/w4a16.h compiles as strict C99 and as C++, and a
C program that quantizes a layer and runs the linear through it compiles and links against
libw4a16.so.  Only the last test, marked gpu, runs the program."""
import os
import shutil
import subprocess

import pytest

import w4a16_gemm_awq_b200 as w4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w4a16.h")
EXAMPLE = os.path.join(ROOT, "tests", "c_abi", "quantize_and_linear.c")
OUT_DIR = os.path.join(ROOT, "tests", "c_abi", "_build")
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")

needs_gcc = pytest.mark.skipif(shutil.which("gcc") is None or shutil.which("g++") is None,
                               reason="no host C compiler")


def _run(cmd):
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, f"{' '.join(cmd)}\n{r.stdout}\n{r.stderr}"


@needs_gcc
def test_header_is_strict_c99():
    _run(["gcc", "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror", "-fsyntax-only", "-x", "c", HEADER])


@needs_gcc
def test_header_is_cxx():
    _run(["g++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-fsyntax-only", "-x", "c++", HEADER])


needs_cuda_headers = pytest.mark.skipif(not os.path.exists(os.path.join(CUDA, "include", "cuda_runtime.h")),
                                        reason="no CUDA toolkit headers")


def _build_example() -> str:
    w4.build()
    os.makedirs(OUT_DIR, exist_ok=True)
    lib_dir = os.path.dirname(w4.LIB_PATH)
    out = os.path.join(OUT_DIR, "quantize_and_linear")
    _run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
          "-I", os.path.join(CUDA, "include"), EXAMPLE, "-L", lib_dir, "-lw4a16",
          "-L", os.path.join(CUDA, "lib64"), "-lcudart", f"-Wl,-rpath,{lib_dir}",
          f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}", "-o", out])
    return out


@needs_gcc
@needs_cuda_headers
def test_c_example_compiles_and_links():
    assert os.path.exists(_build_example())


@pytest.mark.gpu
@needs_gcc
@needs_cuda_headers
def test_c_example_runs_on_the_gpu():
    """The C program quantizes, folds and runs the linear through the C ABI alone."""
    r = subprocess.run([_build_example()], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    lines = r.stdout.strip().splitlines()
    assert lines[-1] == "ok"
    vals = [float(v) for v in lines[0].split("=")[1].split()]
    assert len(vals) == 4 and all(abs(v) < 1e3 for v in vals) and any(v != 0.0 for v in vals)
