"""The boundary is a plain C ABI: include/w4a16.h compiles as strict C99 and as C++, and a
C program that quantizes a layer and runs the linear through it compiles and links against
libw4a16.so.  Only the last test, marked gpu, runs the program."""
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

import oracle
import w4a16_gemm_awq_b200 as w4
from parity import check_close, host_bf16_as_f64, xs_abs

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
def test_c_example_runs_on_the_gpu(tmp_path):
    """The C program quantizes, folds and runs the linear through the C ABI alone; its output
    matches the oracle's quantize, fold and product of the inputs it wrote out, within the
    decode GEMV's bound."""
    r = subprocess.run([_build_example(), str(tmp_path)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip().splitlines()[-1] == "ok"
    N, K, M = 4096, 1024, 4
    W = np.fromfile(tmp_path / "W.f32", np.float32).reshape(N, K)
    act = np.fromfile(tmp_path / "act.f32", np.float32)
    x = np.fromfile(tmp_path / "x.bf16", np.uint16).reshape(M, K)
    y = np.fromfile(tmp_path / "y.bf16", np.uint16).reshape(M, N)
    oracle.build()
    qw, sc, z, s = oracle.awq_quantize_g128(W, act, 0.5)
    xf = (x.astype(np.uint32) << 16).view(np.float32) / s[None, :].astype(np.float32)  # IEEE fp32 division
    xp = np.vectorize(oracle.f32_to_bf16_bits, otypes=[np.uint16])(xf)
    ref, ref_abs = oracle.linear(xp, qw, sc, z, N, with_abs=True)
    yt = torch.from_numpy(y.view(np.int16)).view(torch.bfloat16)
    check_close(host_bf16_as_f64(yt), ref, ref_abs, 0.0, K // 128 + 64, "C program", xs_abs(xp, sc))
