"""The C-ABI library loads on a machine without a GPU, exports every entry point that
include/w4a16.h declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

import w4a16_gemm_awq_b200 as w4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w4a16.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:w4a16_status|const char\s*\*|int|size_t)\s+(\w+)\s*\(", text, flags=re.M)


@pytest.fixture(scope="module")
def L():
    w4.build()
    return w4.lib()


def test_header_declares_the_boundary():
    names = set(declared_functions())
    assert {"awq_quantize_g128", "w4a16_linear", "w4a16_gemv", "w4a16_gemm", "w4a16_check_device_status",
            "w4a16_status_string", "w4a16_version", "w4a16_workspace_bytes"} <= names


def test_every_declared_symbol_is_exported(L):
    out = subprocess.run(["nm", "-D", "--defined-only", w4.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(L, name)


def test_workspace_query_without_gpu(L):
    # no device here: the query reports 0 rather than failing; invalid sizes report 0 too
    assert L.w4a16_workspace_bytes(1, 4096, 4096) == 0
    assert L.w4a16_workspace_bytes(17, 4096, 4096) == 0


def test_status_strings(L):
    for code in range(8):
        assert len(w4.status_string(code)) > 0
    assert w4.status_string(99) == "unknown status"
    assert w4.version() >= 100


FAKE = 1 << 20  # a 16-byte-aligned address that is never dereferenced: validation fails first


def _linear(L, name, x=FAKE, qw=FAKE, sc=FAKE, z=FAKE, csr=None, y=FAKE, M=1, N=128, K=1024, ws=FAKE, wsb=1 << 30):
    fn = getattr(L, name)
    return fn(ctypes.c_void_p(x), ctypes.c_void_p(qw), ctypes.c_void_p(sc), ctypes.c_void_p(z),
              ctypes.byref(csr) if csr is not None else None, ctypes.c_void_p(y), M, N, K,
              ctypes.c_void_p(ws), wsb, None)


@pytest.mark.parametrize("name", ["w4a16_linear", "w4a16_gemv", "w4a16_gemm"])
def test_linear_validation(L, name):
    assert _linear(L, name, x=0) == w4.ERR_NULL
    assert _linear(L, name, y=0) == w4.ERR_NULL
    assert _linear(L, name, K=1000) == w4.ERR_SHAPE
    assert _linear(L, name, N=100) == w4.ERR_SHAPE
    assert _linear(L, name, M=0) == w4.ERR_SHAPE
    assert _linear(L, name, x=FAKE + 2) == w4.ERR_ALIGN
    assert _linear(L, name, sc=FAKE + 8) == w4.ERR_ALIGN
    bad = w4.Csr(None, None, None, 5)
    assert _linear(L, name, csr=bad) == w4.ERR_NULL
    neg = w4.Csr(FAKE, FAKE, FAKE, -1)
    assert _linear(L, name, csr=neg) == w4.ERR_SHAPE
    odd = w4.Csr(FAKE + 2, FAKE, FAKE, 3)
    assert _linear(L, name, csr=odd) == w4.ERR_ALIGN


def test_gemv_rejects_large_m(L):
    assert _linear(L, "w4a16_gemv", M=17) == w4.ERR_SHAPE


def test_gemv_schedule_validation(L):
    def ex(schedule, **kw):
        a = dict(x=FAKE, qw=FAKE, sc=FAKE, z=FAKE, y=FAKE, M=1, N=128, K=1024, ws=FAKE, wsb=1 << 30)
        a.update(kw)
        return L.w4a16_gemv_ex(ctypes.c_void_p(a["x"]), ctypes.c_void_p(a["qw"]), ctypes.c_void_p(a["sc"]),
                               ctypes.c_void_p(a["z"]), None, ctypes.c_void_p(a["y"]), a["M"], a["N"], a["K"],
                               ctypes.c_void_p(a["ws"]), a["wsb"], schedule, None)
    assert ex(3) == w4.ERR_VALUE
    assert ex(-1) == w4.ERR_VALUE
    assert ex(w4.GEMV_CLUSTER, M=17) == w4.ERR_SHAPE
    assert ex(w4.GEMV_STREAM_K, x=0) == w4.ERR_NULL
    r = ctypes.c_int(-5)
    assert L.w4a16_gemv_plan(1, 100, 1024, 0, ctypes.byref(r), None, None) == w4.ERR_SHAPE
    assert L.w4a16_gemv_plan(17, 128, 1024, 0, None, None, None) == w4.ERR_SHAPE
    assert L.w4a16_gemv_plan(1, 128, 1024, 9, None, None, None) == w4.ERR_VALUE
    assert r.value == -5  # untouched on error


def test_quantize_validation(L):
    def q(W=FAKE, a=FAKE, alpha=0.5, N=128, K=1024, qw=FAKE, sc=FAKE, z=FAKE, s=None):
        return L.awq_quantize_g128(ctypes.c_void_p(W), ctypes.c_void_p(a), ctypes.c_float(alpha), N, K,
                                   ctypes.c_void_p(qw), ctypes.c_void_p(sc), ctypes.c_void_p(z),
                                   ctypes.c_void_p(s) if s else None, None)
    assert q(W=0) == w4.ERR_NULL
    assert q(z=0) == w4.ERR_NULL
    assert q(K=1536) == w4.ERR_SHAPE
    assert q(N=0) == w4.ERR_SHAPE
    assert q(W=FAKE + 4) == w4.ERR_ALIGN
    assert q(s=FAKE + 4) == w4.ERR_ALIGN
    assert q(alpha=float("nan")) == w4.ERR_VALUE
    assert q(alpha=float("inf")) == w4.ERR_VALUE


def test_grouped_validation(L):
    def q(gs, N=128, K=4096, W=FAKE):
        return L.awq_quantize(ctypes.c_void_p(W), ctypes.c_void_p(FAKE), ctypes.c_float(0.5), N, K, gs,
                              ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE), None, None)
    for gs in (0, 64, 100, 384, 1536, 3072, 8192, 65536):
        assert q(gs) == w4.ERR_SHAPE, gs
    assert q(256, W=0) == w4.ERR_NULL
    assert q(2048, K=5120) == w4.ERR_SHAPE            # 2048 does not divide 5120
    assert q(40960, K=40960) == w4.ERR_SHAPE          # above 32768

    def lx(gs, schedule=0, K=4096, M=1):
        return L.w4a16_linear_ex(ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE),
                                 ctypes.c_void_p(FAKE), None, ctypes.c_void_p(FAKE), M, 128, K, gs,
                                 ctypes.c_void_p(FAKE), 1 << 30, schedule, None)
    for gs in (0, 64, 192, 3072, 8192):
        assert lx(gs) == w4.ERR_SHAPE, gs
    assert lx(256, schedule=5) == w4.ERR_VALUE
    assert lx(2048, K=5120) == w4.ERR_SHAPE            # 2048 does not divide 5120


def test_folded_gemv_validation(L):
    def f(s=FAKE, M=1, gs=128, schedule=0, K=4096, x=FAKE):
        return L.w4a16_gemv_folded(ctypes.c_void_p(x), ctypes.c_void_p(s) if s else None, ctypes.c_void_p(FAKE),
                                   ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE), None, ctypes.c_void_p(FAKE), M,
                                   128, K, gs, ctypes.c_void_p(FAKE), 1 << 30, schedule, None)
    assert f(x=0) == w4.ERR_NULL
    assert f(M=17) == w4.ERR_SHAPE                     # decode only
    assert f(M=0) == w4.ERR_SHAPE
    assert f(gs=192) == w4.ERR_SHAPE
    assert f(gs=2048, K=5120) == w4.ERR_SHAPE
    assert f(schedule=4) == w4.ERR_VALUE
    assert f(s=FAKE + 4) == w4.ERR_ALIGN               # s is read 16 bytes at a time


def test_split_validation(L):
    def sp(W=FAKE, a=FAKE, alpha=0.5, N=16, K=256, nnz=10, Wd=FAKE, rp=FAKE, ci=FAKE, v=FAKE, ws=FAKE, wsb=1 << 30):
        return L.awq_split_outliers(ctypes.c_void_p(W), ctypes.c_void_p(a), ctypes.c_float(alpha), N, K, nnz,
                                    ctypes.c_void_p(Wd), ctypes.c_void_p(rp), ctypes.c_void_p(ci), ctypes.c_void_p(v),
                                    ctypes.c_void_p(ws), wsb, None)
    assert sp(W=0) == w4.ERR_NULL
    assert sp(rp=0) == w4.ERR_NULL
    assert sp(nnz=16 * 256 + 1) == w4.ERR_SHAPE
    assert sp(nnz=-1) == w4.ERR_SHAPE
    assert sp(N=0) == w4.ERR_SHAPE
    assert sp(N=1 << 16, K=1 << 16) == w4.ERR_SHAPE  # N * K must stay below 2^32
    assert sp(alpha=-0.5) == w4.ERR_VALUE
    assert sp(alpha=float("nan")) == w4.ERR_VALUE
    assert L.awq_split_outliers_workspace_bytes(0, 5) == 0
    assert L.awq_split_outliers_workspace_bytes(100, 5) >= 256 + 4096 * 4 + 3 * 400


def test_selftest_timeout_validation(L):
    assert L.w4a16_selftest_timeout(-1, None) == w4.ERR_VALUE
    assert L.w4a16_selftest_timeout(10 ** 11, None) == w4.ERR_VALUE


def test_binding_has_no_cpu_path():
    """The binding refuses CPU tensors instead of computing anything itself."""
    import torch
    x = torch.zeros(1, 1024, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        w4.w4a16_linear(x, torch.zeros(128, 128, dtype=torch.int32), torch.zeros(128, 8, dtype=torch.int16),
                        torch.zeros(128, 1, dtype=torch.int32))


def test_binding_has_every_entry_point_by_name():
    """The Python binding offers each C entry point under the same name."""
    for name in declared_functions():
        assert callable(getattr(w4, name, None)), name
    want = int(w4.lib().awq_split_outliers_workspace_bytes(256, 1024))
    assert w4.awq_split_outliers_workspace_bytes(256, 1024) == want
    assert w4.w4a16_version() == w4.version()
    assert w4.w4a16_status_string(w4.ERR_SHAPE) == w4.status_string(w4.ERR_SHAPE)


def test_linear_shape_checks_before_any_launch():
    """Mismatched operands are refused by the binding with ValueError (CPU tensors suffice:
    the shapes are checked before the device)."""
    M, N, K = 3, 256, 2048
    x = torch.zeros(M, K, dtype=torch.bfloat16)
    qw = torch.zeros(N, K // 8, dtype=torch.int32)
    sc = torch.zeros(K // 128, N, dtype=torch.int16)
    z = torch.zeros(K // 128, N // 8, dtype=torch.int32)
    w4.check_linear_shapes(x, qw, sc, z)
    bad = [
        (x, qw[:, :-1], sc, z, None, None),                    # qweight too short for K
        (x, qw, sc[:, :-8], z, None, None),                    # scales for fewer rows
        (x, qw, sc, z[:-1], None, None),                       # zeros for fewer groups
        (x, qw, sc, z, (torch.zeros(N, dtype=torch.int32), None, None), None),  # row_ptr of N entries
        (x, qw, sc, z, None, torch.zeros(M, N - 128, dtype=torch.bfloat16)),    # out of the wrong shape
    ]
    for args in bad:
        with pytest.raises(ValueError):
            w4.check_linear_shapes(*args)
    for fn in (w4.w4a16_gemv_noalloc, w4.w4a16_gemv):
        with pytest.raises(ValueError):
            fn(x, qw[:, :-1], sc, z)


def test_three_bit_validation(L):
    def q(gs=128, N=128, K=4096, W=FAKE, alpha=0.5):
        return L.awq_quantize3(ctypes.c_void_p(W), ctypes.c_void_p(FAKE), ctypes.c_float(alpha), N, K, gs,
                               ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE), None, None)
    assert q(W=0) == w4.ERR_NULL
    for gs in (64, 192, 2048, 4096):          # the 3-bit quantizer takes 128 .. 1024
        assert q(gs) == w4.ERR_SHAPE, gs
    assert q(K=1000) == w4.ERR_SHAPE
    assert q(alpha=float("nan")) == w4.ERR_VALUE

    def g3(M=1, gs=128, schedule=0, x=FAKE, K=4096):
        return L.w3a16_gemv(ctypes.c_void_p(x), ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE),
                            None, ctypes.c_void_p(FAKE), M, 128, K, gs, ctypes.c_void_p(FAKE), 1 << 30, schedule,
                            None)
    assert g3(x=0) == w4.ERR_NULL
    assert g3(M=17) == w4.ERR_SHAPE           # decode only: no 3-bit prefill GEMM
    assert g3(gs=192) == w4.ERR_SHAPE
    assert g3(schedule=7) == w4.ERR_VALUE


def test_nvfp4_validation(L):
    def q(W=FAKE, N=128, K=4096, g=FAKE, s=FAKE, alpha=0.5):
        return L.awq_quantize_nvfp4(ctypes.c_void_p(W), ctypes.c_void_p(FAKE), ctypes.c_float(alpha), N, K,
                                    ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE), ctypes.c_void_p(g),
                                    ctypes.c_void_p(s) if s else None, None)
    assert q(W=0) == w4.ERR_NULL
    assert q(s=0) == w4.ERR_NULL              # s_out is required: the kernels read it back
    assert q(N=12) == w4.ERR_SHAPE
    assert q(K=40) == w4.ERR_SHAPE
    assert q(g=FAKE + 2) == w4.ERR_ALIGN
    assert q(alpha=float("inf")) == w4.ERR_VALUE

    def gv(M=1, N=128, K=4096, x=FAKE, g=FAKE):
        return L.w4a16_gemv_nvfp4(ctypes.c_void_p(x), ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE),
                                  ctypes.c_void_p(g), ctypes.c_void_p(FAKE), M, N, K, None)
    assert gv(x=0) == w4.ERR_NULL
    assert gv(M=17) == w4.ERR_SHAPE
    assert gv(N=24) == w4.ERR_SHAPE
    assert gv(K=24) == w4.ERR_SHAPE
    assert gv(x=FAKE + 4) == w4.ERR_ALIGN


def test_variant_wrappers_check_shapes_first():
    import torch
    x = torch.zeros(2, 1024, dtype=torch.bfloat16)
    with pytest.raises(ValueError):           # a 4-bit qweight handed to the 3-bit GEMV
        w4.w3a16_gemv(x, torch.zeros(128, 128, dtype=torch.int32), torch.zeros(8, 128, dtype=torch.int16),
                      torch.zeros(8, 16, dtype=torch.int32))
    with pytest.raises(ValueError):           # CPU tensors never reach the library
        w4.w4a16_gemv_nvfp4(x, torch.zeros(128, 128, dtype=torch.int32), torch.zeros(64, 128, dtype=torch.uint8),
                            torch.ones(1))
