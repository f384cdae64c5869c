"""w4a16_gemv_noalloc, the GEMV entry point for callers that cannot allocate device memory
(its scratch is a static array inside the library), against w4a16_gemv with a caller
workspace.  Collected last, so a run that stops at the first failure has run the rest."""
import ctypes

import numpy as np
import pytest
import torch

import w4a16_gemm_awq_b200 as w4
from parity import Case, check_close, host_bf16_as_f64, xs_abs

pytestmark = pytest.mark.gpu


def noalloc(L, x, qw, sc, z, csr, y, M, N, K):
    fn = L.w4a16_gemv_noalloc
    fn.argtypes = [ctypes.c_void_p] * 4 + [ctypes.POINTER(w4.Csr), ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                           ctypes.c_int64, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    cs = None
    if csr is not None:
        rp, ci, v = csr
        cs = w4.Csr(rp.data_ptr(), ci.data_ptr(), v.data_ptr(), int(ci.numel()))
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return fn(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(qw.data_ptr()), ctypes.c_void_p(sc.data_ptr()),
              ctypes.c_void_p(z.data_ptr()), ctypes.byref(cs) if cs is not None else None,
              ctypes.c_void_p(y.data_ptr()), M, N, K, stream)


@pytest.mark.parametrize("K,N,M,csr", [(4096, 4096, 1, False), (4096, 2048, 16, True), (16384, 640, 5, False)])
def test_gemv_noalloc_matches_gemv_twice(orc, K, N, M, csr):
    """Same launch plan as w4a16_gemv, so the same bits, on two calls in a row (the second
    reuses the scratch the first left behind); and within the GEMV's bound of the oracle."""
    L = w4.lib()
    c = Case(orc, seed=K + N + M, K=K, N=N, M=M, csr=csr)
    d = c.device()
    want = w4.w4a16_gemv(d["x"], d["qweight"], d["scales"], d["zeros"], csr=d["csr"])
    w4.check_device_status()
    for _ in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        code = noalloc(L, d["x"], d["qweight"], d["scales"], d["zeros"], d["csr"], y, M, N, K)
        assert code == w4.OK, w4.status_string(code)
        w4.check_device_status()
        assert torch.equal(y.view(torch.int16), want.view(torch.int16))
    r, ra = c.reference(orc)
    check_close(host_bf16_as_f64(y), r, ra, 0.0, K // 128 + 64, f"noalloc K={K} N={N} M={M}", xs_abs(c.x, c.sc))


def test_gemv_noalloc_python_wrapper(orc):
    """The binding's w4a16_gemv_noalloc gives the C entry point's bits."""
    c = Case(orc, seed=77, K=2048, N=512, M=3, csr=True)
    d = c.device()
    want = w4.w4a16_gemv(d["x"], d["qweight"], d["scales"], d["zeros"], csr=d["csr"])
    got = w4.w4a16_gemv_noalloc(d["x"], d["qweight"], d["scales"], d["zeros"], csr=d["csr"])
    w4.check_device_status()
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))
    with pytest.raises(ValueError):
        w4.w4a16_gemv_noalloc(d["x"], d["qweight"][:, :-1].contiguous(), d["scales"], d["zeros"])


def test_gemv_noalloc_rejects_oversize(orc):
    L = w4.lib()
    c = Case(orc, seed=3, K=1024, N=128, M=17)
    d = c.device()
    y = torch.empty(17, 128, dtype=torch.bfloat16, device="cuda")
    assert noalloc(L, d["x"], d["qweight"], d["scales"], d["zeros"], None, y, 17, 128, 1024) == w4.ERR_SHAPE
