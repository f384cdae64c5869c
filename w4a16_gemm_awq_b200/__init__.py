"""Python binding of libw4a16.so (the B200 W4A16 quantized-linear library).

Argument marshalling only: every step of the computation runs in the library's CUDA
kernels.  PyTorch provides device memory and the current stream.  The entry points
mirror the C ABI in include/w4a16.h:

  awq_quantize_g128(W, act_absmean, alpha)      -> (qweight, scales, zeros, s)
  awq_quantize(W, act_absmean, alpha, gs)       -> the same with groups of gs along K (gs = K: per row)
  awq_quantize3(W, act_absmean, alpha, gs=128)  -> the same with 3-bit codes (qweight3 [N][3K/32])
  awq_quantize_nvfp4(W, act_absmean, alpha)     -> (qweight, scales8, g, s): NVFP4 weights
  w4a16_gemv_nvfp4(x, qweight, scales8, g)      -> y      (1 <= M <= 16, NVFP4 weights)
  w3a16_gemv(x, qweight3, scales, zeros, csr)   -> y      (1 <= M <= 16, 3-bit codes)
  w4a16_linear(x, qweight, scales, zeros, csr)  -> y      (any M)
  w4a16_gemv(...)                               -> y      (1 <= M <= 16)
  w4a16_gemv_ex(..., schedule)                  -> y      (GEMV_AUTO, GEMV_STREAM_K or GEMV_CLUSTER)
  w4a16_linear_ex(..., group_size, schedule)    -> y      (weights from awq_quantize with that group size)
  gemv_plan(M, N, K, schedule)                  -> (schedule, cluster size, CTAs) the call would launch
  w4a16_gemm(...)                               -> y      (tcgen05 path, any M)
  workspace_bytes(M, N, K, csr=True)            -> bytes of zeroed device workspace a call needs
  check_device_status()                         -> raises W4A16Error on a recorded problem

Bit containers: qweight [N][K/8] and zeros [K/128][N/8] are int32 tensors holding uint32
words, scales [K/128][N] is an int16 tensor holding fp16 bits, x and y are bfloat16 tensors.  A CSR is a tuple
(row_ptr int32 [N+1], col_idx int32 [nnz], values int16 fp16-bits [nnz]) of CUDA tensors.

There is no fallback: if the library is not built, or there is no sm_100 GPU, the calls
raise.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libw4a16.so")

STATUS = {0: "W4A16_OK", 1: "W4A16_ERR_NULL", 2: "W4A16_ERR_SHAPE", 3: "W4A16_ERR_ALIGN",
          4: "W4A16_ERR_VALUE", 5: "W4A16_ERR_CUDA", 6: "W4A16_ERR_TIMEOUT", 7: "W4A16_ERR_UNSUPPORTED"}
OK, ERR_NULL, ERR_SHAPE, ERR_ALIGN, ERR_VALUE, ERR_CUDA, ERR_TIMEOUT, ERR_UNSUPPORTED = range(8)
GEMV_AUTO, GEMV_STREAM_K, GEMV_CLUSTER = range(3)


class W4A16Error(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {STATUS.get(code, code)}")
        self.code = code


class Csr(ctypes.Structure):
    _fields_ = [("row_ptr", ctypes.c_void_p), ("col_idx", ctypes.c_void_p), ("values", ctypes.c_void_p),
                ("nnz", ctypes.c_int64)]


_lib = None


def build(force: bool = False) -> str:
    from . import buildlib
    return buildlib.build(force=force)


def lib() -> ctypes.CDLL:
    """Load libw4a16.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with w4a16_gemm_awq_b200.build()")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float
        L.awq_quantize_g128.argtypes = [P, P, F, I64, I64, P, P, P, P, P]
        L.awq_quantize.argtypes = [P, P, F, I64, I64, I64, P, P, P, P, P]
        L.awq_quantize3.argtypes = [P, P, F, I64, I64, I64, P, P, P, P, P]
        L.awq_quantize_nvfp4.argtypes = [P, P, F, I64, I64, P, P, P, P, P]
        L.w4a16_gemv_nvfp4.argtypes = [P, P, P, P, P, I64, I64, I64, P]
        L.w3a16_gemv.argtypes = [P, P, P, P, ctypes.POINTER(Csr), P, I64, I64, I64, I64, P, ctypes.c_size_t,
                                 ctypes.c_int, P]
        L.w4a16_linear_ex.argtypes = [P, P, P, P, ctypes.POINTER(Csr), P, I64, I64, I64, I64, P, ctypes.c_size_t,
                                      ctypes.c_int, P]
        for name in ("w4a16_linear", "w4a16_gemv", "w4a16_gemm"):
            fn = getattr(L, name)
            fn.argtypes = [P, P, P, P, ctypes.POINTER(Csr), P, I64, I64, I64, P, ctypes.c_size_t, P]
        L.w4a16_gemv_ex.argtypes = [P, P, P, P, ctypes.POINTER(Csr), P, I64, I64, I64, P, ctypes.c_size_t,
                                    ctypes.c_int, P]
        L.w4a16_gemv_folded.argtypes = [P, P, P, P, P, ctypes.POINTER(Csr), P, I64, I64, I64, I64, P,
                                        ctypes.c_size_t, ctypes.c_int, P]
        L.w4a16_gemv_noalloc.argtypes = [P, P, P, P, ctypes.POINTER(Csr), P, I64, I64, I64, P]
        PI = ctypes.POINTER(ctypes.c_int)
        L.w4a16_gemv_plan.argtypes = [I64, I64, I64, ctypes.c_int, PI, PI, PI]
        L.w4a16_gemm_plan.argtypes = [I64, I64, I64, ctypes.c_int, PI, PI, PI, ctypes.POINTER(ctypes.c_size_t)]
        L.w4a16_workspace_bytes.argtypes = [I64, I64, I64]
        L.w4a16_workspace_bytes.restype = ctypes.c_size_t
        L.w4a16_workspace_bytes_ex.argtypes = [I64, I64, I64, ctypes.c_int]
        L.w4a16_workspace_bytes_ex.restype = ctypes.c_size_t
        L.w4a16_check_device_status.argtypes = [P]
        L.w4a16_selftest_timeout.argtypes = [I64, P]
        L.w4a16_selftest_quotient.argtypes = [ctypes.POINTER(ctypes.c_uint64), ctypes.POINTER(ctypes.c_uint32), P]
        L.awq_split_outliers.argtypes = [P, P, F, I64, I64, I64, P, P, P, P, P, ctypes.c_size_t, P]
        L.awq_split_outliers_workspace_bytes.argtypes = [I64, I64]
        L.awq_split_outliers_workspace_bytes.restype = ctypes.c_size_t
        L.awq_search_alpha.argtypes = [P, P, P, I64, I64, I64, P, ctypes.c_int, P, P, P, ctypes.c_size_t, P]
        L.awq_search_alpha_workspace_bytes.argtypes = [I64, I64, I64, ctypes.c_int]
        L.awq_search_alpha_workspace_bytes.restype = ctypes.c_size_t
        L.awq_fold_activations.argtypes = [P, P, P, I64, I64, P]
        L.w4a16_status_string.argtypes = [ctypes.c_int]
        L.w4a16_status_string.restype = ctypes.c_char_p
        L.w4a16_version.argtypes = []
        for name in ("awq_quantize_g128", "awq_quantize", "w4a16_linear_ex", "w4a16_linear", "w4a16_gemv", "w4a16_gemv_ex", "w4a16_gemv_plan",
                     "w4a16_gemm", "w4a16_check_device_status",
                     "w4a16_selftest_timeout", "w4a16_selftest_quotient", "awq_split_outliers", "awq_search_alpha", "awq_fold_activations", "w4a16_version"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _stream(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _check(code: int, what: str):
    if code != OK:
        raise W4A16Error(code, what)


def _need(t, dtype, ndim, name):
    if not (t.is_cuda and t.dtype == dtype and t.dim() == ndim and t.is_contiguous()):
        raise ValueError(f"{name}: expected a contiguous CUDA {dtype} tensor of rank {ndim}, got "
                         f"{t.dtype} {tuple(t.shape)} on {t.device}")


def check_linear_shapes(x, qweight, scales, zeros, csr=None, out=None, group_size: int = 128, bits: int = 4):
    """Raise ValueError unless the operands of a linear call agree: x [M][K], qweight [N][K/8]
    ([N][3K/32] for 3-bit codes), scales [K/gs][N], zeros [K/gs][N/8], csr row_ptr [N+1], out
    [M][N] bf16.  Shapes only, so a mismatch is reported before anything reaches the library."""
    if x.dim() != 2 or qweight.dim() != 2:
        raise ValueError("x and qweight must be matrices")
    M, K = x.shape
    N = qweight.shape[0]
    gs = int(group_size)
    if (qweight.shape[1] * 8 != K) if bits == 4 else (qweight.shape[1] * 32 != 3 * K):
        raise ValueError(f"qweight {tuple(qweight.shape)} does not match K = {K} ({bits}-bit codes)")
    if gs < 1 or K % gs != 0:
        raise ValueError(f"group size {gs} does not divide K = {K}")
    if tuple(scales.shape) != (K // gs, N):
        raise ValueError(f"scales {tuple(scales.shape)}: expected ({K // gs}, {N})")
    if tuple(zeros.shape) != (K // gs, N // 8):
        raise ValueError(f"zeros {tuple(zeros.shape)}: expected ({K // gs}, {N // 8})")
    if csr is not None and csr[0].numel() != N + 1:
        raise ValueError(f"CSR row_ptr has {csr[0].numel()} entries, expected N + 1 = {N + 1}")
    if out is not None:
        if tuple(out.shape) != (M, N) or out.dtype != torch.bfloat16 or not out.is_contiguous():
            raise ValueError(f"out: expected a contiguous bf16 ({M}, {N}) tensor, got {out.dtype} {tuple(out.shape)}")
        if out.device != x.device:
            raise ValueError("out is on another device than x")


def awq_quantize(W: torch.Tensor, act_absmean: torch.Tensor, alpha: float, group_size: int, out=None):
    """awq_quantize_g128 with groups of group_size along K -> (qweight int32 [N][K/8],
    scales int16 [K/gs][N], zeros int32 [K/gs][N/8], s fp32 [K])."""
    _need(W, torch.float32, 2, "W")
    _need(act_absmean, torch.float32, 1, "act_absmean")
    N, K = W.shape
    dev = W.device
    G = max(K // max(group_size, 1), 1)
    if out is None:
        out = (torch.empty(N, K // 8, dtype=torch.int32, device=dev),
               torch.empty(G, N, dtype=torch.int16, device=dev),
               torch.empty(G, max(N // 8, 1), dtype=torch.int32, device=dev),
               torch.empty(K, dtype=torch.float32, device=dev))
    qw, sc, z, s = out
    code = lib().awq_quantize(_ptr(W), _ptr(act_absmean), ctypes.c_float(alpha), N, K, int(group_size), _ptr(qw),
                              _ptr(sc), _ptr(z), _ptr(s), _stream(dev))
    _check(code, "awq_quantize")
    return qw, sc, z, s


def awq_quantize3(W: torch.Tensor, act_absmean: torch.Tensor, alpha: float, group_size: int = 128, out=None):
    """awq_quantize with 3-bit codes -> (qweight3 int32 [N][3K/32], scales int16 [K/gs][N],
    zeros int32 [K/gs][N/8] (values 0..7), s fp32 [K])."""
    _need(W, torch.float32, 2, "W")
    _need(act_absmean, torch.float32, 1, "act_absmean")
    N, K = W.shape
    dev = W.device
    G = max(K // max(group_size, 1), 1)
    if out is None:
        out = (torch.empty(N, max(3 * K // 32, 1), dtype=torch.int32, device=dev),
               torch.empty(G, N, dtype=torch.int16, device=dev),
               torch.empty(G, max(N // 8, 1), dtype=torch.int32, device=dev),
               torch.empty(K, dtype=torch.float32, device=dev))
    qw, sc, z, s = out
    code = lib().awq_quantize3(_ptr(W), _ptr(act_absmean), ctypes.c_float(alpha), N, K, int(group_size), _ptr(qw),
                               _ptr(sc), _ptr(z), _ptr(s), _stream(dev))
    _check(code, "awq_quantize3")
    return qw, sc, z, s


def awq_quantize_nvfp4(W: torch.Tensor, act_absmean: torch.Tensor, alpha: float, out=None):
    """AWQ scaling then NVFP4 -> (qweight int32 [N][K/8] (E2M1 codes), scales8 uint8 [K/16][N]
    (E4M3), g fp32 [1] (tensor scale), s fp32 [K])."""
    _need(W, torch.float32, 2, "W")
    _need(act_absmean, torch.float32, 1, "act_absmean")
    N, K = W.shape
    dev = W.device
    if out is None:
        out = (torch.empty(N, max(K // 8, 1), dtype=torch.int32, device=dev),
               torch.empty(max(K // 16, 1), N, dtype=torch.uint8, device=dev),
               torch.empty(1, dtype=torch.float32, device=dev),
               torch.empty(K, dtype=torch.float32, device=dev))
    qw, sc, g, s = out
    code = lib().awq_quantize_nvfp4(_ptr(W), _ptr(act_absmean), ctypes.c_float(alpha), N, K, _ptr(qw), _ptr(sc),
                                    _ptr(g), _ptr(s), _stream(dev))
    _check(code, "awq_quantize_nvfp4")
    return qw, sc, g, s


def w4a16_gemv_nvfp4(x, qweight, scales8, gscale, out=None):
    """Decode GEMV (M <= 16) on NVFP4 weights from awq_quantize_nvfp4 -> y bf16 [M][N]."""
    _need(x, torch.bfloat16, 2, "x")
    _need(qweight, torch.int32, 2, "qweight")
    M, K = x.shape
    N = qweight.shape[0]
    if qweight.shape[1] * 8 != K or tuple(scales8.shape) != (K // 16, N) or scales8.dtype != torch.uint8:
        raise ValueError(f"NVFP4 operands do not match x [{M}][{K}]: qweight {tuple(qweight.shape)}, "
                         f"scales8 {tuple(scales8.shape)} {scales8.dtype}")
    if gscale.numel() != 1 or gscale.dtype != torch.float32 or gscale.device != x.device:
        raise ValueError("gscale: one fp32 value on the device of x")
    y = out if out is not None else torch.empty(M, N, dtype=torch.bfloat16, device=x.device)
    code = lib().w4a16_gemv_nvfp4(_ptr(x), _ptr(qweight), _ptr(scales8), _ptr(gscale), _ptr(y), M, N, K,
                                  _stream(x.device))
    _check(code, "w4a16_gemv_nvfp4")
    return y


def awq_quantize_g128(W: torch.Tensor, act_absmean: torch.Tensor, alpha: float, out=None):
    """W fp32 [N][K], act_absmean fp32 [K] -> (qweight int32 [N][K/8], scales int16 [K/128][N],
    zeros int32 [K/128][N/8], s fp32 [K])."""
    _need(W, torch.float32, 2, "W")
    _need(act_absmean, torch.float32, 1, "act_absmean")
    N, K = W.shape
    dev = W.device
    if out is None:
        out = (torch.empty(N, K // 8, dtype=torch.int32, device=dev),
               torch.empty(max(K // 128, 1), N, dtype=torch.int16, device=dev),
               torch.empty(max(K // 128, 1), max(N // 8, 1), dtype=torch.int32, device=dev),
               torch.empty(K, dtype=torch.float32, device=dev))
    qw, sc, z, s = out
    code = lib().awq_quantize_g128(_ptr(W), _ptr(act_absmean), ctypes.c_float(alpha), N, K, _ptr(qw), _ptr(sc),
                                   _ptr(z), _ptr(s), _stream(dev))
    _check(code, "awq_quantize_g128")
    return qw, sc, z, s


_workspaces = {}


def workspace(device: torch.device, nbytes: int, stream=None) -> torch.Tensor:
    """A zero-filled device workspace of at least nbytes for calls on `stream` of `device`,
    cached so that consecutive calls on the same stream reuse it (each call leaves it zeroed).
    Calls on different streams get different workspaces."""
    dev = torch.device(device)
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    key = (dev.index if dev.index is not None else torch.cuda.current_device(), s.cuda_stream)
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=dev)
        _workspaces[key] = ws
    return ws


def workspace_bytes(M: int, N: int, K: int, csr: bool = True) -> int:
    """Bytes of workspace a call with these sizes needs (csr: whether it passes a CSR term)."""
    return int(lib().w4a16_workspace_bytes_ex(M, N, K, 1 if csr else 0))


def _linear(name: str, x, qweight, scales, zeros, csr=None, out=None, ws=None, schedule=None, group_size=None,
            fold=False, s=None, bits=4):
    check_linear_shapes(x, qweight, scales, zeros, csr, out, 128 if group_size is None else group_size, bits)
    _need(x, torch.bfloat16, 2, "x")
    if s is not None:
        _need(s, torch.float32, 1, "s")
    _need(qweight, torch.int32, 2, "qweight")
    _need(scales, torch.int16, 2, "scales")
    _need(zeros, torch.int32, 2, "zeros")
    M, K = x.shape
    N = qweight.shape[0]
    if s is not None and s.numel() != K:
        raise ValueError(f"s has {s.numel()} entries, K = {K}")
    y = out if out is not None else torch.empty(M, N, dtype=torch.bfloat16, device=x.device)
    cs = None
    if csr is not None:
        rp, ci, v = csr
        _need(rp, torch.int32, 1, "row_ptr")
        cs = Csr(rp.data_ptr(), ci.data_ptr() if ci.numel() else None, v.data_ptr() if v.numel() else None,
                 int(ci.numel()))
    need = workspace_bytes(M, N, K, csr is not None)
    if ws is None and need > 0:
        ws = workspace(x.device, need)
    args = [_ptr(x)] + ([_ptr(s)] if fold else []) + [
        _ptr(qweight), _ptr(scales), _ptr(zeros), ctypes.byref(cs) if cs is not None else None, _ptr(y), M, N, K]
    if group_size is not None:
        args.append(int(group_size))
    args += [_ptr(ws), ws.numel() if ws is not None else 0]
    if schedule is not None:
        args.append(int(schedule))
    code = getattr(lib(), name)(*args, _stream(x.device))
    _check(code, name)
    return y


def w4a16_linear(x, qweight, scales, zeros, csr=None, out=None, workspace=None):
    """y = x . dequant(Q)^T (+ CSR term); M <= 16 runs the GEMV (with a cached workspace)."""
    return _linear("w4a16_linear", x, qweight, scales, zeros, csr, out, workspace)


def w4a16_gemv(x, qweight, scales, zeros, csr=None, out=None, workspace=None):
    return _linear("w4a16_gemv", x, qweight, scales, zeros, csr, out, workspace)


def w4a16_gemv_ex(x, qweight, scales, zeros, csr=None, out=None, workspace=None, schedule=GEMV_AUTO):
    return _linear("w4a16_gemv_ex", x, qweight, scales, zeros, csr, out, workspace, schedule)


def w4a16_linear_ex(x, qweight, scales, zeros, csr=None, out=None, workspace=None, group_size=128,
                    schedule=GEMV_AUTO):
    """w4a16_linear for weights quantized in groups of group_size along K."""
    return _linear("w4a16_linear_ex", x, qweight, scales, zeros, csr, out, workspace, schedule, group_size)


def w3a16_gemv(x, qweight3, scales, zeros, csr=None, out=None, workspace=None, group_size=128, schedule=GEMV_AUTO):
    """The decode GEMV (M <= 16) on 3-bit codes as awq_quantize3 writes them."""
    return _linear("w3a16_gemv", x, qweight3, scales, zeros, csr, out, workspace, schedule, group_size, bits=3)


def w4a16_gemv_folded(x, s, qweight, scales, zeros, csr=None, out=None, workspace=None, group_size=128,
                      schedule=GEMV_AUTO):
    """The decode GEMV on the raw layer input in one call: x is divided by the channel scales s
    (fp32 [K], or None for an already divided x) into the workspace, as awq_fold_activations
    would, and the GEMV reads the result."""
    return _linear("w4a16_gemv_folded", x, qweight, scales, zeros, csr, out, workspace, schedule, group_size,
                   fold=True, s=s)


def gemv_plan(M: int, N: int, K: int, schedule: int = GEMV_AUTO):
    """(schedule, CTAs per cluster or 0, CTAs) that w4a16_gemv_ex would launch on the current device."""
    r, c, n = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    _check(lib().w4a16_gemv_plan(M, N, K, int(schedule), ctypes.byref(r), ctypes.byref(c), ctypes.byref(n)),
           "w4a16_gemv_plan")
    return r.value, c.value, n.value


def gemm_plan(M: int, N: int, K: int, num_sms: int):
    """(token tile, splits along K, 128-k slices per split, partial-tile bytes) of the prefill GEMM on a
    device with num_sms SMs (host arithmetic; needs no GPU)."""
    bn, sp, sl, pb = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0), ctypes.c_size_t(0)
    _check(lib().w4a16_gemm_plan(M, N, K, int(num_sms), ctypes.byref(bn), ctypes.byref(sp), ctypes.byref(sl),
                                 ctypes.byref(pb)), "w4a16_gemm_plan")
    return bn.value, sp.value, sl.value, pb.value


def w4a16_gemm(x, qweight, scales, zeros, csr=None, out=None, workspace=None):
    return _linear("w4a16_gemm", x, qweight, scales, zeros, csr, out, workspace)


def check_device_status(stream=None):
    """Synchronize and raise W4A16Error if a kernel recorded a problem since the last check."""
    s = ctypes.c_void_p(stream.cuda_stream) if stream is not None else _stream(torch.device("cuda"))
    _check(lib().w4a16_check_device_status(s), "device status")


def awq_split_outliers(W, act_absmean, alpha: float, nnz: int, out=None, workspace=None):
    """Dense-and-sparse split on the GPU.  W fp32 [N][K], act_absmean fp32 [K] (cuda).
    Returns (W_dense fp32 [N][K], (row_ptr int32 [N+1], col_idx int32 [nnz], values int16
    (fp16 bits) [nnz])), ready for awq_quantize_g128 and the csr= argument of the linear ops."""
    assert W.is_cuda and W.dtype == torch.float32 and W.dim() == 2 and W.is_contiguous()
    assert act_absmean.dtype == torch.float32 and act_absmean.is_contiguous()
    N, K = W.shape
    dev = W.device
    if out is None:
        out = (torch.empty_like(W), torch.empty(N + 1, dtype=torch.int32, device=dev),
               torch.empty(max(nnz, 1), dtype=torch.int32, device=dev),
               torch.empty(max(nnz, 1), dtype=torch.int16, device=dev))
    Wd, rp, ci, vals = out
    nbytes = lib().awq_split_outliers_workspace_bytes(N, K)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
    _check(lib().awq_split_outliers(_ptr(W), _ptr(act_absmean), ctypes.c_float(alpha), N, K, int(nnz), _ptr(Wd),
                                    _ptr(rp), _ptr(ci), _ptr(vals), _ptr(workspace), workspace.numel(),
                                    _stream(dev)), "awq_split_outliers")
    return Wd, (rp, ci[:nnz], vals[:nnz])


def awq_search_alpha(W, act_absmean, x_calib, alphas, workspace=None):
    """AWQ scale search on the GPU.  W fp32 [N][K], act_absmean fp32 [K], x_calib bf16 [M][K]
    (cuda), alphas a sequence of floats.  Returns (errors list, best index); synchronous."""
    assert W.is_cuda and W.dtype == torch.float32 and W.is_contiguous() and x_calib.dtype == torch.bfloat16
    N, K = W.shape
    M = x_calib.shape[0]
    al = (ctypes.c_float * len(alphas))(*[float(a) for a in alphas])
    err = (ctypes.c_float * len(alphas))()
    best = ctypes.c_int(-1)
    nbytes = lib().awq_search_alpha_workspace_bytes(M, N, K, len(alphas))
    if workspace is None:
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=W.device)
    _check(lib().awq_search_alpha(_ptr(W), _ptr(act_absmean), _ptr(x_calib), M, N, K, al, len(alphas), err,
                                  ctypes.byref(best), _ptr(workspace), workspace.numel(), _stream(W.device)),
           "awq_search_alpha")
    return list(err), best.value


def awq_fold_activations(x, s, out=None):
    """x' = bf16(x / s) for bf16 x [M][K] and fp32 s [K] (cuda)."""
    assert x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous() and s.dtype == torch.float32
    M, K = x.shape
    out = torch.empty_like(x) if out is None else out
    _check(lib().awq_fold_activations(_ptr(x), _ptr(s), _ptr(out), M, K, _stream(x.device)), "awq_fold_activations")
    return out


def selftest_timeout(limit_ns: int, stream=None) -> None:
    """Launch the kernel whose wait can never complete (limit in ns); the next
    check_device_status() reports W4A16_ERR_TIMEOUT."""
    s = ctypes.c_void_p(stream.cuda_stream) if stream is not None else _stream(torch.device("cuda"))
    _check(lib().w4a16_selftest_timeout(int(limit_ns), s), "selftest_timeout")


def selftest_quotient():
    """(mismatches, first) of the quantizer's division against the IEEE one on its whole
    domain (w4a16_selftest_quotient); first = (divisor, dividend, got, want) float bits."""
    n = ctypes.c_uint64(0)
    first = (ctypes.c_uint32 * 4)()
    _check(lib().w4a16_selftest_quotient(ctypes.byref(n), first, _stream(torch.device("cuda"))), "selftest_quotient")
    return int(n.value), tuple(int(v) for v in first)


def status_string(code: int) -> str:
    return lib().w4a16_status_string(code).decode()


def version() -> int:
    return lib().w4a16_version()


# ---- the remaining entry points under their C names -------------------------------------

def w4a16_gemv_noalloc(x, qweight, scales, zeros, csr=None, out=None):
    """The decode GEMV without a caller workspace (the library's static scratch)."""
    check_linear_shapes(x, qweight, scales, zeros, csr, out)
    _need(x, torch.bfloat16, 2, "x")
    _need(qweight, torch.int32, 2, "qweight")
    _need(scales, torch.int16, 2, "scales")
    _need(zeros, torch.int32, 2, "zeros")
    M, K = x.shape
    N = qweight.shape[0]
    y = out if out is not None else torch.empty(M, N, dtype=torch.bfloat16, device=x.device)
    cs = None
    if csr is not None:
        rp, ci, v = csr
        _need(rp, torch.int32, 1, "row_ptr")
        cs = Csr(rp.data_ptr(), ci.data_ptr() if ci.numel() else None, v.data_ptr() if v.numel() else None,
                 int(ci.numel()))
    _check(lib().w4a16_gemv_noalloc(_ptr(x), _ptr(qweight), _ptr(scales), _ptr(zeros),
                                    ctypes.byref(cs) if cs is not None else None, _ptr(y), M, N, K,
                                    _stream(x.device)), "w4a16_gemv_noalloc")
    return y


def awq_split_outliers_workspace_bytes(N: int, K: int) -> int:
    return int(lib().awq_split_outliers_workspace_bytes(N, K))


def awq_search_alpha_workspace_bytes(M: int, N: int, K: int, n_alpha: int) -> int:
    return int(lib().awq_search_alpha_workspace_bytes(M, N, K, int(n_alpha)))


w4a16_workspace_bytes = workspace_bytes


def w4a16_workspace_bytes_ex(M: int, N: int, K: int, with_csr: int) -> int:
    return workspace_bytes(M, N, K, bool(with_csr))


w4a16_gemv_plan = gemv_plan
w4a16_gemm_plan = gemm_plan
w4a16_check_device_status = check_device_status
w4a16_selftest_timeout = selftest_timeout
w4a16_selftest_quotient = selftest_quotient
w4a16_status_string = status_string
w4a16_version = version
