"""CPU oracle for the W4A16 AWQ g128 quantized linear layer (numpy front end).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the CPU-baseline leg of the
benchmark are the only callers.  The product library never imports this package, and
this package never imports the product library; they share only the seeded input
generators in ``workloads``.

The arithmetic lives in ``oracle.c`` (plain C, one IEEE-754 float operation per source
operation, double accumulation for the matrix product); this module marshals numpy
arrays into it.  ``build()`` compiles it with gcc.  Every function says which passage of
the pages it follows in the C source.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

OK, ERR_NULL, ERR_SHAPE, ERR_VALUE = 0, 1, 2, 4
GROUP = 128


class OracleError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"oracle {what} failed with status {code}")
        self.code = code


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, no FMA contraction, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-shared",
               "-fPIC", "-std=c11", "-Wall", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


_lib = None


def _L():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        F = ctypes.c_float
        sig = {
            "oracle_f32_to_f16": ([F], ctypes.c_uint16),
            "oracle_f16_to_f32": ([ctypes.c_uint16], F),
            "oracle_f32_to_bf16": ([F], ctypes.c_uint16),
            "oracle_bf16_to_f32": ([ctypes.c_uint16], F),
            "oracle_pack8": ([P, P], ctypes.c_int),
            "oracle_unpack8": ([ctypes.c_uint32, P], None),
            "oracle_awq_scales": ([P, I64, F, P], ctypes.c_int),
            "oracle_quantize_with_scales": ([P, P, I64, I64, P, P, P], ctypes.c_int),
            "oracle_awq_quantize_g128": ([P, P, F, I64, I64, P, P, P, P], ctypes.c_int),
            "oracle_awq_quantize_gs": ([P, P, F, I64, I64, I64, P, P, P, P], ctypes.c_int),
            "oracle_quantize_with_scales_gs": ([P, P, I64, I64, I64, P, P, P], ctypes.c_int),
            "oracle_dequant": ([P, P, P, I64, I64, P], ctypes.c_int),
            "oracle_dequant_gs": ([P, P, P, I64, I64, I64, P], ctypes.c_int),
            "oracle_linear": ([P, I64, I64, P, P, P, I64, P, P, P, I64, P, P], ctypes.c_int),
            "oracle_linear_gs": ([P, I64, I64, I64, P, P, P, I64, P, P, P, I64, P, P], ctypes.c_int),
            "oracle_linear_at": ([P, I64, I64, P, P, P, I64, P, P, P, I64, P, P, I64, P, P],
                                 ctypes.c_int),
            "oracle_linear_at_gs": ([P, I64, I64, I64, P, P, P, I64, P, P, P, I64, P, P, I64, P, P],
                                    ctypes.c_int),
            "oracle_split_outliers": ([P, P, F, I64, I64, I64, P, P, P, P], ctypes.c_int),
            "oracle_awq_search_alpha": ([P, P, P, I64, I64, I64, P, I64, P], ctypes.c_int),
            "oracle_pack32x3": ([P, P], ctypes.c_int),
            "oracle_unpack32x3": ([P, P], None),
            "oracle_awq_quantize3_gs": ([P, P, F, I64, I64, I64, P, P, P, P], ctypes.c_int),
            "oracle_dequant3_gs": ([P, P, P, I64, I64, I64, P], ctypes.c_int),
            "oracle_linear3_gs": ([P, I64, I64, I64, P, P, P, I64, P, P, P, I64, P, P], ctypes.c_int),
            "oracle_linear3_at_gs": ([P, I64, I64, I64, P, P, P, I64, P, P, P, I64, P, P, I64, P, P],
                                     ctypes.c_int),
            "oracle_f32_to_e4m3": ([F], ctypes.c_uint8),
            "oracle_e4m3_to_f32": ([ctypes.c_uint8], F),
            "oracle_f32_to_e2m1": ([F], ctypes.c_uint8),
            "oracle_e2m1_to_f32": ([ctypes.c_uint8], F),
            "oracle_quantize_nvfp4_with_scales": ([P, P, I64, I64, P, P, P], ctypes.c_int),
            "oracle_awq_quantize_nvfp4": ([P, P, F, I64, I64, P, P, P, P], ctypes.c_int),
            "oracle_dequant_nvfp4": ([P, P, F, I64, I64, P], ctypes.c_int),
            "oracle_linear_nvfp4": ([P, I64, I64, P, P, F, I64, P, P, P, I64, P, P], ctypes.c_int),
        }
        for name, (args, res) in sig.items():
            fn = getattr(_lib, name)
            fn.argtypes = args
            fn.restype = res
    return _lib


def _p(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _check(code, what):
    if code != OK:
        raise OracleError(code, what)


# ---- scalar conversions (IEEE-754 round-to-nearest-even, from the definition) ----------

def f32_to_f16_bits(f: float) -> int:
    return int(_L().oracle_f32_to_f16(ctypes.c_float(f)))


def f16_bits_to_f32(h: int) -> float:
    return float(_L().oracle_f16_to_f32(ctypes.c_uint16(h)))


def f32_to_bf16_bits(f: float) -> int:
    return int(_L().oracle_f32_to_bf16(ctypes.c_float(f)))


def bf16_bits_to_f32(h: int) -> float:
    return float(_L().oracle_bf16_to_f32(ctypes.c_uint16(h)))


def pack8(codes) -> int:
    q = _c(codes, np.uint8)
    w = np.zeros(1, np.uint32)
    _check(_L().oracle_pack8(_p(q), _p(w)), "pack8")
    return int(w[0])


def unpack8(word: int) -> np.ndarray:
    q = np.zeros(8, np.uint8)
    _L().oracle_unpack8(ctypes.c_uint32(word), _p(q))
    return q


def pack32x3(codes) -> np.ndarray:
    """32 codes (0..7, element order) -> the 3 words of the 3-bit layout."""
    q = _c(codes, np.uint8)
    w = np.zeros(3, np.uint32)
    _check(_L().oracle_pack32x3(_p(q), _p(w)), "pack32x3")
    return w


def unpack32x3(words) -> np.ndarray:
    w = _c(words, np.uint32)
    q = np.zeros(32, np.uint8)
    _L().oracle_unpack32x3(_p(w), _p(q))
    return q


# ---- the method -------------------------------------------------------------------------

def awq_scales(act_absmean, alpha: float) -> np.ndarray:
    a = _c(act_absmean, np.float32)
    s = np.empty_like(a)
    _check(_L().oracle_awq_scales(_p(a), a.size, ctypes.c_float(alpha), _p(s)), "awq_scales")
    return s


def quantize_with_scales(W, s, group_size: int = 128):
    W = _c(W, np.float32)
    s = _c(s, np.float32)
    N, K = W.shape
    G = max(K // group_size, 1)
    qw = np.zeros((N, K // 8), np.uint32)
    sc = np.zeros((G, N), np.uint16)
    z = np.zeros((G, max(N // 8, 1)), np.uint32)
    _check(_L().oracle_quantize_with_scales_gs(_p(W), _p(s), N, K, group_size, _p(qw), _p(sc), _p(z)),
           "quantize_with_scales")
    return qw, sc, z


def awq_quantize_g128(W, act_absmean, alpha: float):
    """-> (qweight u32 [N][K/8], scales fp16 bits u16 [K/128][N], zeros u32 [K/128][N/8], s f32 [K])"""
    W = _c(W, np.float32)
    a = _c(act_absmean, np.float32)
    N, K = W.shape
    qw = np.zeros((N, K // 8), np.uint32)
    sc = np.zeros((K // 128, N), np.uint16)
    z = np.zeros((K // 128, max(N // 8, 1)), np.uint32)
    s = np.zeros(K, np.float32)
    _check(_L().oracle_awq_quantize_g128(_p(W), _p(a), ctypes.c_float(alpha), N, K, _p(qw), _p(sc),
                                         _p(z), _p(s)), "awq_quantize_g128")
    return qw, sc, z, s


def awq_quantize(W, act_absmean, alpha: float, group_size: int):
    """AWQ quantize with groups of group_size along K (group_size = K: one group per row)
    -> (qweight u32 [N][K/8], scales u16 [K/gs][N], zeros u32 [K/gs][N/8], s f32 [K])"""
    W = _c(W, np.float32)
    a = _c(act_absmean, np.float32)
    N, K = W.shape
    G = max(K // group_size, 1)
    qw = np.zeros((N, K // 8), np.uint32)
    sc = np.zeros((G, N), np.uint16)
    z = np.zeros((G, max(N // 8, 1)), np.uint32)
    s = np.zeros(K, np.float32)
    _check(_L().oracle_awq_quantize_gs(_p(W), _p(a), ctypes.c_float(alpha), N, K, group_size, _p(qw), _p(sc),
                                       _p(z), _p(s)), "awq_quantize")
    return qw, sc, z, s


def dequant(qweight, scales, zeros, N: int, K: int, group_size: int = 128) -> np.ndarray:
    qw, sc, z = _c(qweight, np.uint32), _c(scales, np.uint16), _c(zeros, np.uint32)
    out = np.zeros((N, K), np.float32)
    _check(_L().oracle_dequant_gs(_p(qw), _p(sc), _p(z), N, K, group_size, _p(out)), "dequant")
    return out


def _csr_args(csr):
    if csr is None:
        return None, None, None, 0
    rp, ci, v = csr
    return _c(rp, np.int32), _c(ci, np.int32), _c(v, np.uint16), int(len(ci))


def linear(x_bf16_bits, qweight, scales, zeros, N: int, csr=None, with_abs: bool = False, group_size: int = 128):
    """y[m][n] = sum_k x deq + sum_csr x val, in double.  x is bf16 bits (uint16) [M][K].
    csr = (row_ptr int32 [N+1], col_idx int32 [nnz], values fp16 bits [nnz]) or None."""
    x = _c(x_bf16_bits, np.uint16)
    M, K = x.shape
    qw, sc, z = _c(qweight, np.uint32), _c(scales, np.uint16), _c(zeros, np.uint32)
    rp, ci, v, nnz = _csr_args(csr)
    y = np.zeros((M, N), np.float64)
    ya = np.zeros((M, N), np.float64) if with_abs else None
    _check(_L().oracle_linear_gs(_p(x), M, K, group_size, _p(qw), _p(sc), _p(z), N, _p(rp), _p(ci), _p(v), nnz,
                                 _p(y), _p(ya)), "linear")
    return (y, ya) if with_abs else y


def linear_at(x_bf16_bits, qweight, scales, zeros, N: int, m_idx, n_idx, csr=None,
              with_abs: bool = False, group_size: int = 128):
    """The outputs of ``linear`` at the positions (m_idx[p], n_idx[p]) only."""
    x = _c(x_bf16_bits, np.uint16)
    M, K = x.shape
    qw, sc, z = _c(qweight, np.uint32), _c(scales, np.uint16), _c(zeros, np.uint32)
    mi, ni = _c(m_idx, np.int64), _c(n_idx, np.int64)
    rp, ci, v, nnz = _csr_args(csr)
    y = np.zeros(mi.size, np.float64)
    ya = np.zeros(mi.size, np.float64) if with_abs else None
    _check(_L().oracle_linear_at_gs(_p(x), M, K, group_size, _p(qw), _p(sc), _p(z), N, _p(rp), _p(ci), _p(v),
                                    nnz, _p(mi), _p(ni), mi.size, _p(y), _p(ya)), "linear_at")
    return (y, ya) if with_abs else y


def awq_quantize3(W, act_absmean, alpha: float, group_size: int = 128):
    """AWQ quantize with 3-bit codes -> (qweight3 u32 [N][3K/32], scales u16 [K/gs][N],
    zeros u32 [K/gs][N/8] (nibbles 0..7), s f32 [K])"""
    W = _c(W, np.float32)
    a = _c(act_absmean, np.float32)
    N, K = W.shape
    G = max(K // group_size, 1)
    qw = np.zeros((N, 3 * K // 32), np.uint32)
    sc = np.zeros((G, N), np.uint16)
    z = np.zeros((G, max(N // 8, 1)), np.uint32)
    s = np.zeros(K, np.float32)
    _check(_L().oracle_awq_quantize3_gs(_p(W), _p(a), ctypes.c_float(alpha), N, K, group_size, _p(qw), _p(sc),
                                        _p(z), _p(s)), "awq_quantize3")
    return qw, sc, z, s


def dequant3(qweight3, scales, zeros, N: int, K: int, group_size: int = 128) -> np.ndarray:
    qw, sc, z = _c(qweight3, np.uint32), _c(scales, np.uint16), _c(zeros, np.uint32)
    out = np.zeros((N, K), np.float32)
    _check(_L().oracle_dequant3_gs(_p(qw), _p(sc), _p(z), N, K, group_size, _p(out)), "dequant3")
    return out


def linear3(x_bf16_bits, qweight3, scales, zeros, N: int, csr=None, with_abs: bool = False,
            group_size: int = 128):
    """``linear`` on 3-bit weights."""
    x = _c(x_bf16_bits, np.uint16)
    M, K = x.shape
    qw, sc, z = _c(qweight3, np.uint32), _c(scales, np.uint16), _c(zeros, np.uint32)
    rp, ci, v, nnz = _csr_args(csr)
    y = np.zeros((M, N), np.float64)
    ya = np.zeros((M, N), np.float64) if with_abs else None
    _check(_L().oracle_linear3_gs(_p(x), M, K, group_size, _p(qw), _p(sc), _p(z), N, _p(rp), _p(ci), _p(v), nnz,
                                  _p(y), _p(ya)), "linear3")
    return (y, ya) if with_abs else y


def linear3_at(x_bf16_bits, qweight3, scales, zeros, N: int, m_idx, n_idx, csr=None,
               with_abs: bool = False, group_size: int = 128):
    """The outputs of ``linear3`` at the positions (m_idx[p], n_idx[p]) only."""
    x = _c(x_bf16_bits, np.uint16)
    M, K = x.shape
    qw, sc, z = _c(qweight3, np.uint32), _c(scales, np.uint16), _c(zeros, np.uint32)
    mi, ni = _c(m_idx, np.int64), _c(n_idx, np.int64)
    rp, ci, v, nnz = _csr_args(csr)
    y = np.zeros(mi.size, np.float64)
    ya = np.zeros(mi.size, np.float64) if with_abs else None
    _check(_L().oracle_linear3_at_gs(_p(x), M, K, group_size, _p(qw), _p(sc), _p(z), N, _p(rp), _p(ci), _p(v),
                                     nnz, _p(mi), _p(ni), mi.size, _p(y), _p(ya)), "linear3_at")
    return (y, ya) if with_abs else y


def split_outliers(W, act_absmean, alpha: float, nnz: int):
    """-> (W_dense f32 [N][K], row_ptr i32 [N+1], col_idx i32 [nnz], values fp16 bits [nnz])"""
    W = _c(W, np.float32)
    a = _c(act_absmean, np.float32)
    N, K = W.shape
    Wd = np.zeros_like(W)
    rp = np.zeros(N + 1, np.int32)
    ci = np.zeros(max(nnz, 1), np.int32)
    v = np.zeros(max(nnz, 1), np.uint16)
    _check(_L().oracle_split_outliers(_p(W), _p(a), ctypes.c_float(alpha), N, K, nnz, _p(Wd), _p(rp),
                                      _p(ci), _p(v)), "split_outliers")
    return Wd, rp, ci[:nnz], v[:nnz]


def awq_search_alpha(W, act_absmean, x_bf16_bits, alphas):
    """Relative squared output error of the quantized layer for every alpha of the grid
    (see oracle_awq_search_alpha).  Returns float64 [len(alphas)]."""
    W = _c(W, np.float32)
    a = _c(act_absmean, np.float32)
    x = _c(x_bf16_bits, np.uint16)
    al = _c(alphas, np.float32)
    N, K = W.shape
    M = x.shape[0]
    err = np.zeros(al.size, np.float64)
    _check(_L().oracle_awq_search_alpha(_p(W), _p(a), _p(x), M, N, K, _p(al), al.size, _p(err)),
           "awq_search_alpha")
    return err


# ---- NVFP4 weights (E2M1 codes, an E4M3 scale per 16 weights, an fp32 tensor scale) -----

def f32_to_e4m3_bits(f: float) -> int:
    return int(_L().oracle_f32_to_e4m3(ctypes.c_float(f)))


def e4m3_bits_to_f32(b: int) -> float:
    return float(_L().oracle_e4m3_to_f32(ctypes.c_uint8(b)))


def f32_to_e2m1_code(f: float) -> int:
    return int(_L().oracle_f32_to_e2m1(ctypes.c_float(f)))


def e2m1_code_to_f32(c: int) -> float:
    return float(_L().oracle_e2m1_to_f32(ctypes.c_uint8(c)))


def quantize_nvfp4_with_scales(W, s):
    """NVFP4 of W*s -> (qweight u32 [N][K/8], scales8 u8 [K/16][N], g float)."""
    W = _c(W, np.float32)
    s = _c(s, np.float32)
    N, K = W.shape
    qw = np.zeros((N, max(K // 8, 1)), np.uint32)
    sc = np.zeros((max(K // 16, 1), N), np.uint8)
    g = np.zeros(1, np.float32)
    _check(_L().oracle_quantize_nvfp4_with_scales(_p(W), _p(s), N, K, _p(qw), _p(sc), _p(g)),
           "quantize_nvfp4_with_scales")
    return qw, sc, float(g[0])


def awq_quantize_nvfp4(W, act_absmean, alpha: float):
    """AWQ scaling then NVFP4 -> (qweight u32 [N][K/8], scales8 u8 [K/16][N], g float, s f32 [K])."""
    W = _c(W, np.float32)
    a = _c(act_absmean, np.float32)
    N, K = W.shape
    qw = np.zeros((N, max(K // 8, 1)), np.uint32)
    sc = np.zeros((max(K // 16, 1), N), np.uint8)
    g = np.zeros(1, np.float32)
    s = np.zeros(K, np.float32)
    _check(_L().oracle_awq_quantize_nvfp4(_p(W), _p(a), ctypes.c_float(alpha), N, K, _p(qw), _p(sc), _p(g), _p(s)),
           "awq_quantize_nvfp4")
    return qw, sc, float(g[0]), s


def dequant_nvfp4(qweight, scales8, g: float, N: int, K: int) -> np.ndarray:
    qw, sc = _c(qweight, np.uint32), _c(scales8, np.uint8)
    out = np.zeros((N, K), np.float64)
    _check(_L().oracle_dequant_nvfp4(_p(qw), _p(sc), ctypes.c_float(g), N, K, _p(out)), "dequant_nvfp4")
    return out


def linear_nvfp4(x_bf16_bits, qweight, scales8, g: float, N: int, csr=None, with_abs: bool = False):
    """``linear`` on NVFP4 weights."""
    x = _c(x_bf16_bits, np.uint16)
    M, K = x.shape
    qw, sc = _c(qweight, np.uint32), _c(scales8, np.uint8)
    rp, ci, v, nnz = _csr_args(csr)
    y = np.zeros((M, N), np.float64)
    ya = np.zeros((M, N), np.float64) if with_abs else None
    _check(_L().oracle_linear_nvfp4(_p(x), M, K, _p(qw), _p(sc), ctypes.c_float(g), N, _p(rp), _p(ci), _p(v), nnz,
                                    _p(y), _p(ya)), "linear_nvfp4")
    return (y, ya) if with_abs else y
