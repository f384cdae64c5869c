"""Shared helpers of the GPU parity tests: moving seeded host inputs to the device, and the
comparison of a bf16 GPU result with the oracle's double-precision result.

Tolerance (the output criterion): max_i |y_i - r_i| / max_i |r_i| <= 1e-2 per output row of
tokens.  The tests also check a per-element bound derived from the arithmetic:
  |y - r| <= 2^-8 |r|                       (one bf16 rounding of the output, with slack)
           + c_w * sum_k |x_k w_k|           (c_w: relative error of the weights fed to the MMA;
                                             0 on the GEMV, whose weights are exact integers
                                             scaled in fp32; 2^-8 on the GEMM, which rounds the
                                             scale and the product to bf16)
           + depth * 2^-22 * sum_k |x_k w_k| (fp32 accumulation, depth = sequential adds)
"""
from __future__ import annotations

import numpy as np
import torch

Y_REL_TOL = 1e-2


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def dev_bits(a: np.ndarray, dtype) -> torch.Tensor:
    np_dtype = {torch.int32: np.int32, torch.int16: np.int16}[dtype]
    return torch.from_numpy(np.ascontiguousarray(a).view(np_dtype)).cuda()


def dev_f32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()


def dev_csr(csr):
    rp, ci, v = csr
    return (torch.from_numpy(np.ascontiguousarray(rp, np.int32)).cuda(),
            torch.from_numpy(np.ascontiguousarray(ci, np.int32)).cuda(),
            torch.from_numpy(np.ascontiguousarray(v, np.uint16).view(np.int16)).cuda())


def host_bits(t: torch.Tensor, np_dtype) -> np.ndarray:
    return t.cpu().numpy().view(np_dtype)


def host_bf16_as_f64(y: torch.Tensor) -> np.ndarray:
    bits = y.cpu().view(torch.int16).numpy().view(np.uint16).astype(np.uint32) << 16
    return bits.view(np.float32).astype(np.float64)


# The decode GEMV feeds the MMA the exact biased codes (128 + q) and removes the bias per
# group in fp32: s * (sum (128+q) x - (128+z) X_g).  Its rounding error is then relative to
# 143 * sum_k |x_k| s_g, not to sum |x w|: with <= 24 sequential fp32 adds in the MMA chain
# (2^-23 each, truncating accumulation assumed) and <= 130 in X_g and the correction (2^-24):
GEMV_XS_COEF = 143.0 * (24 * 2.0 ** -23 + 130 * 2.0 ** -24)


def xs_abs(x_bits: np.ndarray, scales: np.ndarray, m_idx=None, n_idx=None) -> np.ndarray:
    """sum_k |x[m][k]| * scale[n][k // 128] for all (m, n) or at the sampled positions."""
    x = (x_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    M, K = x.shape
    xa = np.abs(x).reshape(M, K // 128, 128).sum(-1)              # [M][G]
    sc = scales.view(np.float16).astype(np.float64).T               # stored [G][N] -> [N][G]
    if m_idx is None:
        return xa @ sc.T
    return np.einsum("pg,pg->p", xa[m_idx], sc[n_idx])


def check_close(y: np.ndarray, ref: np.ndarray, ref_abs: np.ndarray, c_w: float, depth: int, what: str = "",
                xsabs: np.ndarray | None = None):
    """y, ref, ref_abs: float64 arrays of the same shape ([M][N] or sampled [P]).  xsabs, when
    given, adds GEMV_XS_COEF * xsabs to the per-element bound (the decode GEMV's arithmetic)."""
    assert y.shape == ref.shape
    assert np.all(np.isfinite(y)), f"{what}: non-finite output"
    err = np.abs(y - ref)
    if ref.ndim == 2:
        rel = err.max(axis=1) / np.maximum(np.abs(ref).max(axis=1), 1e-30)
    else:
        rel = np.array([err.max() / max(np.abs(ref).max(), 1e-30)])
    assert rel.max() <= Y_REL_TOL, f"{what}: max relative error {rel.max():.3e} > {Y_REL_TOL}"
    bound = 2.0 ** -8 * np.abs(ref) + (c_w + depth * 2.0 ** -22) * ref_abs + 1e-30
    if xsabs is not None:
        bound = bound + GEMV_XS_COEF * xsabs
    bad = err > bound
    assert not bad.any(), (f"{what}: {bad.sum()} outputs beyond the per-element bound; worst "
                           f"err/bound = {(err / bound).max():.3f}")
    return float(rel.max())


class Case:
    """A seeded layer quantized by the oracle, its activations and (optionally) its CSR."""

    def __init__(self, orc, seed: int, K: int, N: int, M: int, csr: bool = False, alpha: float = 0.5,
                 nnz: int | None = None):
        import workloads
        L = workloads.make_layer(seed, K=K, N=N)
        W = L.W
        self.csr = None
        if csr:
            n = workloads.outlier_nnz(N, K) if nnz is None else nnz
            Wd, rp, ci, v = orc.split_outliers(W, L.act_absmean, alpha, n)
            self.csr = (rp, ci, v)
            W = Wd
        self.qw, self.sc, self.z, self.s = orc.awq_quantize_g128(W, L.act_absmean, alpha)
        self.x = workloads.make_activations(seed, M, L.mult, alpha)
        self.K, self.N, self.M = K, N, M

    def device(self):
        d = dict(x=dev_bf16(self.x), qweight=dev_bits(self.qw, torch.int32), scales=dev_bits(self.sc, torch.int16),
                 zeros=dev_bits(self.z, torch.int32))
        d["csr"] = dev_csr(self.csr) if self.csr is not None else None
        return d

    def reference(self, orc):
        return orc.linear(self.x, self.qw, self.sc, self.z, self.N, csr=self.csr, with_abs=True)

    def reference_at(self, orc, m_idx, n_idx):
        return orc.linear_at(self.x, self.qw, self.sc, self.z, self.N, m_idx, n_idx, csr=self.csr, with_abs=True)

    def sample(self, seed: int, P: int = 1536):
        """Sampled output positions: P random ones plus every channel of the first and last token."""
        rng = np.random.default_rng(seed)
        m = np.concatenate([rng.integers(0, self.M, P), np.zeros(self.N, np.int64),
                            np.full(self.N, self.M - 1, np.int64)])
        n = np.concatenate([rng.integers(0, self.N, P), np.arange(self.N), np.arange(self.N)])
        return m, n
