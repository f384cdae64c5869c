"""GPU tcgen05 GEMM against the oracle: token tails, every tile width, CSR folded into the
weights, exact-weight cases with a tight bound, and the full prefill shapes (sampled)."""
import numpy as np
import pytest
import torch

import w4a16_gemm_awq_b200 as w4
import workloads
from parity import Case, check_close, dev_bf16, dev_bits, dev_csr, host_bf16_as_f64

pytestmark = pytest.mark.gpu

C_W = 2.0 ** -8 * 1.01   # bf16 scale and bf16 product: the weights' relative error on the MMA
C_W_CSR = 2.0 ** -7      # plus the rounding of (weight + outlier value)


def gemm(d, fn=None):
    fn = fn or w4.w4a16_gemm
    y = fn(d["x"], d["qweight"], d["scales"], d["zeros"], csr=d["csr"])
    w4.check_device_status()
    return y


def depth(K):
    return K // 16 + 64


@pytest.mark.parametrize("M", [1, 16, 17, 32, 33, 64, 100, 128, 129, 200, 256, 300, 640])
def test_gemm_small_full_output(orc, M):
    c = Case(orc, seed=200 + M, K=2048, N=256, M=M)
    y = host_bf16_as_f64(gemm(c.device()))
    ref, ref_abs = c.reference(orc)
    check_close(y, ref, ref_abs, C_W, depth(c.K), f"M={M}")


@pytest.mark.parametrize("M", [3, 70, 257])
def test_gemm_small_with_csr(orc, M):
    c = Case(orc, seed=300 + M, K=2048, N=384, M=M, csr=True)
    y = host_bf16_as_f64(gemm(c.device()))
    ref, ref_abs = c.reference(orc)
    check_close(y, ref, ref_abs, C_W_CSR, depth(c.K), f"M={M} csr")


def _exact_layer(seed, N, K):
    """Weights whose dequantized values are exact in bf16: per group (i - z0) * 2^e."""
    rng = np.random.default_rng(seed)
    W = np.empty((N, K), np.float32)
    i = np.arange(128) % 16
    for n in range(N):
        for g in range(K // 128):
            z0 = int(rng.integers(0, 16))
            W[n, g * 128:(g + 1) * 128] = rng.permutation((i - z0) * 2.0 ** int(rng.integers(-9, -3)))
    return W


@pytest.mark.parametrize("M", [40, 256, 513])
def test_gemm_exact_weights_tight(orc, M):
    """When every dequantized weight is exact in bf16, only accumulation and the output rounding
    remain: a misplaced k, token or channel fails the per-element bound."""
    K, N = 2048, 256
    W = _exact_layer(M, N, K)
    qw, sc, z, _ = orc.awq_quantize_g128(W, np.ones(K, np.float32), 0.0)
    x = workloads.uniform_bf16(M, (M, K), -3, 3)
    d = dict(x=dev_bf16(x), qweight=dev_bits(qw, torch.int32), scales=dev_bits(sc, torch.int16),
             zeros=dev_bits(z, torch.int32), csr=None)
    y = host_bf16_as_f64(gemm(d))
    ref, ref_abs = orc.linear(x, qw, sc, z, N, with_abs=True)
    assert np.array_equal(orc.dequant(qw, sc, z, N, K), W)
    check_close(y, ref, ref_abs, 0.0, depth(K), f"exact M={M}")


def test_gemm_empty_csr_is_bit_identical(orc):
    c = Case(orc, seed=17, K=2048, N=256, M=300)
    d = c.device()
    y0 = gemm(d)
    d["csr"] = (torch.zeros(c.N + 1, dtype=torch.int32, device="cuda"), torch.zeros(0, dtype=torch.int32, device="cuda"),
                torch.zeros(0, dtype=torch.int16, device="cuda"))
    y1 = gemm(d)
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))


def test_gemm_reports_unsorted_csr(orc):
    c = Case(orc, seed=19, K=1024, N=128, M=64)
    d = c.device()
    rp = torch.zeros(c.N + 1, dtype=torch.int32, device="cuda")
    rp[1:] = 2
    d["csr"] = (rp, torch.tensor([600, 100], dtype=torch.int32, device="cuda"),
                torch.tensor([0x3C00, 0x3C00], dtype=torch.int16, device="cuda"))
    w4.w4a16_gemm(d["x"], d["qweight"], d["scales"], d["zeros"], csr=d["csr"])
    with pytest.raises(w4.W4A16Error) as e:
        w4.check_device_status()
    assert e.value.code == w4.ERR_SHAPE


def test_linear_dispatches_to_gemm(orc):
    c = Case(orc, seed=21, K=2048, N=256, M=17)
    d = c.device()
    a = gemm(d)
    b = gemm(d, w4.w4a16_linear)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


FULL = ([(2, i, K, N, M, False) for i, (_, K, N) in enumerate(workloads.LLAMA3_8B) for M in (512, 2048, 8192)]
        + [(3, i, K, N, 1024, True) for i, (_, K, N) in enumerate(workloads.LLAMA2_13B)]
        + [(4, i, K, N, M, False) for i, (_, K, N) in enumerate(workloads.LLAMA2_70B) for M in (64, 4096)])


@pytest.mark.parametrize("cfg,i,K,N,M,csr", FULL, ids=[f"c{c}_{K}x{N}_M{M}" for c, _, K, N, M, _ in FULL])
def test_gemm_full_shapes_sampled(orc, cfg, i, K, N, M, csr):
    c = Case(orc, seed=workloads.seed_of(cfg, i), K=K, N=N, M=M, csr=csr)
    y = host_bf16_as_f64(w4.w4a16_linear(**{k: v for k, v in c.device().items()}))
    w4.check_device_status()
    m, n = c.sample(seed=cfg * 10 + i)
    ref, ref_abs = c.reference_at(orc, m, n)
    check_close(y[m, n], ref, ref_abs, C_W_CSR if csr else C_W, depth(K), f"{K}x{N} M={M}")
