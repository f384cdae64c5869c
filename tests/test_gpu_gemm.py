"""GPU tcgen05 GEMM against the oracle: token tails, every tile width, split-K (the small
layers here with M <= 128 split K over several CTAs per tile, as do the long-K cases) and the
unsplit path, the CSR term in fp32, exact-weight cases with a tight bound, and the full
prefill shapes (sampled)."""
import numpy as np
import pytest
import torch

import w4a16_gemm_awq_b200 as w4
import workloads
from parity import Case, check_close, dev_bf16, dev_bits, dev_csr, host_bf16_as_f64

pytestmark = pytest.mark.gpu

C_W = 2.0 ** -8 * 1.01   # bf16 scale and bf16 product: the weights' relative error on the MMA


def gemm(d, fn=None, workspace=None):
    fn = fn or w4.w4a16_gemm
    y = fn(d["x"], d["qweight"], d["scales"], d["zeros"], csr=d["csr"], workspace=workspace)
    w4.check_device_status()
    return y


def no_workspace():
    """A NULL workspace: the GEMM then runs one CTA per output tile (no split-K)."""
    return torch.empty(0, dtype=torch.uint8, device="cuda")


def depth(K):
    return K // 16 + 64


@pytest.mark.parametrize("M", [1, 16, 17, 32, 33, 64, 100, 128, 129, 200, 256, 300, 640])
def test_gemm_small_full_output(orc, M):
    c = Case(orc, seed=200 + M, K=2048, N=256, M=M)
    y = host_bf16_as_f64(gemm(c.device()))
    ref, ref_abs = c.reference(orc)
    check_close(y, ref, ref_abs, C_W, depth(c.K), f"M={M}")


@pytest.mark.parametrize("M", [17, 100, 300])
def test_gemm_without_workspace_does_not_split(orc, M):
    c = Case(orc, seed=250 + M, K=2048, N=256, M=M)
    y = host_bf16_as_f64(gemm(c.device(), workspace=no_workspace()))
    ref, ref_abs = c.reference(orc)
    check_close(y, ref, ref_abs, C_W, depth(c.K), f"M={M} unsplit")


@pytest.mark.parametrize("M", [3, 70, 257])
def test_gemm_small_with_csr(orc, M):
    """The sparse term is added in fp32 before the one rounding: only the dense weights carry
    the bf16 error C_W."""
    c = Case(orc, seed=300 + M, K=2048, N=384, M=M, csr=True)
    y = host_bf16_as_f64(gemm(c.device()))
    ref, ref_abs = c.reference(orc)
    check_close(y, ref, ref_abs, C_W, depth(c.K), f"M={M} csr")


@pytest.mark.parametrize("M", [20, 300])
def test_gemm_csr_only_and_dense_rows(orc, M):
    """All-zero dense part, so every output is the fp32 sparse term rounded once: one CSR row
    fully dense, others empty or single."""
    K, N = 1024, 128
    qw, sc, z, _ = orc.awq_quantize_g128(np.zeros((N, K), np.float32), np.ones(K, np.float32), 0.0)
    rng = np.random.default_rng(M)
    rows = [np.arange(K) if n == 5 else (np.array([n * 7 % K]) if n % 3 == 0 else np.array([], np.int64))
            for n in range(N)]
    rp = np.concatenate([[0], np.cumsum([len(r) for r in rows])]).astype(np.int32)
    ci = np.concatenate(rows).astype(np.int32)
    v = rng.standard_normal(ci.size).astype(np.float16).view(np.uint16)
    x = workloads.uniform_bf16(M + 1, (M, K))
    d = dict(x=dev_bf16(x), qweight=dev_bits(qw, torch.int32), scales=dev_bits(sc, torch.int16),
             zeros=dev_bits(z, torch.int32), csr=dev_csr((rp, ci, v)))
    y = host_bf16_as_f64(gemm(d))
    ref, ref_abs = orc.linear(x, qw, sc, z, N, csr=(rp, ci, v), with_abs=True)
    check_close(y, ref, ref_abs, 0.0, K + 64, f"csr only M={M}")


def test_gemm_csr_needs_a_workspace(orc):
    c = Case(orc, seed=23, K=1024, N=128, M=40, csr=True)
    d = c.device()
    with pytest.raises(w4.W4A16Error) as e:
        gemm(d, workspace=no_workspace())
    assert e.value.code == w4.ERR_NULL
    need = w4.workspace_bytes(40, 128, 1024, csr=True)
    with pytest.raises(w4.W4A16Error) as e:
        gemm(d, workspace=torch.zeros(need - 256, dtype=torch.uint8, device="cuda"))
    assert e.value.code == w4.ERR_SHAPE


def test_gemm_split_k_is_deterministic_and_leaves_counters_zero(orc):
    """A small grid with a long K: the plan splits K over 8 CTAs per tile.  Repeated calls give
    the same bits, the counters are zero again afterwards, and the result is within the bound
    of the unsplit one."""
    c = Case(orc, seed=29, K=8192, N=256, M=64)
    d = c.device()
    ws = torch.zeros(w4.workspace_bytes(64, 256, 8192, csr=False), dtype=torch.uint8, device="cuda")
    a = gemm(d, workspace=ws)
    b = gemm(d, workspace=ws)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert int(ws[:128 * 1024].count_nonzero()) == 0
    ref, ref_abs = c.reference(orc)
    check_close(host_bf16_as_f64(a), ref, ref_abs, C_W, depth(c.K), "split-K")
    u = gemm(d, workspace=no_workspace())
    check_close(host_bf16_as_f64(u), ref, ref_abs, C_W, depth(c.K), "unsplit")


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


@pytest.mark.parametrize("M,K", [(40, 2048), (256, 2048), (513, 2048), (64, 8192), (300, 8192)])
def test_gemm_exact_weights_tight(orc, M, K):
    """When every dequantized weight is exact in bf16, only accumulation and the output rounding
    remain: a misplaced k, token, channel or split fails the per-element bound."""
    N = 256
    W = _exact_layer(M, N, K)
    qw, sc, z, _ = orc.awq_quantize_g128(W, np.ones(K, np.float32), 0.0)
    x = workloads.uniform_bf16(M, (M, K), -3, 3)
    d = dict(x=dev_bf16(x), qweight=dev_bits(qw, torch.int32), scales=dev_bits(sc, torch.int16),
             zeros=dev_bits(z, torch.int32), csr=None)
    y = host_bf16_as_f64(gemm(d))
    ref, ref_abs = orc.linear(x, qw, sc, z, N, with_abs=True)
    assert np.array_equal(orc.dequant(qw, sc, z, N, K), W)
    check_close(y, ref, ref_abs, 0.0, depth(K), f"exact M={M}")


@pytest.mark.parametrize("M", [40, 300])
def test_gemm_empty_csr_is_bit_identical(orc, M):
    c = Case(orc, seed=17, K=2048, N=256, M=M)
    d = c.device()
    y0 = gemm(d)
    d["csr"] = (torch.zeros(c.N + 1, dtype=torch.int32, device="cuda"), torch.zeros(0, dtype=torch.int32, device="cuda"),
                torch.zeros(0, dtype=torch.int16, device="cuda"))
    y1 = gemm(d)
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))


def test_gemm_reports_bad_csr_column(orc):
    c = Case(orc, seed=19, K=1024, N=128, M=64)
    d = c.device()
    rp = torch.zeros(c.N + 1, dtype=torch.int32, device="cuda")
    rp[1:] = 2
    d["csr"] = (rp, torch.tensor([600, c.K + 5], dtype=torch.int32, device="cuda"),
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
    check_close(y[m, n], ref, ref_abs, C_W, depth(K), f"{K}x{N} M={M}")
