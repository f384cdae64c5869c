"""GPU dense-and-sparse split (awq_split_outliers) against the oracle: the selection is an
index computation with a unique answer, so W_dense, row_ptr, col_idx and the fp16 values
must match bit for bit."""
import numpy as np
import pytest
import torch

import w4a16_gemm_awq_b200 as w4
import workloads
from parity import Case, check_close, dev_bf16, dev_bits, dev_f32, host_bf16_as_f64, host_bits

pytestmark = pytest.mark.gpu


def run_gpu(W, act, alpha, nnz):
    Wd, (rp, ci, v) = w4.awq_split_outliers(dev_f32(W), dev_f32(act), alpha, nnz)
    w4.check_device_status()
    return (Wd.cpu().numpy(), rp.cpu().numpy(), ci.cpu().numpy(), host_bits(v, np.uint16))


def assert_same(orc, W, act, alpha, nnz, what):
    g = run_gpu(W, act, alpha, nnz)
    r = orc.split_outliers(W, act, alpha, nnz)
    for name, a, b in zip(("W_dense", "row_ptr", "col_idx", "values"), g, r):
        a = np.asarray(a).reshape(-1)
        b = np.asarray(b).reshape(-1)
        assert a.shape == b.shape, f"{what}: {name} shape {a.shape} vs {b.shape}"
        diff = np.flatnonzero(a.view(np.uint32 if a.dtype.itemsize == 4 else np.uint16) !=
                              b.view(np.uint32 if b.dtype.itemsize == 4 else np.uint16))
        assert diff.size == 0, f"{what}: {name} differs at {diff.size} places, first {diff[:5].tolist()}"


@pytest.mark.parametrize("N,K,frac", [(64, 1024, 0.01), (200, 3072, 0.0045), (37, 1000, 0.05), (1, 4096, 0.1),
                                      (512, 128, 0.3), (29, 1001, 0.02), (70, 250, 0.1), (3, 7, 0.5)])
def test_split_random_bit_exact(orc, N, K, frac):
    """K % 4 != 0 (1001, 250, 7) runs the one-column-per-lane passes; the others
    the 128-bit passes, including K not a multiple of 128 (1000)."""
    L = workloads.make_layer(seed=N + K, K=K, N=N)
    assert_same(orc, L.W, L.act_absmean, workloads.ALPHA, int(np.floor(frac * N * K)), f"{N}x{K}")


def test_split_ties_broken_by_index(orc):
    """Scores drawn from a few values, so the threshold falls inside a large tie class."""
    rng = np.random.default_rng(5)
    N, K = 96, 2048
    W = rng.choice(np.array([-2.0, -1.0, 1.0, 2.0, 0.5], np.float32), size=(N, K))
    act = np.ones(K, np.float32)
    act[::7] = 2.0
    for nnz in (1, 100, 5000, 30000, N * K - 3):
        assert_same(orc, W, act, 0.5, nnz, f"ties nnz={nnz}")


def test_split_extremes(orc):
    L = workloads.make_layer(seed=9, K=1024, N=48)
    assert_same(orc, L.W, L.act_absmean, 0.5, 0, "nnz=0")
    assert_same(orc, L.W, L.act_absmean, 0.5, 48 * 1024, "nnz=N*K")
    W = L.W.copy()
    W[5, :] = 0.0
    act = L.act_absmean.copy()
    act[:10] = 0.0  # zero scores
    assert_same(orc, W, act, 0.25, 2000, "zeros")


def test_split_errors():
    W = torch.zeros(16, 256, device="cuda")
    a = torch.ones(256, device="cuda")
    with pytest.raises(w4.W4A16Error) as e:
        w4.awq_split_outliers(W, a, -1.0, 10)
    assert e.value.code == w4.ERR_VALUE
    with pytest.raises(w4.W4A16Error) as e:
        w4.awq_split_outliers(W, a, 0.5, 16 * 256 + 1)
    assert e.value.code == w4.ERR_SHAPE
    with pytest.raises(w4.W4A16Error) as e:
        w4.awq_split_outliers(W, a, 0.5, 10, workspace=torch.empty(256, dtype=torch.uint8, device="cuda"))
    assert e.value.code == w4.ERR_SHAPE
    W[3, 7] = float("nan")
    w4.awq_split_outliers(W, a, 0.5, 10)
    with pytest.raises(w4.W4A16Error) as e:
        w4.check_device_status()
    assert e.value.code == w4.ERR_VALUE
    w4.check_device_status()


SPLIT_SHAPES = [(i, K, N) for i, (_, K, N) in enumerate(workloads.DENSE_SPARSE_13B["shapes"])]


@pytest.mark.parametrize("i,K,N", SPLIT_SHAPES, ids=[f"{K}x{N}" for _, K, N in SPLIT_SHAPES])
def test_split_full_config3_bit_exact(orc, i, K, N):
    """The dense-and-sparse layers (Llama-2-13B shapes, 0.45% outliers) at full size."""
    L = workloads.make_layer(workloads.seed_of(3, i), K=K, N=N)
    assert_same(orc, L.W, L.act_absmean, workloads.ALPHA, workloads.outlier_nnz(N, K), f"{K}x{N}")


def test_split_then_quantize_then_linear(orc):
    """The whole dense-and-sparse path on the GPU (split, quantize W_dense, GEMV and GEMM with
    the CSR) against the oracle's own split, quantize and product."""
    K, N = 2048, 384
    L = workloads.make_layer(seed=123, K=K, N=N)
    nnz = workloads.outlier_nnz(N, K)
    Wd, csr = w4.awq_split_outliers(dev_f32(L.W), dev_f32(L.act_absmean), workloads.ALPHA, nnz)
    qw, sc, z, _ = w4.awq_quantize_g128(Wd, dev_f32(L.act_absmean), workloads.ALPHA)
    w4.check_device_status()
    Wd_o, rp_o, ci_o, v_o = orc.split_outliers(L.W, L.act_absmean, workloads.ALPHA, nnz)
    qw_o, sc_o, z_o, _ = orc.awq_quantize_g128(Wd_o, L.act_absmean, workloads.ALPHA)
    assert np.array_equal(host_bits(qw, np.uint32), qw_o)
    for M, fn in ((4, w4.w4a16_gemv), (300, w4.w4a16_gemm)):
        x = workloads.make_activations(7, M, L.mult)
        y = host_bf16_as_f64(fn(dev_bf16(x), qw, sc, z, csr=csr))
        w4.check_device_status()
        ref, ref_abs = orc.linear(x, qw_o, sc_o, z_o, N, csr=(rp_o, ci_o, v_o), with_abs=True)
        rel = np.abs(y - ref).max(axis=1) / np.abs(ref).max(axis=1)
        assert rel.max() <= 1e-2, (M, rel.max())
