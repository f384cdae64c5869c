"""Group sizes other than 128 (up to one group per row) on the GPU, against the oracle:
quantize bit for bit, the decode GEMV (both schedules) and the tcgen05 GEMM within the
output tolerance.  [SqueezeLLM article, section 4.1: the group size option.]"""
import numpy as np
import pytest
import torch

import w4a16_gemm_awq_b200 as w4
import workloads
from parity import GEMV_XS_COEF, check_close, dev_bf16, dev_bits, host_bf16_as_f64, host_bits

pytestmark = pytest.mark.gpu


def _quantize_both(orc, seed, N, K, gs, alpha=0.5):
    L = workloads.make_layer(seed, K=K, N=N)
    ref = orc.awq_quantize(L.W, L.act_absmean, alpha, gs)
    W = torch.from_numpy(L.W).cuda()
    act = torch.from_numpy(L.act_absmean).cuda()
    got = w4.awq_quantize(W, act, alpha, gs)
    w4.check_device_status()
    return L, ref, got


@pytest.mark.parametrize("K,N,gs", [(4096, 512, 256), (4096, 512, 512), (4096, 200, 1024), (4096, 136, 2048),
                                    (4096, 512, 4096), (5120, 72, 5120), (28672, 64, 28672), (14336, 48, 7168)])
def test_quantize_groups_bit_exact(orc, K, N, gs):
    _, (qw, sc, z, s), (gqw, gsc, gz, gs_) = _quantize_both(orc, K + N + gs, N, K, gs)
    assert np.array_equal(host_bits(gqw, np.uint32), qw)
    assert np.array_equal(host_bits(gsc, np.uint16), sc)
    assert np.array_equal(host_bits(gz, np.uint32), z)
    assert np.array_equal(gs_.cpu().numpy(), s)


def _xs_abs(x_bits, sc, gs, m_idx=None, n_idx=None):
    """sum_k |x[m][k]| * scale[n][k // gs]: the scale of the GEMV's per-group rounding error."""
    x = (x_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    M, K = x.shape
    xa = np.abs(x).reshape(M, K // gs, gs).sum(-1)
    scf = sc.view(np.float16).astype(np.float64).T
    if m_idx is None:
        return xa @ scf.T
    return np.einsum("pg,pg->p", xa[m_idx], scf[n_idx])


CASES = [(4096, 512, 256), (4096, 256, 1024), (4096, 384, 4096), (5120, 256, 5120)]


@pytest.mark.parametrize("schedule", [w4.GEMV_STREAM_K, w4.GEMV_CLUSTER], ids=["stream_k", "cluster"])
@pytest.mark.parametrize("M", [1, 9])
@pytest.mark.parametrize("K,N,gs", CASES)
def test_gemv_groups(orc, K, N, gs, M, schedule):
    L, (qw, sc, z, s), _ = _quantize_both(orc, 7 * K + N, N, K, gs)
    x = workloads.make_activations(7 * K + N, M, L.mult)
    y = w4.w4a16_linear_ex(dev_bf16(x), dev_bits(qw, torch.int32), dev_bits(sc, torch.int16),
                           dev_bits(z, torch.int32), group_size=gs, schedule=schedule)
    w4.check_device_status()
    ref, ref_abs = orc.linear(x, qw, sc, z, N, with_abs=True, group_size=gs)
    check_close(host_bf16_as_f64(y), ref, ref_abs, 0.0, K // 128 + 64, f"gemv gs={gs} M={M}",
                _xs_abs(x, sc, gs))


@pytest.mark.parametrize("M", [40, 300])
@pytest.mark.parametrize("K,N,gs", CASES)
def test_gemm_groups(orc, K, N, gs, M):
    L, (qw, sc, z, s), _ = _quantize_both(orc, 11 * K + N, N, K, gs)
    x = workloads.make_activations(11 * K + N, M, L.mult)
    y = w4.w4a16_linear_ex(dev_bf16(x), dev_bits(qw, torch.int32), dev_bits(sc, torch.int16),
                           dev_bits(z, torch.int32), group_size=gs)
    w4.check_device_status()
    ref, ref_abs = orc.linear(x, qw, sc, z, N, with_abs=True, group_size=gs)
    # the GEMM rounds each dequantized weight to bf16 before the tensor cores
    check_close(host_bf16_as_f64(y), ref, ref_abs, 2.0 ** -8 * 1.01, K // 16 + 64, f"gemm gs={gs} M={M}")


@pytest.mark.parametrize("M", [4, 64])
def test_per_row_groups_full_shape_sampled(orc, M):
    """One group per row on the Llama-3-8B gate/up shape, sampled outputs."""
    K, N = 4096, 28672
    L, (qw, sc, z, s), (gqw, gsc, gz, _) = _quantize_both(orc, 123, N, K, K)
    assert np.array_equal(host_bits(gqw, np.uint32), qw)
    x = workloads.make_activations(123, M, L.mult)
    y = host_bf16_as_f64(w4.w4a16_linear_ex(dev_bf16(x), gqw, gsc, gz, group_size=K))
    w4.check_device_status()
    rng = np.random.default_rng(M)
    m = np.concatenate([rng.integers(0, M, 1536), np.zeros(N, np.int64)])
    n = np.concatenate([rng.integers(0, N, 1536), np.arange(N)])
    ref, ref_abs = orc.linear_at(x, qw, sc, z, N, m, n, with_abs=True, group_size=K)
    if M <= 16:
        check_close(y[m, n], ref, ref_abs, 0.0, K // 128 + 64, "per-row gemv", _xs_abs(x, sc, K, m, n))
    else:
        check_close(y[m, n], ref, ref_abs, 2.0 ** -8 * 1.01, K // 16 + 64, "per-row gemm")
