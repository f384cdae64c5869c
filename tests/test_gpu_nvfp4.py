"""The NVFP4 quantizer on the GPU against the oracle, bit for bit: E2M1 codes, E4M3 block
scales, the fp32 tensor scale and s, on small, ragged and full layer shapes, plus the all-zero
and non-finite cases.  [DeepCompressor README: FP4_E2M1 and NVFP4.]"""
import numpy as np
import pytest
import torch

import w4a16_gemm_awq_b200 as w4
import workloads
from parity import host_bits

pytestmark = pytest.mark.gpu


def _both(orc, W, act, alpha=0.5):
    ref = orc.awq_quantize_nvfp4(W, act, alpha)
    got = w4.awq_quantize_nvfp4(torch.from_numpy(W).cuda(), torch.from_numpy(act).cuda(), alpha)
    w4.check_device_status()
    return ref, got


@pytest.mark.parametrize("N,K", [(8, 64), (256, 2048), (200, 1024), (72, 5120), (4096, 4096)])
def test_nvfp4_quantize_bit_exact(orc, N, K):
    L = workloads.make_layer(5 * N + K, K=K, N=N)
    (qw, sc, g, s), (gqw, gsc, gg, gs) = _both(orc, L.W, L.act_absmean)
    assert float(gg.item()) == g
    assert np.array_equal(gs.cpu().numpy(), s)
    assert np.array_equal(gsc.cpu().numpy(), sc)
    assert np.array_equal(host_bits(gqw, np.uint32), qw)


def test_nvfp4_wide_range_and_ties(orc):
    """Weights spread over many binades and values placed on E2M1 midpoints of their block."""
    rng = np.random.default_rng(11)
    N, K = 64, 512
    W = (rng.standard_normal((N, K)) * 2.0 ** rng.integers(-20, 20, (N, 1))).astype(np.float32)
    W[:, 16:32] = np.array([6, 5, 3.5, 2.5, 1.75, 1.25, 0.75, 0.25, -5, -3.5, -2.5, -1.75, -1.25, -0.75, -0.25, 0],
                           np.float32)[None, :]
    (qw, sc, g, _), (gqw, gsc, gg, _) = _both(orc, W, np.ones(K, np.float32), 0.0)
    assert float(gg.item()) == g
    assert np.array_equal(gsc.cpu().numpy(), sc)
    assert np.array_equal(host_bits(gqw, np.uint32), qw)


def test_nvfp4_all_zero(orc):
    W = np.zeros((16, 256), np.float32)
    (qw, sc, g, _), (gqw, gsc, gg, _) = _both(orc, W, np.ones(256, np.float32))
    assert g == 1.0 and float(gg.item()) == 1.0
    assert not gsc.cpu().numpy().any() and not host_bits(gqw, np.uint32).any()


def test_nvfp4_reports_non_finite_and_bad_shapes():
    W = torch.zeros(16, 256, device="cuda")
    W[3, 7] = float("inf")
    w4.awq_quantize_nvfp4(W, torch.ones(256, device="cuda"), 0.5)
    with pytest.raises(w4.W4A16Error) as e:
        w4.check_device_status()
    assert e.value.code == w4.ERR_VALUE
    with pytest.raises(w4.W4A16Error) as e:
        w4.awq_quantize_nvfp4(torch.zeros(16, 40, device="cuda"), torch.ones(40, device="cuda"), 0.5)
    assert e.value.code == w4.ERR_SHAPE


@pytest.mark.parametrize("M", [1, 5, 8, 9, 16])
@pytest.mark.parametrize("N,K", [(256, 2048), (48, 1040)])
def test_nvfp4_gemv_full_output(orc, N, K, M):
    """The decode product on GPU-quantized weights (checked bit for bit against the oracle's)
    against the oracle's double-precision product, within the GEMV's output bound: the
    weights are exact, only fp32 sums round (16-term MMA blocks, then K/16 block sums)."""
    from parity import check_close, dev_bf16, host_bf16_as_f64
    L = workloads.make_layer(3 * N + K + M, K=K, N=N)
    (qw, sc, g, _), (gqw, gsc, gg, _) = _both(orc, L.W, L.act_absmean)
    assert np.array_equal(host_bits(gqw, np.uint32), qw) and np.array_equal(gsc.cpu().numpy(), sc)
    x = workloads.make_activations(3 * N + K + M, M, L.mult)
    y = w4.w4a16_gemv_nvfp4(dev_bf16(x), gqw, gsc, gg)
    w4.check_device_status()
    ref, ref_abs = orc.linear_nvfp4(x, qw, sc, g, N, with_abs=True)
    check_close(host_bf16_as_f64(y), ref, ref_abs, 0.0, K // 16 + 64, f"nvfp4 gemv M={M}")
    y2 = w4.w4a16_gemv_nvfp4(dev_bf16(x), gqw, gsc, gg)
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))


def test_nvfp4_gemv_full_shape(orc):
    """4096 x 4096 at M = 16, every output."""
    from parity import check_close, dev_bf16, host_bf16_as_f64
    K, N, M = 4096, 4096, 16
    L = workloads.make_layer(808, K=K, N=N)
    (qw, sc, g, _), (gqw, gsc, gg, _) = _both(orc, L.W, L.act_absmean)
    x = workloads.make_activations(808, M, L.mult)
    y = w4.w4a16_gemv_nvfp4(dev_bf16(x), gqw, gsc, gg)
    w4.check_device_status()
    ref, ref_abs = orc.linear_nvfp4(x, qw, sc, g, N, with_abs=True)
    check_close(host_bf16_as_f64(y), ref, ref_abs, 0.0, K // 16 + 64, "nvfp4 gemv 4096x4096")


def test_nvfp4_gemv_shape_checks():
    x = torch.zeros(17, 256, dtype=torch.bfloat16, device="cuda")
    qw = torch.zeros(32, 32, dtype=torch.int32, device="cuda")
    sc = torch.zeros(16, 32, dtype=torch.uint8, device="cuda")
    g = torch.ones(1, device="cuda")
    with pytest.raises(w4.W4A16Error) as e:
        w4.w4a16_gemv_nvfp4(x, qw, sc, g)
    assert e.value.code == w4.ERR_SHAPE
    with pytest.raises(ValueError):
        w4.w4a16_gemv_nvfp4(x[:4], qw[:, :16], sc, g)
