"""The decode GEMV on raw activations with the 1/s fold in the same call (w4a16_gemv_folded).

x' = bf16(x / s) is what the linear entry points take [AWQ translation, section 3.2: the
weights are multiplied by s and the activations divided by it].  The folded call divides x
once into its workspace and runs the GEMV on the result; it must give the same bits as
awq_fold_activations followed by the GEMV (same conversions, same arithmetic afterwards), and
the oracle's result for the folded activations within the tolerance of the unfused GEMV."""
import numpy as np
import pytest
import torch

import w4a16_gemm_awq_b200 as w4
import workloads
from parity import check_close, dev_bf16, dev_bits, dev_csr, dev_f32, host_bf16_as_f64, host_bits, xs_abs

pytestmark = pytest.mark.gpu

ALPHA = 0.5


def _layer(orc, seed, K, N, M, csr, gs=128):
    """Raw activations x (before the fold), the oracle's quantized layer and its scales s."""
    L = workloads.make_layer(seed, K=K, N=N)
    W, c = L.W, None
    if csr:
        Wd, rp, ci, v = orc.split_outliers(W, L.act_absmean, ALPHA, workloads.outlier_nnz(N, K))
        W, c = Wd, (rp, ci, v)
    qw, sc, z, s = orc.awq_quantize(W, L.act_absmean, ALPHA, gs)
    x = workloads.make_activations(seed, M, L.mult, alpha=0.0)
    return x, qw, sc, z, s, c


def _dev(qw, sc, z, c):
    return (dev_bits(qw, torch.int32), dev_bits(sc, torch.int16), dev_bits(z, torch.int32),
            dev_csr(c) if c is not None else None)


def _oracle_fold(orc, x, s):
    """bf16(x / s): fp32 IEEE division (numpy), then the oracle's bf16 rounding."""
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    q = xf / s[None, :].astype(np.float32)
    assert q.dtype == np.float32
    return np.vectorize(orc.f32_to_bf16_bits, otypes=[np.uint16])(q)


@pytest.mark.parametrize("schedule", [w4.GEMV_STREAM_K, w4.GEMV_CLUSTER], ids=["stream_k", "cluster"])
@pytest.mark.parametrize("M", [1, 7, 16])
@pytest.mark.parametrize("K,N,csr", [(4096, 384, True), (2048, 256, False)])
def test_folded_equals_fold_then_gemv(orc, K, N, csr, M, schedule):
    x, qw, sc, z, s, c = _layer(orc, 3 * K + N + M, K, N, M, csr)
    dqw, dsc, dz, dc = _dev(qw, sc, z, c)
    xd, sd = dev_bf16(x), dev_f32(s)
    y = w4.w4a16_gemv_folded(xd, sd, dqw, dsc, dz, csr=dc, schedule=schedule)
    xp = w4.awq_fold_activations(xd, sd)
    y2 = w4.w4a16_gemv_ex(xp, dqw, dsc, dz, csr=dc, schedule=schedule)
    w4.check_device_status()
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))


@pytest.mark.parametrize("M", [1, 5, 16])
def test_folded_matches_oracle(orc, M):
    K, N = 4096, 256
    x, qw, sc, z, s, c = _layer(orc, 500 + M, K, N, M, True)
    dqw, dsc, dz, dc = _dev(qw, sc, z, c)
    y = w4.w4a16_gemv_folded(dev_bf16(x), dev_f32(s), dqw, dsc, dz, csr=dc)
    w4.check_device_status()
    xp = _oracle_fold(orc, x, s)
    ref, ref_abs = orc.linear(xp, qw, sc, z, N, csr=c, with_abs=True)
    check_close(host_bf16_as_f64(y), ref, ref_abs, 0.0, K // 128 + 64, f"folded M={M}", xs_abs(xp, sc))


@pytest.mark.parametrize("schedule", [w4.GEMV_STREAM_K, w4.GEMV_CLUSTER], ids=["stream_k", "cluster"])
@pytest.mark.parametrize("gs", [512, 4096])
def test_folded_groups(orc, gs, schedule):
    K, N, M = 4096, 256, 9
    x, qw, sc, z, s, c = _layer(orc, 900 + gs, K, N, M, False, gs)
    dqw, dsc, dz, _ = _dev(qw, sc, z, c)
    xd, sd = dev_bf16(x), dev_f32(s)
    y = w4.w4a16_gemv_folded(xd, sd, dqw, dsc, dz, group_size=gs, schedule=schedule)
    y2 = w4.w4a16_linear_ex(w4.awq_fold_activations(xd, sd), dqw, dsc, dz, group_size=gs, schedule=schedule)
    w4.check_device_status()
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))


def test_folded_without_s_is_the_plain_gemv(orc):
    K, N, M = 2048, 256, 3
    x, qw, sc, z, s, c = _layer(orc, 77, K, N, M, True)
    dqw, dsc, dz, dc = _dev(qw, sc, z, c)
    xp = w4.awq_fold_activations(dev_bf16(x), dev_f32(s))
    y = w4.w4a16_gemv_folded(xp, None, dqw, dsc, dz, csr=dc)
    y2 = w4.w4a16_gemv(xp, dqw, dsc, dz, csr=dc)
    w4.check_device_status()
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))


def test_folded_full_shape_sampled(orc):
    """The Llama-3-8B down_proj shape (K = 14336) at M = 16, sampled outputs."""
    K, N, M = 14336, 4096, 16
    x, qw, sc, z, s, c = _layer(orc, 4242, K, N, M, False)
    dqw, dsc, dz, _ = _dev(qw, sc, z, c)
    y = host_bf16_as_f64(w4.w4a16_gemv_folded(dev_bf16(x), dev_f32(s), dqw, dsc, dz))
    w4.check_device_status()
    xp = _oracle_fold(orc, x, s)
    rng = np.random.default_rng(5)
    m_idx = np.concatenate([rng.integers(0, M, 1024), np.zeros(N, np.int64)])
    n_idx = np.concatenate([rng.integers(0, N, 1024), np.arange(N)])
    ref, ref_abs = orc.linear_at(xp, qw, sc, z, N, m_idx, n_idx, with_abs=True)
    check_close(y[m_idx, n_idx], ref, ref_abs, 0.0, K // 128 + 64, "folded 14336x4096",
                xs_abs(xp, sc, m_idx, n_idx))


def test_folded_argument_errors():
    K, N = 1024, 128
    x = torch.zeros(2, K, dtype=torch.bfloat16, device="cuda")
    qw = torch.zeros(N, K // 8, dtype=torch.int32, device="cuda")
    sc = torch.zeros(K // 128, N, dtype=torch.int16, device="cuda")
    z = torch.zeros(K // 128, N // 8, dtype=torch.int32, device="cuda")
    buf = torch.ones(K + 4, dtype=torch.float32, device="cuda")
    with pytest.raises(w4.W4A16Error) as e:
        w4.w4a16_gemv_folded(x, buf[1:K + 1], qw, sc, z)
    assert e.value.code == w4.ERR_ALIGN
    with pytest.raises(ValueError):
        w4.w4a16_gemv_folded(x, buf[:K - 4], qw, sc, z)
    with pytest.raises(w4.W4A16Error) as e:
        w4.w4a16_gemv_folded(torch.zeros(17, K, dtype=torch.bfloat16, device="cuda"), buf[:K], qw, sc, z)
    assert e.value.code == w4.ERR_SHAPE


@pytest.mark.parametrize("schedule", [w4.GEMV_STREAM_K, w4.GEMV_CLUSTER], ids=["stream_k", "cluster"])
def test_folded_quotients_near_bf16_midpoints(orc, schedule):
    """Scales chosen so that x / s falls on or next to a bf16 rounding midpoint for token 0
    (ties included), exact quotients (powers of two), huge and tiny scales, zeros, -0 and
    subnormal activations: where any shortcut in the conversion would show.  The fused call
    must still match the separate fold bit for bit, and the fold the oracle's conversion."""
    K, N, M = 2048, 256, 16
    rng = np.random.default_rng(2024)
    x = workloads.make_activations(17, M, np.ones(K, np.float32), alpha=0.0)
    x0 = (x[0].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    # a midpoint between two bf16 values: 9 significant bits with the last one set
    mid = (rng.integers(256, 512, K) * 2 + 1).astype(np.float64) * 2.0 ** rng.integers(-20, 10, K).astype(np.float64)
    s = (np.abs(x0) / mid).astype(np.float32)
    s *= (1 + rng.integers(-4, 5, K) * 2.0 ** -23).astype(np.float32)      # a few ulp either side
    s[0::16] = np.float32(2.0) ** rng.integers(-10, 10, K // 16)            # exact quotients
    s[1::64] = np.float32(3e30)                                             # huge: IEEE path
    s[2::64] = np.float32(2e-38)                                            # tiny: IEEE path
    s[s == 0] = 1.0
    xb = x.copy()
    xb[1, 0::8] = 0                                                         # zeros
    xb[2, 0::8] = 0x0001                                                    # subnormal bf16
    xb[3, 0::8] = 0x8000                                                    # -0
    L = workloads.make_layer(88, K=K, N=N)
    qw, sc, z, _ = orc.awq_quantize(L.W, L.act_absmean, ALPHA, 128)
    dqw, dsc, dz, _ = _dev(qw, sc, z, None)
    xd, sd = dev_bf16(xb), dev_f32(s)
    y = w4.w4a16_gemv_folded(xd, sd, dqw, dsc, dz, schedule=schedule)
    xp = w4.awq_fold_activations(xd, sd)
    y2 = w4.w4a16_gemv_ex(xp, dqw, dsc, dz, schedule=schedule)
    w4.check_device_status()
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
    # and the separate fold is the oracle's conversion, value for value
    assert np.array_equal(host_bits(xp.view(torch.int16), np.uint16), _oracle_fold(orc, xb, s))
