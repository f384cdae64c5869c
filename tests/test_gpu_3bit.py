"""3-bit codes on the GPU, against the oracle: the quantizer bit for bit (qweight3, scales,
zeros, s) and the decode GEMV within the GEMV's output bound, both schedules, with and without
a CSR term, several group sizes, and the Llama-3-8B gate/up shape sampled.
[SqueezeLLM article, sections 2.1-2.2: a dense part with eight levels once the outliers are
split off.]"""
import numpy as np
import pytest
import torch

import w4a16_gemm_awq_b200 as w4
import workloads
from parity import check_close, dev_bf16, dev_bits, dev_csr, host_bf16_as_f64, host_bits

pytestmark = pytest.mark.gpu


def _quantize3_both(orc, seed, N, K, gs, alpha=0.5, W=None):
    L = workloads.make_layer(seed, K=K, N=N)
    Wh = L.W if W is None else W
    ref = orc.awq_quantize3(Wh, L.act_absmean, alpha, gs)
    got = w4.awq_quantize3(torch.from_numpy(Wh).cuda(), torch.from_numpy(L.act_absmean).cuda(), alpha, gs)
    w4.check_device_status()
    return L, ref, got


def _xs_abs(x_bits, sc, gs, m_idx=None, n_idx=None):
    """sum_k |x[m][k]| * scale[n][k // gs]: the scale of the GEMV's per-group rounding error."""
    x = (x_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    M, K = x.shape
    xa = np.abs(x).reshape(M, K // gs, gs).sum(-1)
    scf = sc.view(np.float16).astype(np.float64).T
    if m_idx is None:
        return xa @ scf.T
    return np.einsum("pg,pg->p", xa[m_idx], scf[n_idx])


@pytest.mark.parametrize("K,N,gs", [(2048, 256, 128), (4096, 200, 128), (4096, 512, 256), (4096, 136, 512),
                                    (8192, 64, 1024), (4096, 4096, 128)])
def test_quantize3_bit_exact(orc, K, N, gs):
    _, (qw, sc, z, s), (gqw, gsc, gz, gs_) = _quantize3_both(orc, 3 * K + N + gs, N, K, gs)
    assert np.array_equal(host_bits(gqw, np.uint32), qw)
    assert np.array_equal(host_bits(gsc, np.uint16), sc)
    assert np.array_equal(host_bits(gz, np.uint32), z)
    assert np.array_equal(gs_.cpu().numpy(), s)
    assert int((host_bits(gz, np.uint32) & np.uint32(0x88888888)).max()) == 0  # zero points 0..7


def test_quantize3_closed_form_groups(orc):
    """w' = (i - z0) 2^-6 per group, i = 0..7 cycling: scale 2^-6, zero z0, codes i, exactly."""
    K, N = 1024, 64
    rng = np.random.default_rng(5)
    W = np.empty((N, K), np.float32)
    for n in range(N):
        for g in range(K // 128):
            z0 = int(rng.integers(0, 8))
            W[n, g * 128:(g + 1) * 128] = (np.arange(128) % 8 - z0) * 2.0 ** -6
    act = np.ones(K, np.float32)
    ref = orc.awq_quantize3(W, act, 0.0, 128)
    got = w4.awq_quantize3(torch.from_numpy(W).cuda(), torch.from_numpy(act).cuda(), 0.0, 128)
    w4.check_device_status()
    for a, b, t in zip(got[:3], ref[:3], (np.uint32, np.uint16, np.uint32)):
        assert np.array_equal(host_bits(a, t), b)
    assert np.array_equal(orc.dequant3(ref[0], ref[1], ref[2], N, K), W)


def test_quantize3_rejects_large_groups():
    W = torch.zeros(64, 4096, device="cuda")
    a = torch.ones(4096, device="cuda")
    with pytest.raises(w4.W4A16Error) as e:
        w4.awq_quantize3(W, a, 0.5, 2048)
    assert e.value.code == w4.ERR_SHAPE


@pytest.mark.parametrize("schedule", [w4.GEMV_STREAM_K, w4.GEMV_CLUSTER], ids=["stream_k", "cluster"])
@pytest.mark.parametrize("M", [1, 3, 8, 9, 16])
@pytest.mark.parametrize("csr", [False, True])
def test_gemv3_small_full_output(orc, M, schedule, csr):
    K, N, gs = 2048, 256, 128
    seed = 900 + M
    L = workloads.make_layer(seed, K=K, N=N)
    W, c = L.W, None
    if csr:
        Wd, rp, ci, v = orc.split_outliers(L.W, L.act_absmean, 0.5, workloads.outlier_nnz(N, K))
        W, c = Wd, (rp, ci, v)
    qw, sc, z, _ = orc.awq_quantize3(W, L.act_absmean, 0.5, gs)
    x = workloads.make_activations(seed, M, L.mult)
    y = w4.w3a16_gemv(dev_bf16(x), dev_bits(qw, torch.int32), dev_bits(sc, torch.int16), dev_bits(z, torch.int32),
                      csr=dev_csr(c) if c is not None else None, group_size=gs, schedule=schedule)
    w4.check_device_status()
    ref, ref_abs = orc.linear3(x, qw, sc, z, N, csr=c, with_abs=True, group_size=gs)
    check_close(host_bf16_as_f64(y), ref, ref_abs, 0.0, K // 128 + 64, f"gemv3 M={M} csr={csr}",
                _xs_abs(x, sc, gs))


@pytest.mark.parametrize("K,N,gs", [(4096, 512, 256), (4096, 256, 1024), (4096, 384, 4096)])
@pytest.mark.parametrize("M", [1, 12])
def test_gemv3_group_sizes(orc, K, N, gs, M):
    """Groups larger than one 128-slice: the GEMV reuses a group's scale over its slices (the
    quantizer takes up to 1024; larger groups come from the oracle)."""
    L = workloads.make_layer(K + N + gs, K=K, N=N)
    qw, sc, z, _ = orc.awq_quantize3(L.W, L.act_absmean, 0.5, gs)
    x = workloads.make_activations(K + N + gs, M, L.mult)
    y = w4.w3a16_gemv(dev_bf16(x), dev_bits(qw, torch.int32), dev_bits(sc, torch.int16), dev_bits(z, torch.int32),
                      group_size=gs)
    w4.check_device_status()
    ref, ref_abs = orc.linear3(x, qw, sc, z, N, with_abs=True, group_size=gs)
    check_close(host_bf16_as_f64(y), ref, ref_abs, 0.0, K // 128 + 64, f"gemv3 gs={gs} M={M}", _xs_abs(x, sc, gs))


def test_gemv3_repeatable_and_shape_checks(orc):
    K, N, M = 2048, 256, 5
    L, (qw, sc, z, _), (gqw, gsc, gz, _) = _quantize3_both(orc, 31, N, K, 128)
    x = dev_bf16(workloads.make_activations(31, M, L.mult))
    a = w4.w3a16_gemv(x, gqw, gsc, gz)
    b = w4.w3a16_gemv(x, gqw, gsc, gz)
    w4.check_device_status()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    with pytest.raises(ValueError):  # a 4-bit qweight shape is refused before the library
        w4.w3a16_gemv(x, torch.zeros(N, K // 8, dtype=torch.int32, device="cuda"), gsc, gz)
    x17 = dev_bf16(workloads.make_activations(31, 17, L.mult))
    with pytest.raises(w4.W4A16Error) as e:  # no 3-bit prefill GEMM
        w4.w3a16_gemv(x17, gqw, gsc, gz)
    assert e.value.code == w4.ERR_SHAPE


@pytest.mark.parametrize("M", [1, 16])
def test_gemv3_full_shape_sampled(orc, M):
    """The Llama-3-8B gate/up shape: GPU-quantized weights (checked bit for bit) into the GEMV,
    sampled outputs against the oracle."""
    K, N = 4096, 28672
    L, (qw, sc, z, _), (gqw, gsc, gz, _) = _quantize3_both(orc, 77, N, K, 128)
    assert np.array_equal(host_bits(gqw, np.uint32), qw)
    x = workloads.make_activations(77, M, L.mult)
    y = host_bf16_as_f64(w4.w3a16_gemv(dev_bf16(x), gqw, gsc, gz))
    w4.check_device_status()
    rng = np.random.default_rng(M)
    m = np.concatenate([rng.integers(0, M, 1536), np.zeros(N, np.int64)])
    n = np.concatenate([rng.integers(0, N, 1536), np.arange(N)])
    ref, ref_abs = orc.linear3_at(x, qw, sc, z, N, m, n, with_abs=True)
    check_close(y[m, n], ref, ref_abs, 0.0, K // 128 + 64, "gemv3 4096x28672", _xs_abs(x, sc, 128, m, n))
