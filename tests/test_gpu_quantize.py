"""GPU awq_quantize_g128 against the oracle: qweight, scales, zeros and s must be bit-exact."""
import numpy as np
import pytest
import torch

import w4a16_gemm_awq_b200 as w4
import workloads
from parity import dev_f32, host_bits

pytestmark = pytest.mark.gpu


def run_gpu(W, act, alpha):
    qw, sc, z, s = w4.awq_quantize_g128(dev_f32(W), dev_f32(act), alpha)
    w4.check_device_status()
    return (host_bits(qw, np.uint32), host_bits(sc, np.uint16), host_bits(z, np.uint32),
            s.cpu().numpy())


def assert_same(orc, W, act, alpha, what=""):
    got = run_gpu(W, act, alpha)
    want = orc.awq_quantize_g128(W, act, alpha)
    for name, g, r in zip(("qweight", "scales", "zeros", "s"), got, want):
        if name == "s":
            assert np.array_equal(g.view(np.uint32), r.view(np.uint32)), f"{what}: s differs"
        else:
            diff = np.argwhere(g != r)
            assert diff.size == 0, f"{what}: {name} differs at {len(diff)} places, first {diff[:3].tolist()}"


@pytest.mark.parametrize("N,K,alpha", [(128, 1024, 0.5), (64, 2048, 0.5), (256, 4096, 0.25), (192, 1024, 0.0),
                                       (8, 1024, 1.0), (104, 3072, 0.5), (200, 2048, 0.5)])
def test_quantize_small_bit_exact(orc, N, K, alpha):
    L = workloads.make_layer(seed=N * 7 + K, K=K, N=N)
    assert_same(orc, L.W, L.act_absmean, alpha, f"{N}x{K}")


def test_quantize_wide_dynamic_range(orc):
    """Rows spanning many binades, all-zero groups, same-sign groups, exact ties."""
    rng = np.random.default_rng(31)
    N, K = 96, 2048
    W = (rng.standard_normal((N, K)) * np.exp(rng.uniform(-12, 6, (N, 1)))).astype(np.float32)
    W[3, :] = 0.0
    W[5, 128:256] = np.abs(W[5, 128:256]) + 1.0
    W[7, 256:384] = -np.abs(W[7, 256:384]) - 1.0
    i = np.arange(128) % 16
    W[9, 0:128] = ((i - 5) * 2.0 ** -6).astype(np.float32)
    W[9, 0:4] = np.array([0.5, 1.5, -0.5, 2.5], np.float32) * np.float32(2.0 ** -6)
    act = np.exp(rng.standard_normal(K) * 2).astype(np.float32)
    act[:16] = 0.0  # s floors at 1e-4
    assert_same(orc, W, act, 0.5, "wide range")


def test_quantize_closed_form_on_gpu(orc):
    K = 1024
    i = np.arange(K) % 16
    W = ((i - 5) * 2.0 ** -6).astype(np.float32)[None, :].repeat(8, 0)
    qw, sc, z, s = run_gpu(W, np.ones(K, np.float32), 0.0)
    assert np.all(sc == 0x2400)
    assert np.all(z == 0x55555555)  # zero point 5 in the nibbles of all 8 rows


def test_quantize_reports_bad_values():
    K = 1024
    W = torch.zeros(128, K, device="cuda")
    W[3, 5] = float("nan")
    w4.awq_quantize_g128(W, torch.ones(K, device="cuda"), 0.5)
    with pytest.raises(w4.W4A16Error) as e:
        w4.check_device_status()
    assert e.value.code == w4.ERR_VALUE
    act = -torch.ones(K, device="cuda")
    w4.awq_quantize_g128(torch.zeros(128, K, device="cuda"), act, 0.5)
    with pytest.raises(w4.W4A16Error) as e:
        w4.check_device_status()
    assert e.value.code == w4.ERR_VALUE
    w4.check_device_status()  # cleared


ALL_SHAPES = [(w["family"], i, K, N) for w in (workloads.DECODE_SWEEP, workloads.LARGE_LAYERS_70B)
              for i, (_, K, N) in enumerate(w["shapes"])]


@pytest.mark.parametrize("cfg,i,K,N", ALL_SHAPES, ids=[f"c{c}_{K}x{N}" for c, _, K, N in ALL_SHAPES])
def test_quantize_full_shapes_bit_exact(orc, cfg, i, K, N):
    """The eight layer shapes (Llama-3-8B and 70B) at full size, packing bit-exact."""
    L = workloads.make_layer(workloads.seed_of(cfg, i), K=K, N=N)
    assert_same(orc, L.W, L.act_absmean, workloads.ALPHA, f"{K}x{N}")


def test_quantizer_division_matches_ieee_everywhere():
    """The quantizer divides each weight by its group's fp16 scale with Markstein's correction
    of w' * RN(1/sf) instead of an IEEE division.  Over every 11-bit divisor significand and
    every dividend significand (both signs, quotients 2^-4 .. 2^7: all that can change a
    4-bit code) the quotient must be the IEEE one, bit for bit."""
    n, first = w4.selftest_quotient()
    assert n == 0, f"{n} quotients differ; first: b, a, got, want = {[hex(v) for v in first]}"
