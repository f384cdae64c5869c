"""GPU AWQ alpha search (awq_search_alpha) against the oracle's search: the same grid, the
same quantizer and fold, errors within the rounding differences of the two products
(fp32 reference on the GPU vs fp64 in the oracle, fp32-accumulated bf16 y_q vs fp64)."""
import numpy as np
import pytest
import torch

import w4a16_gemm_awq_b200 as w4
import workloads
from parity import dev_bf16, dev_f32

pytestmark = pytest.mark.gpu

ALPHAS = [0.0, 0.25, 0.5, 0.75, 1.0]


def raw_x(seed, M, mult):
    return workloads.make_activations(seed, M, mult, alpha=0.0)  # activations before the fold


def compare(orc, W, act, x, alphas, what, rel=2e-2):
    err, best = w4.awq_search_alpha(dev_f32(W), dev_f32(act), dev_bf16(x), alphas)
    ref = orc.awq_search_alpha(W, act, x, alphas)
    err = np.asarray(err, np.float64)
    assert np.all(np.isfinite(err)) and np.all(err > 0), what
    assert np.allclose(err, ref, rtol=rel, atol=0), f"{what}: gpu {err} oracle {ref}"
    # the chosen alpha is the oracle's, or one whose oracle error is within the tolerance of it
    assert ref[best] <= ref.min() * (1 + 2 * rel), f"{what}: best {best} gpu {err} oracle {ref}"
    assert best == int(np.argmin(err))
    return err, ref


@pytest.mark.parametrize("M", [8, 64])
def test_search_matches_oracle(orc, M):
    """M = 8 runs the GEMV, M = 64 the GEMM."""
    L = workloads.make_layer(31 + M, K=1024, N=256)
    compare(orc, L.W, L.act_absmean, raw_x(31 + M, M, L.mult), ALPHAS, f"M={M}")


def test_search_full_layer(orc):
    """A Llama-3-8B o_proj-sized layer with 64 calibration tokens."""
    L = workloads.make_layer(workloads.seed_of(1, 1), K=4096, N=4096)
    compare(orc, L.W, L.act_absmean, raw_x(77, 64, L.mult), [0.0, 0.5, 1.0], "4096x4096")


def test_search_protects_salient_channel():
    rng = np.random.default_rng(23)
    N, K = 256, 1024
    W = rng.standard_normal((N, K)).astype(np.float32)
    mult = np.ones(K, np.float32)
    mult[0] = 100.0
    xf = rng.uniform(-1, 1, (16, K)).astype(np.float32) * mult
    x = torch.from_numpy(xf).to(torch.bfloat16).cuda()
    act = np.abs(xf).mean(axis=0).astype(np.float32) + np.float32(1e-3)
    err, best = w4.awq_search_alpha(dev_f32(W), dev_f32(act), x, [0.0, 0.5])
    assert err[1] < 0.5 * err[0] and best == 1


def test_search_argument_errors():
    W = torch.zeros(128, 1024, device="cuda")
    a = torch.ones(1024, device="cuda")
    x = torch.zeros(4, 1024, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(w4.W4A16Error) as e:
        w4.awq_search_alpha(W, a, x, [0.5, -1.0])
    assert e.value.code == w4.ERR_VALUE
    with pytest.raises(w4.W4A16Error) as e:
        w4.awq_search_alpha(W, a, x, [0.5], workspace=torch.empty(256, dtype=torch.uint8, device="cuda"))
    assert e.value.code == w4.ERR_SHAPE
    with pytest.raises(w4.W4A16Error) as e:
        w4.awq_search_alpha(W, a, x, [0.5] * 65)
    assert e.value.code == w4.ERR_SHAPE


def test_fold_activations_bit_exact(orc):
    """x' = bf16(x / s) with IEEE division: bit-exact against the oracle's conversions."""
    L = workloads.make_layer(41, K=2048, N=128)
    x = raw_x(41, 5, L.mult)
    s = orc.awq_scales(L.act_absmean, 0.5)
    got = w4.awq_fold_activations(dev_bf16(x), dev_f32(s)).view(torch.int16).cpu().numpy().view(np.uint16)
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    want = np.array([[orc.f32_to_bf16_bits(float(np.float32(xf[m, k]) / s[k])) for k in range(2048)]
                     for m in range(5)], np.uint16)
    assert np.array_equal(got, want)
