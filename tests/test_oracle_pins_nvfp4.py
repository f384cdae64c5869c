"""Pins of the oracle's NVFP4-weight functions against what the format definition and
independent routines fix: the E2M1 table and rounding (brute force), E4M3 against torch's
float8_e4m3fn, a numpy/torch re-implementation of the whole quantizer, closed-form layers,
invariants (sign, powers of two), the rounding bound and the product (numpy matmul).
[DeepCompressor README: FP4_E2M1 among the toolbox's data types, NVFP4 in its tables.]"""
import numpy as np
import pytest
import torch

import oracle

E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
ORDER = [0, 2, 4, 6, 1, 3, 5, 7]  # element ORDER[j] sits in nibble j


@pytest.fixture(scope="module", autouse=True)
def _built():
    oracle.build()


def test_e2m1_table():
    got = [oracle.e2m1_code_to_f32(c) for c in range(16)]
    want = list(E2M1) + list(-E2M1)
    assert got == want
    assert np.signbit(oracle.e2m1_code_to_f32(8))  # code 8 is -0


def _e2m1_nearest(r: float) -> int:
    """Brute force: nearest grid value, ties to the even code, saturation at 6, sign kept."""
    a = abs(r)
    d = np.abs(E2M1 - a)
    best = [c for c in range(8) if d[c] == d.min()]
    c = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
    return c | (8 if np.signbit(r) else 0)


def test_e2m1_rounding_brute_force():
    rng = np.random.default_rng(1)
    vals = list(rng.uniform(-8, 8, 4000)) + [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -5.0, 6.0, 7.0, 100.0,
                                              -0.0, 0.0, 1e-30, -1e-30, 0.2500001, 0.2499999]
    for v in vals:
        v32 = float(np.float32(v))
        assert oracle.f32_to_e2m1_code(v32) == _e2m1_nearest(v32), v32
    # ties go to the even code
    assert [oracle.f32_to_e2m1_code(t) for t in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)] == [0, 2, 2, 4, 4, 6, 6]
    assert oracle.f32_to_e2m1_code(float("nan")) == 0xFF


def test_e4m3_decode_matches_torch():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).float().numpy()
    for b in range(256):
        got = oracle.e4m3_bits_to_f32(b)
        if (b & 0x7F) == 0x7F:
            assert np.isnan(got)
        else:
            assert got == ref[b] and np.signbit(got) == np.signbit(ref[b]), hex(b)


def test_e4m3_encode_matches_torch():
    rng = np.random.default_rng(2)
    vals = np.concatenate([rng.uniform(-464, 464, 3000), rng.uniform(-1, 1, 3000) * 2.0 ** rng.integers(-12, 2, 3000),
                           np.array([448.0, 464.0, -464.0, 2.0 ** -10, 1.5 * 2.0 ** -9, 1.0625, 1.1875, 0.0, -0.0])])
    vals = vals.astype(np.float32)
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.f32_to_e4m3_bits(float(v)) for v in vals], np.uint8)
    assert np.array_equal(got, ref)
    # every finite code round-trips
    for b in range(256):
        if (b & 0x7F) != 0x7F:
            assert oracle.f32_to_e4m3_bits(oracle.e4m3_bits_to_f32(b)) == b
    # the reading saturates (torch would give NaN above 464)
    assert oracle.f32_to_e4m3_bits(500.0) == 0x7E and oracle.f32_to_e4m3_bits(-1e30) == 0xFE


def _quantize_numpy(W, s):
    """The section's steps, restated with numpy float32 and torch's E4M3 conversion."""
    Wp = (W.astype(np.float32) * s.astype(np.float32)[None, :]).astype(np.float32)
    N, K = W.shape
    amax = np.float32(np.abs(Wp).max())
    g = np.float32(amax / np.float32(2688.0)) if amax > 0 else np.float32(1.0)
    six_g = np.float32(np.float32(6.0) * g)
    blocks = Wp.reshape(N, K // 16, 16)
    bmax = np.abs(blocks).max(-1).astype(np.float32)
    sb = (bmax / six_g).astype(np.float32)
    s8 = torch.from_numpy(sb).to(torch.float8_e4m3fn).view(torch.uint8).numpy()  # sb <= 448 here
    S = (torch.from_numpy(s8.copy()).view(torch.float8_e4m3fn).float().numpy() * g).astype(np.float32)
    codes = np.zeros((N, K // 16, 16), np.uint32)
    for n in range(N):
        for b in range(K // 16):
            if S[n, b] == 0:
                continue
            for i in range(16):
                codes[n, b, i] = _e2m1_nearest(float(np.float32(blocks[n, b, i] / S[n, b])))
    codes = codes.reshape(N, K)
    qw = np.zeros((N, K // 8), np.uint32)
    for j in range(8):
        qw |= codes[:, ORDER[j]::8] << np.uint32(4 * j)
    return qw, s8.T.copy(), float(g)


@pytest.mark.parametrize("N,K,seed", [(8, 64, 1), (32, 256, 2), (16, 1024, 3)])
def test_quantize_matches_numpy_restatement(N, K, seed):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((N, K)) * np.exp(rng.standard_normal((N, 1)))).astype(np.float32)
    s = np.exp(rng.standard_normal(K) * 0.5).astype(np.float32)
    qw, sc, g = oracle.quantize_nvfp4_with_scales(W, s)
    rqw, rsc, rg = _quantize_numpy(W, s)
    assert g == rg
    assert np.array_equal(sc, rsc)
    assert np.array_equal(qw, rqw)


def test_quantize_closed_form():
    """amax = 2688 * 2^-10 makes g = 2^-10; each block is E2M1 grid values times an E4M3
    value v times g, with max |code value| 6: s8 = v, the codes are the grid indices and the
    dequantized weights are W exactly."""
    rng = np.random.default_rng(4)
    N, K = 16, 128
    e4m3_vals = np.array([oracle.e4m3_bits_to_f32(b) for b in range(1, 0x7F)])
    W = np.zeros((N, K), np.float32)
    for n in range(N):
        for b in range(K // 16):
            v = 448.0 if (n, b) == (0, 0) else float(rng.choice(e4m3_vals[e4m3_vals >= 2.0 ** -3]))
            idx = rng.integers(0, 8, 16)
            idx[0] = 7  # the block's maximum is 6 v g
            sign = rng.choice([-1.0, 1.0], 16)
            W[n, 16 * b:16 * b + 16] = sign * E2M1[idx] * v * 2.0 ** -10
    qw, sc, g = oracle.quantize_nvfp4_with_scales(W, np.ones(K, np.float32))
    assert g == 2.0 ** -10
    assert np.array_equal(oracle.dequant_nvfp4(qw, sc, g, N, K), W.astype(np.float64))


def test_invariants_sign_and_power_of_two():
    rng = np.random.default_rng(5)
    W = rng.standard_normal((16, 256)).astype(np.float32)
    one = np.ones(256, np.float32)
    qw, sc, g = oracle.quantize_nvfp4_with_scales(W, one)
    nqw, nsc, ng = oracle.quantize_nvfp4_with_scales(-W, one)
    assert ng == g and np.array_equal(nsc, sc)
    assert np.array_equal(nqw, qw ^ np.uint32(0x88888888))  # every code's sign bit flips
    pqw, psc, pg = oracle.quantize_nvfp4_with_scales(W * np.float32(32.0), one)
    assert pg == g * 32.0 and np.array_equal(psc, sc) and np.array_equal(pqw, qw)


def test_rounding_bound():
    rng = np.random.default_rng(6)
    N, K = 32, 512
    W = (rng.standard_normal((N, K)) ** 3).astype(np.float32)
    qw, sc, g = oracle.quantize_nvfp4_with_scales(W, np.ones(K, np.float32))
    deq = oracle.dequant_nvfp4(qw, sc, g, N, K)
    S = np.repeat(np.array([[oracle.e4m3_bits_to_f32(b) for b in row] for row in sc.T]) * g, 16, axis=1)
    w = W.astype(np.float64)
    # half the widest grid gap (1 between 4 and 6) plus what saturation at 6 S cuts off
    bound = 1.0 * S + np.maximum(0.0, np.abs(w) - 6.0 * S) + 1e-12
    assert np.all(np.abs(w - deq) <= bound)


def test_linear_matches_numpy():
    rng = np.random.default_rng(7)
    N, K, M = 16, 256, 3
    W = rng.standard_normal((N, K)).astype(np.float32)
    qw, sc, g, _ = oracle.awq_quantize_nvfp4(W, np.abs(rng.standard_normal(K)).astype(np.float32) + 0.1, 0.5)
    x = (torch.from_numpy(rng.standard_normal((M, K)).astype(np.float32)).to(torch.bfloat16)
         .view(torch.int16).numpy().view(np.uint16))
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    deq = oracle.dequant_nvfp4(qw, sc, g, N, K)
    rp = np.array([0, 2] + [2] * (N - 1), np.int32)
    ci = np.array([3, 100], np.int32)
    v = np.array([0.5, -2.0], np.float16).view(np.uint16)
    y, ya = oracle.linear_nvfp4(x, qw, sc, g, N, csr=(rp, ci, v), with_abs=True)
    want = xf @ deq.T
    want[:, 0] += xf[:, 3] * 0.5 - xf[:, 100] * 2.0
    assert np.allclose(y, want, rtol=1e-12, atol=1e-12)
    assert np.all(ya >= np.abs(y) - 1e-12)
