"""Pins of the oracle's 3-bit variant against hand-derived words, the layout rule, closed
forms, error bounds and numpy (CPU only).

[SqueezeLLM article, sections 2.1-2.2: once its outliers are split off, the dense part takes
uniform quantization as coarse as 3 bits (eight levels).]  Read as the library's min/max RTN
with 2^3 - 1 steps; codes packed 32 per three 32-bit words (the layout rule is in the golden
file's header)."""
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
ORDER = [0, 2, 4, 6, 1, 3, 5, 7]


def golden_cases():
    cases = []
    with open(os.path.join(GOLDEN, "pack3_order.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            codes, words = line.split("->")
            cases.append(([int(c) for c in codes.split()], [int(w, 16) for w in words.split()]))
    return cases


def test_pack3_golden_words(orc):
    cases = golden_cases()
    assert len(cases) == 5
    for codes, words in cases:
        assert list(orc.pack32x3(codes)) == words, codes
        assert list(orc.unpack32x3(np.array(words, np.uint32))) == codes


def test_pack3_every_position_and_value(orc):
    """One nonzero code at a time: exactly the bits the rule names are set."""
    for e in range(32):
        for v in range(1, 8):
            q = np.zeros(32, np.uint8)
            q[e] = v
            want = [0, 0, 0]
            if e < 24:
                want[e // 8] = v << (4 * ORDER.index(e % 8))
            else:
                j = ORDER.index(e - 24)
                for b in range(3):
                    if (v >> b) & 1:
                        want[b] |= 1 << (4 * j + 3)
            assert list(orc.pack32x3(q)) == want, (e, v)
            assert list(orc.unpack32x3(np.array(want, np.uint32))) == list(q)


def test_pack3_pairs_for_magic_unpack(orc):
    """What the layout is for: each 16-bit half of ((w >> 4i) & 0x00070007) is one code,
    elements (8w + 2i, 8w + 2i + 1); the bit-3 planes, shifted by 4i + 3 - b and masked
    with bit b of each half, assemble elements (24 + 2i, 24 + 2i + 1)."""
    rng = np.random.default_rng(3)
    for _ in range(200):
        q = rng.integers(0, 8, 32).astype(np.uint8)
        w = [int(x) for x in orc.pack32x3(q)]
        for i in range(4):
            for wi in range(3):
                t = (w[wi] >> (4 * i)) & 0x00070007
                assert (t & 0xFFFF, t >> 16) == (q[8 * wi + 2 * i], q[8 * wi + 2 * i + 1])
            t = 0
            for b in range(3):
                t |= (w[b] >> (4 * i + 3 - b)) & (0x00010001 << b)
            assert (t & 0xFFFF, t >> 16) == (q[24 + 2 * i], q[24 + 2 * i + 1])


def test_pack3_rejects_code_above_7(orc):
    q = np.zeros(32, np.uint8)
    q[5] = 8
    with pytest.raises(orc.OracleError):
        orc.pack32x3(q)


def unpack3_all(qw3, sc, z, N, K, gs=128):
    """Codes [N][K], zeros [N][G], scales f32 [N][G] from the 3-bit layout (numpy)."""
    codes = np.zeros((N, K), np.int64)
    words = qw3.reshape(N, K // 32, 3).astype(np.int64)
    for wi in range(3):
        for j in range(8):
            codes[:, 8 * wi + ORDER[j]::32] = (words[:, :, wi] >> (4 * j)) & 7
    for j in range(8):
        c = np.zeros((N, K // 32), np.int64)
        for b in range(3):
            c |= ((words[:, :, b] >> (4 * j + 3)) & 1) << b
        codes[:, 24 + ORDER[j]::32] = c
    G = K // gs
    zz = np.zeros((G, N), np.int64)
    for j in range(8):
        zz[:, j::8] = (z.astype(np.int64) >> (4 * j)) & 15
    return codes, zz.T.copy(), sc.view(np.float16).astype(np.float32).T.copy()


def test_quantize3_closed_form(orc):
    """w' = (i - z0) 2^-6 with i cycling 0..7: scale 7 * 2^-6 / 7 = 2^-6 exactly, zero z0,
    codes i, dequantized values w' exactly (s = 1: alpha = 0)."""
    N, K = 8, 1024
    W = np.zeros((N, K), np.float32)
    z0 = np.zeros((N, K // 128), np.int64)
    for n in range(N):
        for g in range(K // 128):
            z0[n, g] = (n + 3 * g) % 8
            W[n, 128 * g:128 * (g + 1)] = ((np.arange(128) % 8) - z0[n, g]) * 2.0 ** -6
    qw3, sc, z, s = orc.awq_quantize3(W, np.ones(K, np.float32), 0.0)
    assert np.all(s == 1.0)
    codes, zz, scale = unpack3_all(qw3, sc, z, N, K)
    assert np.all(scale == 2.0 ** -6)
    assert np.array_equal(zz, z0)
    assert np.array_equal(codes, np.tile(np.arange(K) % 8, (N, 1)))
    assert np.array_equal(orc.dequant3(qw3, sc, z, N, K), W)


def test_quantize3_bounds_mixed_sign_groups(orc):
    """Codes and zeros in 0..7; |w' - deq| <= sf (1/2 + 7 * 2^-11) in groups that contain 0
    (half a step, plus the fp16 rounding of the scale at the ends); the stored scale is the
    fp16 rounding of (max - min) / 7."""
    rng = np.random.default_rng(8)
    N, K = 64, 2048
    W = (rng.standard_normal((N, K)) * np.exp(rng.uniform(-8, 4, (N, 1)))).astype(np.float32)
    a = np.exp(rng.standard_normal(K)).astype(np.float32)
    qw3, sc, z, s = orc.awq_quantize3(W, a, 0.5)
    Ws = (W * s[None, :]).astype(np.float32)
    codes, zz, scale = unpack3_all(qw3, sc, z, N, K)
    assert codes.min() >= 0 and codes.max() <= 7 and zz.min() >= 0 and zz.max() <= 7
    deq = orc.dequant3(qw3, sc, z, N, K)
    g = np.arange(K) // 128
    sf = scale[:, g]
    assert np.array_equal(deq, ((codes - zz[:, g]) * sf).astype(np.float32))
    Wg = Ws.reshape(N, K // 128, 128)
    mixed = ((Wg.min(-1) <= 0) & (Wg.max(-1) >= 0))[:, g]
    assert mixed.mean() > 0.9
    bound = sf * (0.5 + 7 * 2.0 ** -11) * (1 + 1e-6)
    assert np.all(np.abs(Ws - deq)[mixed] <= bound[mixed])
    want = np.maximum((Wg.max(-1) - Wg.min(-1)) / np.float32(7), np.float32(1e-5))
    assert np.all(np.abs(scale - want) / want <= 2.0 ** -11 * 1.0001)


def test_quantize3_groups_and_validation(orc):
    """Groups of 256 and one per row; sizes that are not whole 32-code blocks are rejected."""
    rng = np.random.default_rng(9)
    N, K = 16, 2048
    W = rng.standard_normal((N, K)).astype(np.float32)
    a = np.ones(K, np.float32)
    for gs in (256, K):
        qw3, sc, z, _ = orc.awq_quantize3(W, a, 0.0, gs)
        assert qw3.shape == (N, 3 * K // 32) and sc.shape == (K // gs, N)
        codes, zz, scale = unpack3_all(qw3, sc, z, N, K, gs)
        deq = orc.dequant3(qw3, sc, z, N, K, gs)
        g = np.arange(K) // gs
        assert np.array_equal(deq, ((codes - zz[:, g]) * scale[:, g]).astype(np.float32))
        assert np.all(np.abs(deq - W) <= 1.5 * scale[:, g] * (1 + 1e-6))
    for gs in (16, 200, 3000):
        with pytest.raises(orc.OracleError):
            orc.awq_quantize3(W, a, 0.0, gs)


def test_linear3_is_x_times_dequant3(orc):
    """The product equals numpy's matmul of the bf16 activations and the dequantized 3-bit
    weights (both exact in double up to the order of the additions), with and without a CSR."""
    import workloads
    rng = np.random.default_rng(10)
    N, K, M = 48, 1024, 5
    W = rng.standard_normal((N, K)).astype(np.float32)
    qw3, sc, z, _ = orc.awq_quantize3(W, np.ones(K, np.float32), 0.0)
    x = workloads.uniform_bf16(11, (M, K), -2, 2)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    deq = orc.dequant3(qw3, sc, z, N, K).astype(np.float64)
    y, ya = orc.linear3(x, qw3, sc, z, N, with_abs=True)
    ref = xf @ deq.T
    absref = np.abs(xf) @ np.abs(deq).T
    assert np.all(np.abs(y - ref) <= 1e-12 * absref)
    assert np.allclose(ya, absref, rtol=1e-12)
    # a CSR term adds x . W_sparse^T
    rp = np.array([0] + [2] * 1 + [2] * (N - 1), np.int32)
    ci = np.array([3, 700], np.int32)
    v = np.array([0x3C00, 0xC000], np.uint16)  # fp16 1.0 and -2.0 in row 0
    yc = orc.linear3(x, qw3, sc, z, N, csr=(rp, ci, v))
    extra = xf[:, 3] * 1.0 - xf[:, 700] * 2.0
    assert np.allclose(yc[:, 0] - y[:, 0], extra, rtol=1e-12, atol=1e-12)
    assert np.array_equal(yc[:, 1:], y[:, 1:])
    # sampled outputs are the same numbers
    m_idx = rng.integers(0, M, 64)
    n_idx = rng.integers(0, N, 64)
    assert np.array_equal(orc.linear3_at(x, qw3, sc, z, N, m_idx, n_idx), y[m_idx, n_idx])
