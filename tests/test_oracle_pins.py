"""Pins for the CPU oracle: each check ties the oracle to something other than itself --
library conversion routines, hand-derived fixtures, closed forms, invariants of the
method, brute force on tiny inputs.  No GPU is used here."""
import os

import numpy as np
import pytest
import torch

import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
ORDER = [0, 2, 4, 6, 1, 3, 5, 7]  # the documented nibble order, restated for brute force


# ------------------------------------------------------------------ conversions ----------

def _np_f16_bits(a):
    return np.asarray(a, np.float32).astype(np.float16).view(np.uint16)


def _torch_bf16_bits(a):
    t = torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _interesting_floats(rng, n):
    specials = np.array([0.0, -0.0, 1.0, -1.0, 65504.0, 65519.99, 65520.0, 65536.0, 1e-5, 6.1e-5,
                         2.0 ** -14, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -25, 1.5 * 2.0 ** -24,
                         np.inf, -np.inf, 3.4e38, 1e-38, 1e-40, 1e-45, 2.0 ** -126, 2.0 ** -133,
                         1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8],
                        np.float32)
    bits = rng.integers(0, 2 ** 32, size=n, dtype=np.uint64).astype(np.uint32)
    rnd = bits.view(np.float32)
    rnd = rnd[np.isfinite(rnd)]
    small = (rng.standard_normal(n) * np.exp(rng.uniform(-30, 12, n))).astype(np.float32)
    return np.concatenate([specials, rnd, small])


def test_f32_to_f16_matches_numpy(orc):
    rng = np.random.default_rng(1)
    xs = _interesting_floats(rng, 20000)
    ref = _np_f16_bits(xs)
    got = np.array([orc.f32_to_f16_bits(float(v)) for v in xs], np.uint16)
    assert np.array_equal(got, ref)


def test_f16_to_f32_all_patterns(orc):
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = pats.view(np.float16).astype(np.float32)
    got = np.array([orc.f16_bits_to_f32(int(h)) for h in pats], np.float32)
    fin = np.isfinite(ref)
    assert np.array_equal(got[fin].view(np.uint32), ref[fin].view(np.uint32))
    assert np.all(np.isnan(got[np.isnan(ref)]))
    assert np.array_equal(got[np.isinf(ref)], ref[np.isinf(ref)])


def test_f32_to_bf16_matches_torch(orc):
    rng = np.random.default_rng(2)
    xs = _interesting_floats(rng, 20000)
    ref = _torch_bf16_bits(xs)
    got = np.array([orc.f32_to_bf16_bits(float(v)) for v in xs], np.uint16)
    assert np.array_equal(got, ref)


def test_bf16_to_f32_all_patterns(orc):
    pats = np.arange(65536, dtype=np.uint32)
    ref = (pats << 16).astype(np.uint32).view(np.float32)
    got = np.array([orc.bf16_bits_to_f32(int(h)) for h in pats], np.float32)
    fin = np.isfinite(ref)
    assert np.array_equal(got[fin].view(np.uint32), ref[fin].view(np.uint32))
    assert np.all(np.isnan(got[np.isnan(ref)]))


# ------------------------------------------------------------------ packing --------------

def test_pack_golden_words(orc):
    for line in open(os.path.join(GOLDEN, "pack_order.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        *codes, word = line.split()
        codes = [int(c) for c in codes]
        assert orc.pack8(codes) == int(word, 16), line
        assert list(orc.unpack8(int(word, 16))) == codes


def test_pack_every_position_and_value(orc):
    for e in range(8):
        for v in range(16):
            codes = [0] * 8
            codes[e] = v
            w = orc.pack8(codes)
            j = ORDER.index(e)
            assert w == v << (4 * j)
            assert list(orc.unpack8(w)) == codes


def test_pack_roundtrip_random(orc):
    rng = np.random.default_rng(3)
    for w in rng.integers(0, 2 ** 32, size=20000, dtype=np.uint64):
        q = orc.unpack8(int(w))
        assert orc.pack8(q) == int(w)


def test_pack_pairs_for_magic_unpack(orc):
    """The order puts elements (2i, 2i+1) in the low/high 16-bit halves of (w >> 4i) & 0x000F000F."""
    rng = np.random.default_rng(4)
    for _ in range(2000):
        q = rng.integers(0, 16, 8)
        w = orc.pack8(q)
        for i in range(4):
            pair = (w >> (4 * i)) & 0x000F000F
            assert pair & 0xFFFF == q[2 * i] and pair >> 16 == q[2 * i + 1]


def test_pack_rejects_out_of_range_code(orc):
    with pytest.raises(orc.OracleError):
        orc.pack8([16, 0, 0, 0, 0, 0, 0, 0])


# ------------------------------------------------------------------ helpers --------------

def unpack_all(qw, sc, z, N, K):
    """Format definition restated with numpy: codes [N][K], zero [N][G], scale f32 [N][G].
    scales are stored [G][N]; zeros [G][N/8] with nibble j of word n/8 for row 8*(n/8) + j."""
    codes = np.zeros((N, K), np.int64)
    for j in range(8):
        codes[:, ORDER[j]::8] = (qw >> np.uint32(4 * j)) & np.uint32(15)
    G = K // 128
    zz = np.zeros((G, N), np.int64)
    for j in range(8):
        zz[:, j::8] = (z >> np.uint32(4 * j)) & np.uint32(15)
    s = sc.view(np.float16).astype(np.float32)
    return codes, zz.T.copy(), s.T.copy()


def closed_form_group(z0, scale=2.0 ** -6):
    i = np.arange(128) % 16
    return ((i - z0) * scale).astype(np.float32)


# ------------------------------------------------------------------ quantizer ------------

def test_closed_form_golden(orc):
    for line in open(os.path.join(GOLDEN, "quant_closed_form.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, z0, sbits, zero, *head = line.split()
        K = 1024
        if name == "T":
            grp = closed_form_group(int(z0))
            grp[:4] = np.array([0.5, 1.5, -0.5, 2.5], np.float32) * np.float32(2.0 ** -6)
            W = np.tile(grp, K // 128)[None, :]
            want_codes = np.arange(K) % 16
            for i, c in enumerate(head):
                want_codes[i::128] = int(c)
        elif name == "Z":
            W = np.zeros((1, K), np.float32)
            want_codes = np.zeros(K, np.int64)
        else:
            W = np.tile(closed_form_group(int(z0)), K // 128)[None, :]
            want_codes = np.arange(K) % 16
        W = np.repeat(W, 8, axis=0)   # 8 identical rows: one whole word of zero points
        qw, sc, z, s = orc.awq_quantize_g128(W, np.ones(K, np.float32), 0.0)
        assert np.all(s == 1.0)
        codes, zz, scale = unpack_all(qw, sc, z, 8, K)
        assert np.all(sc == int(sbits, 16)), name
        assert np.all(zz == int(zero)), name
        assert np.all(z == int(zero) * 0x11111111), name   # the zero point in all 8 nibbles
        assert np.array_equal(codes[0], want_codes) and np.all(codes == codes[0]), name
        deq = orc.dequant(qw, sc, z, 8, K)
        if name == "Z":
            assert np.all(deq == 0.0)
        else:
            want = W.copy()
            if name == "T":   # the tied weights reconstruct to (q - z) * 2^-6
                for i, c in enumerate(head):
                    want[:, i::128] = (int(c) - int(zero)) * 2.0 ** -6
            assert np.array_equal(deq, want)  # zero reconstruction error off the ties


def test_bounds_mixed_sign_groups(orc):
    """q, z in [0,15] and |w' - deq| <= sf (1/2 + 15 * 2^-11) for groups containing 0's sign change."""
    rng = np.random.default_rng(5)
    N, K = 64, 2048
    W = (rng.standard_normal((N, K)) * np.exp(rng.uniform(-8, 4, (N, 1)))).astype(np.float32)
    a = np.exp(rng.standard_normal(K)).astype(np.float32)
    qw, sc, z, s = orc.awq_quantize_g128(W, a, 0.5)
    Ws = (W * s[None, :]).astype(np.float32)
    codes, zz, scale = unpack_all(qw, sc, z, N, K)
    deq = orc.dequant(qw, sc, z, N, K)
    g = np.arange(K) // 128
    sf = scale[:, g]
    Wg = Ws.reshape(N, K // 128, 128)
    mixed = ((Wg.min(-1) <= 0) & (Wg.max(-1) >= 0))[:, g]
    assert mixed.mean() > 0.9
    err = np.abs(Ws - deq)
    bound = sf * (0.5 + 15 * 2.0 ** -11) * (1 + 1e-6)
    assert np.all(err[mixed] <= bound[mixed])
    assert codes.min() >= 0 and codes.max() <= 15 and zz.min() >= 0 and zz.max() <= 15
    # the stored scale is the fp16 rounding of (max - min)/15 (floored at 1e-5)
    want = np.maximum((Wg.max(-1) - Wg.min(-1)) / np.float32(15), np.float32(1e-5))
    rel = np.abs(scale - want) / want
    assert np.all(rel <= 2.0 ** -11 * 1.0001)


def test_same_sign_groups_clamp(orc):
    """All-positive groups: z = 0; codes saturate at 15 above 15.5 sf, are RTN below 14.5 sf."""
    rng = np.random.default_rng(6)
    K = 1024
    W = rng.uniform(0.5, 1.5, (8, K)).astype(np.float32)
    qw, sc, z, _ = orc.awq_quantize_g128(W, np.ones(K, np.float32), 0.0)
    codes, zz, scale = unpack_all(qw, sc, z, 8, K)
    assert np.all(zz == 0)
    t = W / scale[:, np.arange(K) // 128]
    assert np.all(codes[t >= 15.5] == 15)
    low = t <= 14.5
    assert np.all(np.abs(codes[low] - t[low]) <= 0.5 + 1e-6)
    # all-negative groups: z = 15 only if -min/sf >= 14.5; codes clamp at 0 for w/sf + z < -0.5
    Wn = -W
    qw, sc, z, _ = orc.awq_quantize_g128(Wn, np.ones(K, np.float32), 0.0)
    codes, zz, scale = unpack_all(qw, sc, z, 8, K)
    tn = Wn / scale[:, np.arange(K) // 128]
    zb = zz[:, np.arange(K) // 128]
    assert np.all(codes[tn + zb <= -0.5] == 0)


def test_alpha_zero_is_plain_rtn(orc):
    rng = np.random.default_rng(7)
    N, K = 32, 2048
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    a = np.exp(rng.standard_normal(K)).astype(np.float32)
    q1 = orc.awq_quantize_g128(W, a, 0.0)
    q2 = orc.quantize_with_scales(W, np.ones(K, np.float32))
    assert np.all(q1[3] == 1.0)
    for u, v in zip(q1[:3], q2):
        assert np.array_equal(u, v)


def test_power_of_two_scales_commute(orc):
    """With s constant and a power of two within each group (a_k = 4^j, alpha = 1/2 -> s = 2^j),
    codes and zeros equal plain RTN of W and each scale is the RTN scale times 2^j, bit-exact."""
    rng = np.random.default_rng(8)
    N, K = 32, 2048
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    j = rng.integers(-3, 4, K // 128)
    a = np.repeat(4.0 ** j, 128).astype(np.float32)
    qw, sc, z, s = orc.awq_quantize_g128(W, a, 0.5)
    assert np.array_equal(s, np.repeat(2.0 ** j, 128).astype(np.float32))
    qw0, sc0, z0 = orc.quantize_with_scales(W, np.ones(K, np.float32))
    assert np.array_equal(qw, qw0) and np.array_equal(z, z0)
    want = (sc0.view(np.float16).astype(np.float64) * (2.0 ** j)[:, None]).astype(np.float16)
    assert np.array_equal(sc, want.view(np.uint16))


def test_scale_vector(orc):
    a = np.array([0.0, 1.0, 4.0, 0.25, 1e-12, 100.0, 2.0], np.float32)
    s = orc.awq_scales(a, 0.5)
    assert s[0] == np.float32(1e-4) and s[4] == np.float32(1e-4)  # the floor
    assert s[1] == 1.0 and s[2] == 2.0 and s[3] == 0.5 and s[5] == 10.0
    assert s[6] == np.float32(np.sqrt(2.0))  # correctly rounded sqrt(2) in fp32
    assert np.all(orc.awq_scales(a, 0.0) == 1.0)
    assert np.array_equal(orc.awq_scales(a, 1.0), np.maximum(a, np.float32(1e-4)))


def test_value_errors(orc):
    K = 1024
    W = np.zeros((8, K), np.float32)
    W[1, 7] = np.nan
    with pytest.raises(orc.OracleError) as e:
        orc.awq_quantize_g128(W, np.ones(K, np.float32), 0.5)
    assert e.value.code == orc.ERR_VALUE
    W = np.zeros((8, K), np.float32)
    W[0, :64] = 1e6   # (max - min)/15 = 66667 > 65504: the fp16 scale overflows
    with pytest.raises(orc.OracleError) as e:
        orc.awq_quantize_g128(W, np.ones(K, np.float32), 0.5)
    assert e.value.code == orc.ERR_VALUE
    with pytest.raises(orc.OracleError) as e:
        orc.awq_quantize_g128(np.zeros((8, 1000), np.float32), np.ones(1000, np.float32), 0.5)
    assert e.value.code == orc.ERR_SHAPE
    with pytest.raises(orc.OracleError) as e:   # zero points pack 8 rows per word
        orc.awq_quantize_g128(np.zeros((12, 1024), np.float32), np.ones(1024, np.float32), 0.5)
    assert e.value.code == orc.ERR_SHAPE
    with pytest.raises(orc.OracleError) as e:
        orc.awq_scales(np.array([-1.0], np.float32), 0.5)
    assert e.value.code == orc.ERR_VALUE


# ------------------------------------------------------------------ linear ---------------

def test_linear_brute_force(orc):
    rng = np.random.default_rng(9)
    M, N, K = 3, 16, 1024
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    a = np.exp(rng.standard_normal(K)).astype(np.float32)
    qw, sc, z, s = orc.awq_quantize_g128(W, a, 0.5)
    x = workloads.uniform_bf16(10, (M, K), -2, 2)
    y, ya = orc.linear(x, qw, sc, z, N, with_abs=True)
    codes, zz, scale = unpack_all(qw, sc, z, N, K)
    g = np.arange(K) // 128
    deq = ((codes - zz[:, g]) * scale[:, g].astype(np.float64))
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ref = xf @ deq.T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(ya, np.abs(xf) @ np.abs(deq).T, rtol=1e-12, atol=1e-12)
    # the dequantized matrix of the oracle is the same
    assert np.array_equal(orc.dequant(qw, sc, z, N, K).astype(np.float64), deq)
    # sampled outputs agree with the full product
    mi = rng.integers(0, M, 40)
    ni = rng.integers(0, N, 40)
    ys = orc.linear_at(x, qw, sc, z, N, mi, ni)
    assert np.array_equal(ys, y[mi, ni])


def test_linear_exact_weights_is_plain_matmul(orc):
    """When every group is closed-form (deq == W exactly), y = x W^T computed by numpy."""
    rng = np.random.default_rng(11)
    M, N, K = 4, 8, 1024
    W = np.stack([np.concatenate([closed_form_group(int(rng.integers(0, 16)),
                                                    2.0 ** int(rng.integers(-8, -2)))
                                  for _ in range(K // 128)]) for _ in range(N)])
    qw, sc, z, _ = orc.awq_quantize_g128(W, np.ones(K, np.float32), 0.0)
    x = workloads.uniform_bf16(12, (M, K))
    y = orc.linear(x, qw, sc, z, N)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.array_equal(y, xf @ W.astype(np.float64).T)


def test_scaling_invariant(orc):
    """(x/s)(W s)^T == x W^T for power-of-two s constant per group (exact on the oracle)."""
    rng = np.random.default_rng(13)
    M, N, K = 2, 8, 1024
    W = np.stack([np.concatenate([closed_form_group(int(rng.integers(0, 16)), 2.0 ** -5)
                                  for _ in range(K // 128)]) for _ in range(N)])
    x = workloads.uniform_bf16(14, (M, K))
    j = rng.integers(-2, 3, K // 128)
    a = np.repeat(4.0 ** j, 128).astype(np.float32)      # s = 2^j
    qw, sc, z, s = orc.awq_quantize_g128(W, a, 0.5)
    xs = ((x.astype(np.uint32) << 16).view(np.float32) / s).astype(np.float32)
    x2 = _torch_bf16_bits(xs)   # exact: dividing a bf16 by a power of two
    y_scaled = orc.linear(x2, qw, sc, z, N)
    qw1, sc1, z1, _ = orc.awq_quantize_g128(W, np.ones(K, np.float32), 0.0)
    y_plain = orc.linear(x, qw1, sc1, z1, N)
    assert np.array_equal(y_scaled, y_plain)


def test_csr_only_is_spmm(orc):
    """With an all-zero dense part, y is the sparse product (checked against scipy)."""
    import scipy.sparse as sp
    rng = np.random.default_rng(15)
    M, N, K = 5, 32, 1024
    qw, sc, z, _ = orc.awq_quantize_g128(np.zeros((N, K), np.float32), np.ones(K, np.float32), 0.0)
    dense = sp.random(N, K, density=0.01, format="csr", random_state=16, dtype=np.float64)
    dense.data = rng.standard_normal(dense.nnz).astype(np.float16).astype(np.float64)
    dense.sort_indices()
    vals = dense.data.astype(np.float16).view(np.uint16)
    x = workloads.uniform_bf16(17, (M, K))
    y = orc.linear(x, qw, sc, z, N, csr=(dense.indptr, dense.indices, vals))
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.allclose(y, (dense @ xf.T).T, rtol=1e-13, atol=1e-13)


def test_csr_empty_equals_dense_only(orc):
    rng = np.random.default_rng(18)
    M, N, K = 2, 16, 1024
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    qw, sc, z, _ = orc.awq_quantize_g128(W, np.ones(K, np.float32), 0.5)
    x = workloads.uniform_bf16(19, (M, K))
    y0 = orc.linear(x, qw, sc, z, N)
    y1 = orc.linear(x, qw, sc, z, N, csr=(np.zeros(N + 1, np.int32), np.zeros(0, np.int32),
                                           np.zeros(0, np.uint16)))
    assert np.array_equal(y0, y1)
    # and a CSR row changes exactly its own output column
    rp = np.zeros(N + 1, np.int32)
    rp[4:] = 1
    y2 = orc.linear(x, qw, sc, z, N, csr=(rp, np.array([3], np.int32),
                                           np.array([0x3C00], np.uint16)))  # +1.0 * x[:, 3]
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    d = y2 - y0
    assert np.allclose(d[:, 3], xf[:, 3]) and np.all(np.delete(d, 3, axis=1) == 0)


def test_csr_validation(orc):
    N, K = 8, 1024
    qw, sc, z, _ = orc.awq_quantize_g128(np.zeros((N, K), np.float32), np.ones(K, np.float32), 0.0)
    x = workloads.uniform_bf16(20, (1, K))
    bad_sorted = (np.array([0, 2] + [2] * 7, np.int32), np.array([5, 3], np.int32),
                  np.array([0x3C00, 0x3C00], np.uint16))
    with pytest.raises(orc.OracleError):
        orc.linear(x, qw, sc, z, N, csr=bad_sorted)
    bad_col = (np.array([0] + [1] * 8, np.int32), np.array([K], np.int32), np.array([0], np.uint16))
    with pytest.raises(orc.OracleError):
        orc.linear(x, qw, sc, z, N, csr=bad_col)


# ------------------------------------------------------------------ outlier split --------

def _brute_split(W, a, s, nnz):
    N, K = W.shape
    score = (np.abs(W) * a[None, :]).astype(np.float32).ravel()
    idx = np.arange(N * K)
    order = np.lexsort((idx, -score.astype(np.float64)))   # score desc, then index asc
    chosen = np.zeros(N * K, bool)
    chosen[order[:nnz]] = True
    chosen = chosen.reshape(N, K)
    Wd = np.where(chosen, np.float32(0), W)
    rows, cols = np.nonzero(chosen)
    rp = np.zeros(N + 1, np.int64)
    np.add.at(rp, rows + 1, 1)
    rp = np.cumsum(rp)
    vals = (W[rows, cols] * s[cols]).astype(np.float32).astype(np.float16).view(np.uint16)
    return Wd, rp, cols, vals


@pytest.mark.parametrize("seed,ties", [(21, False), (22, True)])
def test_split_outliers_brute_force(orc, seed, ties):
    rng = np.random.default_rng(seed)
    N, K = 24, 256
    if ties:   # few distinct magnitudes and a constant act_absmean: many equal scores
        W = (rng.integers(-3, 4, (N, K)) * 0.01).astype(np.float32)
        a = np.ones(K, np.float32)
    else:
        W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
        a = np.exp(rng.standard_normal(K)).astype(np.float32)
    nnz = 97
    Wd, rp, ci, v = orc.split_outliers(W, a, 0.5, nnz)
    s = orc.awq_scales(a, 0.5)
    Wd2, rp2, ci2, v2 = _brute_split(W, a, s, nnz)
    assert np.array_equal(Wd, Wd2)
    assert np.array_equal(rp, rp2) and np.array_equal(ci, ci2) and np.array_equal(v, v2)
    # the split is lossless up to the fp16 rounding of the scaled values
    back = Wd.astype(np.float64).copy()
    rows = np.repeat(np.arange(N), np.diff(rp))
    back[rows, ci] += v.view(np.float16).astype(np.float64) / s[ci]
    assert np.allclose(back, W, rtol=2.0 ** -10, atol=0)


def test_split_outliers_edge_counts(orc):
    rng = np.random.default_rng(23)
    N, K = 4, 64
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    a = np.ones(K, np.float32)
    Wd, rp, ci, v = orc.split_outliers(W, a, 0.0, 0)
    assert np.array_equal(Wd, W) and np.all(rp == 0) and ci.size == 0
    Wd, rp, ci, v = orc.split_outliers(W, a, 0.0, N * K)
    assert np.all(Wd == 0) and np.array_equal(rp, np.arange(N + 1) * K)
    assert np.array_equal(v, W.ravel().astype(np.float16).view(np.uint16))


# ---- AWQ alpha search (oracle_awq_search_alpha) ------------------------------------------

def _raw_activations(seed, M, mult):
    """Calibration activations before the 1/s fold: N(0,1) * m_k."""
    return workloads.make_activations(seed, M, mult, alpha=0.0)


def test_search_power_of_two_invariance(orc):
    """a -> 4a multiplies s by 4^alpha = 1, 2, 4 for alpha = 0, 0.5, 1: W*s, the group scales
    and x/s all change by exact powers of two, so every error is unchanged bit for bit."""
    L = workloads.make_layer(21, K=1024, N=128)
    x = _raw_activations(21, 6, L.mult)
    alphas = [0.0, 0.5, 1.0]
    e1 = orc.awq_search_alpha(L.W, L.act_absmean, x, alphas)
    e4 = orc.awq_search_alpha(L.W, (L.act_absmean * np.float32(4.0)).astype(np.float32), x, alphas)
    assert np.array_equal(e1, e4)
    assert np.all(np.isfinite(e1)) and np.all(e1 > 0)


def test_search_alpha0_is_plain_rtn(orc):
    """alpha = 0 is plain RTN of W with x unchanged: recompute that error from the dequantized
    matrix with numpy and torch's bf16 rounding, independently of the oracle's product."""
    import torch
    L = workloads.make_layer(22, K=2048, N=128)
    x = _raw_activations(22, 4, L.mult)
    e = orc.awq_search_alpha(L.W, L.act_absmean, x, [0.0])[0]
    qw, sc, z = orc.quantize_with_scales(L.W, np.ones(2048, np.float32))
    deq = orc.dequant(qw, sc, z, 128, 2048).astype(np.float64)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    yq = xf @ deq.T
    yq = torch.from_numpy(yq.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    yr = xf @ L.W.astype(np.float64).T
    want = ((yq - yr) ** 2).sum() / (yr ** 2).sum()
    assert e == pytest.approx(want, rel=1e-9)


def test_search_scaling_protects_a_salient_channel(orc):
    """One input channel carries 100x larger activations.  Without scaling its weights are
    quantized with their group's step like all others and the error is dominated by that
    channel; alpha = 0.5 scales them up by ~10, so they set their group's range and the
    output error drops -- the effect the AWQ translation describes in section 3.2."""
    rng = np.random.default_rng(23)
    N, K = 128, 1024
    W = rng.standard_normal((N, K)).astype(np.float32)
    mult = np.ones(K, np.float32)
    mult[0] = 100.0
    x = workloads.uniform_bf16(24, (8, K))
    xf = (x.astype(np.uint32) << 16).view(np.float32) * mult
    x = torch_bf16(xf)
    act = np.abs(xf).mean(axis=0).astype(np.float32) + np.float32(1e-3)
    e = orc.awq_search_alpha(W, act, x, [0.0, 0.5])
    assert e[1] < 0.5 * e[0]


def torch_bf16(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


# ------------------------------------------------------------------ other group sizes -----
# [SqueezeLLM article, section 4.1: the group size option, per-row by default]

def _equal_range_layer(rng, N, K, gs):
    """W whose every 128-wide slice of a group of gs holds that group's minimum and maximum,
    so quantizing with groups of gs and with groups of 128 must agree code for code."""
    W = rng.uniform(-0.9, 0.9, size=(N, K)).astype(np.float32)
    for n in range(N):
        for g in range(K // gs):
            mn, mx = -1.0 - rng.uniform(0, 2), 1.0 + rng.uniform(0, 2)
            for c in range(g * gs, (g + 1) * gs, 128):
                W[n, c + rng.integers(0, 64)] = mn
                W[n, c + 64 + rng.integers(0, 64)] = mx
    return W


@pytest.mark.parametrize("gs", [256, 1024, 2048, 4096])
def test_groups_of_equal_range_reduce_to_g128(orc, gs):
    N, K = 16, 4096
    rng = np.random.default_rng(gs)
    W = _equal_range_layer(rng, N, K, gs)
    act = np.ones(K, np.float32)                           # s = 1 for any alpha
    qa, sa, za, _ = orc.awq_quantize(W, act, 0.5, gs)
    qb, sb, zb, _ = orc.awq_quantize_g128(W, act, 0.5)
    R = gs // 128
    assert np.array_equal(qa, qb)
    assert np.array_equal(np.repeat(sa, R, axis=0), sb)
    assert np.array_equal(np.repeat(za, R, axis=0), zb)
    assert sa.shape == (K // gs, N) and za.shape == (K // gs, N // 8)


@pytest.mark.parametrize("gs", [256, 512, 5120])
def test_group_rtn_error_bound(orc, gs):
    """Round-to-nearest with each element's own group parameters: |deq - w s| <= 1.5 sf_g
    (half a step, plus one step where the fp16-rounded scale makes the top code clamp)."""
    N, K = 24, 5120
    rng = np.random.default_rng(gs + 1)
    W = (rng.standard_normal((N, K)) * rng.uniform(0.01, 2.0, size=(N, 1))).astype(np.float32)
    act = np.exp(rng.uniform(-3, 3, K)).astype(np.float32)
    qw, sc, z, s = orc.awq_quantize(W, act, 0.5, gs)
    deq = orc.dequant(qw, sc, z, N, K, group_size=gs).astype(np.float64)
    ws = (W * s[None, :]).astype(np.float64)               # one IEEE product per element
    sf = sc.view(np.float16).astype(np.float64).T          # [N][K/gs]
    step = np.repeat(sf, gs, axis=1)
    assert np.all(np.abs(deq - ws) <= 1.5 * step + 1e-12)
    # every group's range is covered: its extremes land within one step of the group's min/max
    for g in range(K // gs):
        blk = slice(g * gs, (g + 1) * gs)
        assert np.all(np.abs(deq[:, blk].max(1) - ws[:, blk].max(1)) <= 1.5 * sf[:, g] + 1e-12)
        assert np.all(np.abs(deq[:, blk].min(1) - ws[:, blk].min(1)) <= 1.5 * sf[:, g] + 1e-12)


def test_group_dequant_closed_form(orc):
    """Hand-packed codes q = (n + 3k) mod 16, scales 2^(g mod 5 - 2), zeros (g + n) mod 16."""
    N, K, gs = 16, 2048, 512
    G = K // gs
    n_i, k_i = np.meshgrid(np.arange(N), np.arange(K), indexing="ij")
    q = (n_i + 3 * k_i) % 16
    qw = np.zeros((N, K // 8), np.uint32)
    for n in range(N):
        for w in range(K // 8):
            qw[n, w] = orc.pack8(q[n, 8 * w: 8 * w + 8])
    g_i = np.arange(G)
    sc = np.repeat((2.0 ** (g_i % 5 - 2)).astype(np.float16).view(np.uint16)[:, None], N, axis=1)
    zg = (g_i[:, None] + np.arange(N)[None, :]) % 16           # [G][N]
    zeros = np.zeros((G, N // 8), np.uint32)
    for j in range(8):
        zeros |= (zg[:, j::8].astype(np.uint32) << np.uint32(4 * j))
    deq = orc.dequant(qw, sc, zeros, N, K, group_size=gs)
    expect = (q - zg.T[:, k_i[0] // gs]) * (2.0 ** (k_i // gs % 5 - 2))
    assert np.array_equal(deq.astype(np.float64), expect)


@pytest.mark.parametrize("gs", [256, 2048])
def test_group_linear_is_x_times_dequant(orc, gs):
    """The product with groups of gs equals numpy's matmul of x and the dequantized weights."""
    N, K, M = 40, 2048, 3
    rng = np.random.default_rng(gs + 2)
    W = rng.standard_normal((N, K)).astype(np.float32) * 0.05
    act = np.exp(rng.uniform(-2, 2, K)).astype(np.float32)
    qw, sc, z, _ = orc.awq_quantize(W, act, 0.5, gs)
    x = _torch_bf16_bits(rng.standard_normal((M, K)))
    y = orc.linear(x, qw, sc, z, N, group_size=gs)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ref = xf @ orc.dequant(qw, sc, z, N, K, group_size=gs).astype(np.float64).T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)
    m, n = np.array([0, 2, 1]), np.array([5, 39, 0])
    assert np.allclose(orc.linear_at(x, qw, sc, z, N, m, n, group_size=gs), ref[m, n], rtol=1e-12, atol=1e-12)


def test_group_size_validation(orc):
    W = np.zeros((8, 2048), np.float32)
    a = np.ones(2048, np.float32)
    for gs in (0, 100, 3072, 4096):
        with pytest.raises(Exception):
            orc.awq_quantize(W, a, 0.5, gs)
