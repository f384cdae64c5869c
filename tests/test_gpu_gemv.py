"""GPU decode GEMV (1 <= M <= 16) against the oracle, with and without the CSR outlier term."""
import numpy as np
import pytest
import torch

import w4a16_gemm_awq_b200 as w4
import workloads
from parity import Case, check_close, dev_bf16, dev_bits, dev_csr, host_bf16_as_f64, xs_abs

pytestmark = pytest.mark.gpu

SCHEDULES = [w4.GEMV_STREAM_K, w4.GEMV_CLUSTER]


def gemv(case_dev, fn=None):
    fn = fn or w4.w4a16_gemv
    y = fn(case_dev["x"], case_dev["qweight"], case_dev["scales"], case_dev["zeros"], csr=case_dev["csr"])
    w4.check_device_status()
    return y


def depth(K):
    return K // 128 + 64


@pytest.mark.parametrize("M", [1, 2, 3, 7, 8, 9, 15, 16])
@pytest.mark.parametrize("csr", [False, True])
def test_gemv_small_full_output(orc, M, csr):
    c = Case(orc, seed=100 + M, K=2048, N=256, M=M, csr=csr)
    y = host_bf16_as_f64(gemv(c.device()))
    ref, ref_abs = c.reference(orc)
    check_close(y, ref, ref_abs, 0.0, depth(c.K), f"M={M} csr={csr}", xs_abs(c.x, c.sc))


@pytest.mark.parametrize("K,N", [(1024, 128), (3072, 384), (8192, 128), (1024, 4096), (65536, 128), (16384, 640),
                                 (4096, 2048)])
def test_gemv_odd_shapes(orc, K, N):
    """Includes shapes with more work units than CTAs, where a CTA streams several groups
    through the ring and row blocks are split between CTAs."""
    c = Case(orc, seed=K + N, K=K, N=N, M=5, csr=True)
    y = host_bf16_as_f64(gemv(c.device()))
    ref, ref_abs = c.reference(orc)
    check_close(y, ref, ref_abs, 0.0, depth(K), f"{K}x{N}", xs_abs(c.x, c.sc))


@pytest.mark.parametrize("schedule", SCHEDULES, ids=["stream_k", "cluster"])
@pytest.mark.parametrize("M", [4, 12])
def test_gemv_activation_ranges(orc, schedule, M):
    """Tokens whose magnitudes differ by up to 2^80, groups from 2^-40 to 2^65 (beyond fp16's
    range), all-zero groups and single huge values: every token keeps its own accuracy."""
    c = Case(orc, seed=41 + M, K=2048, N=256, M=M, csr=True)
    rng = np.random.default_rng(M)
    x = (c.x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    G = c.K // 128
    for m in range(M):
        kind = m % 4
        if kind == 1:
            x[m] *= 2.0 ** 40
        elif kind == 2:
            x[m] *= 2.0 ** -40
        elif kind == 3:
            x[m] *= np.repeat(2.0 ** (7.0 * np.arange(G) - 40.0), 128)
        if m % 3 == 0:
            x[m, 256:384] = 0.0                      # an all-zero group
        x[m, rng.integers(0, c.K)] *= 2.0 ** 20      # one value far above the rest of its group
    c.x = (x.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)  # exact: powers of two
    d = c.device()
    y = w4.w4a16_gemv_ex(d["x"], d["qweight"], d["scales"], d["zeros"], csr=d["csr"], schedule=schedule)
    w4.check_device_status()
    ref, ref_abs = c.reference(orc)
    check_close(host_bf16_as_f64(y), ref, ref_abs, 0.0, depth(c.K), f"ranges M={M}", xs_abs(c.x, c.sc))


def test_gemv_empty_csr_is_bit_identical(orc):
    c = Case(orc, seed=7, K=2048, N=256, M=4)
    d = c.device()
    y0 = gemv(d)
    d["csr"] = (torch.zeros(c.N + 1, dtype=torch.int32, device="cuda"), torch.zeros(0, dtype=torch.int32, device="cuda"),
                torch.zeros(0, dtype=torch.int16, device="cuda"))
    y1 = gemv(d)
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))


def test_gemv_csr_only_and_dense_rows(orc):
    """All-zero dense part; one CSR row fully dense, others empty or single."""
    K, N, M = 1024, 128, 3
    qw, sc, z, _ = orc.awq_quantize_g128(np.zeros((N, K), np.float32), np.ones(K, np.float32), 0.0)
    rng = np.random.default_rng(8)
    rows = [np.arange(K) if n == 5 else (np.array([n * 7 % K]) if n % 3 == 0 else np.array([], np.int64))
            for n in range(N)]
    rp = np.concatenate([[0], np.cumsum([len(r) for r in rows])]).astype(np.int32)
    ci = np.concatenate(rows).astype(np.int32)
    v = rng.standard_normal(ci.size).astype(np.float16).view(np.uint16)
    x = workloads.uniform_bf16(9, (M, K))
    d = dict(x=torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda(), qweight=dev_bits(qw, torch.int32),
             scales=dev_bits(sc, torch.int16), zeros=dev_bits(z, torch.int32), csr=dev_csr((rp, ci, v)))
    y = host_bf16_as_f64(gemv(d))
    ref, ref_abs = orc.linear(x, qw, sc, z, N, csr=(rp, ci, v), with_abs=True)
    check_close(y, ref, ref_abs, 0.0, K + 64, "csr only", xs_abs(x, sc))


def test_gemv_reports_bad_csr(orc):
    c = Case(orc, seed=11, K=1024, N=128, M=2)
    d = c.device()
    rp = torch.zeros(c.N + 1, dtype=torch.int32, device="cuda")
    rp[1:] = 1
    d["csr"] = (rp, torch.tensor([c.K + 5], dtype=torch.int32, device="cuda"),
                torch.tensor([0x3C00], dtype=torch.int16, device="cuda"))
    w4.w4a16_gemv(d["x"], d["qweight"], d["scales"], d["zeros"], csr=d["csr"])
    with pytest.raises(w4.W4A16Error) as e:
        w4.check_device_status()
    assert e.value.code == w4.ERR_SHAPE


def test_gemv_workspace_contract(orc):
    """A NULL or short workspace is refused; a workspace is all-zero again after calls that
    split row blocks between CTAs; concurrent-stream calls get their own workspaces."""
    c = Case(orc, seed=13, K=4096, N=512, M=3)
    d = c.device()
    need = w4.workspace_bytes(3, c.N, c.K)
    assert need > 0 and w4.workspace_bytes(17, c.N, c.K, csr=False) >= 128 * 1024  # prefill: counters at least
    with pytest.raises(w4.W4A16Error) as e:
        w4.w4a16_gemv(d["x"], d["qweight"], d["scales"], d["zeros"],
                      workspace=torch.zeros(need - 256, dtype=torch.uint8, device="cuda"))
    assert e.value.code == w4.ERR_SHAPE
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    y0 = w4.w4a16_gemv(d["x"], d["qweight"], d["scales"], d["zeros"], workspace=ws)
    y1 = w4.w4a16_gemv(d["x"], d["qweight"], d["scales"], d["zeros"], workspace=ws)
    w4.check_device_status()
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))
    assert int(ws.count_nonzero()) == ws.numel() - int((ws == 0).sum())  # sanity
    # layout: the row-block counters come first (one uint32 per 128 rows), then the partial
    # tiles, then the fold region of w4a16_gemv_folded
    counters = ws[:c.N // 128 * 4]
    assert int(counters.count_nonzero()) == 0


@pytest.mark.parametrize("schedule", SCHEDULES, ids=["stream_k", "cluster"])
@pytest.mark.parametrize("K,N,M", [(1024, 128, 1), (3072, 384, 16), (4096, 2048, 9), (16384, 640, 5), (8192, 128, 3)])
def test_gemv_schedules_full_output(orc, schedule, K, N, M):
    """Both schedules against the oracle on every output, including shapes where a cluster
    holds several row blocks and where a row block is split over the most CTAs."""
    c = Case(orc, seed=K + 3 * N + M, K=K, N=N, M=M, csr=True)
    d = c.device()
    y = w4.w4a16_gemv_ex(d["x"], d["qweight"], d["scales"], d["zeros"], csr=d["csr"], schedule=schedule)
    w4.check_device_status()
    ref, ref_abs = c.reference(orc)
    check_close(host_bf16_as_f64(y), ref, ref_abs, 0.0, depth(K), f"{K}x{N} M={M} schedule={schedule}",
                xs_abs(c.x, c.sc))


@pytest.mark.parametrize("schedule", SCHEDULES, ids=["stream_k", "cluster"])
@pytest.mark.parametrize("K,N,M", [(4096, 4096, 1), (4096, 6144, 16), (14336, 4096, 8), (4096, 28672, 4)])
def test_gemv_schedules_sampled(orc, schedule, K, N, M):
    c = Case(orc, seed=K + N + M + schedule, K=K, N=N, M=M, csr=False)
    d = c.device()
    y = host_bf16_as_f64(w4.w4a16_gemv_ex(d["x"], d["qweight"], d["scales"], d["zeros"], schedule=schedule))
    w4.check_device_status()
    m, n = c.sample(seed=K + schedule)
    ref, ref_abs = c.reference_at(orc, m, n)
    check_close(y[m, n], ref, ref_abs, 0.0, depth(K), f"{K}x{N} M={M} schedule={schedule}", xs_abs(c.x, c.sc, m, n))


def test_gemv_plan_choices():
    """Few row blocks: clusters of 2..8 CTAs that together cover at most the SMs; many row
    blocks: stream-K.  A forced schedule is honoured."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    sched, cl, ctas = w4.gemv_plan(1, 4096, 4096)
    assert sched == w4.GEMV_CLUSTER and 2 <= cl <= 8 and ctas % cl == 0 and ctas <= sms
    assert w4.gemv_plan(1, 28672, 4096)[0] == w4.GEMV_STREAM_K
    assert w4.gemv_plan(16, 4096, 4096, w4.GEMV_STREAM_K) == (w4.GEMV_STREAM_K, 0, min(sms, 32 * 8))
    sched, cl, ctas = w4.gemv_plan(16, 57344, 8192, w4.GEMV_CLUSTER)
    assert sched == w4.GEMV_CLUSTER and 2 <= cl <= 8 and ctas % cl == 0


@pytest.mark.parametrize("schedule", [w4.GEMV_AUTO] + SCHEDULES, ids=["auto", "stream_k", "cluster"])
@pytest.mark.parametrize("K,N,M", [(4096, 28672, 1), (4096, 28672, 16), (14336, 4096, 4), (4096, 4096, 1),
                                   (4096, 6144, 9)])
def test_gemv_repeat_bit_identical(schedule, K, N, M):
    """Which CTA completes a split row block, and whether it fetched the other partial early,
    depends on timing; y must not.  Repeated calls give the same bits and leave the
    workspace counters at zero."""
    g = torch.Generator(device="cuda").manual_seed(K + N + M)
    qw = torch.randint(-2**31, 2**31 - 1, (N, K // 8), dtype=torch.int32, device="cuda", generator=g)
    sc = (torch.rand(K // 128, N, device="cuda", generator=g) * 0.02 + 0.001).half().view(torch.int16)
    z = torch.randint(-2**31, 2**31 - 1, (K // 128, N // 8), dtype=torch.int32, device="cuda", generator=g)
    x = torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16)
    need = w4.workspace_bytes(M, N, K)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    ys = [w4.w4a16_gemv_ex(x, qw, sc, z, workspace=ws, schedule=schedule) for _ in range(12)]
    w4.check_device_status()
    for y in ys[1:]:
        assert torch.equal(ys[0].view(torch.int16), y.view(torch.int16))
    counters = ws[need - 256 * ((N // 128 * 4 + 255) // 256):]
    assert int(counters.count_nonzero()) == 0


def test_linear_dispatches_to_gemv(orc):
    c = Case(orc, seed=12, K=2048, N=256, M=16, csr=True)
    d = c.device()
    a = gemv(d)
    b = gemv(d, w4.w4a16_linear)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_gemv_single_layer_full(orc):
    """4096 x 4096, M = 1, alpha = 0.5: the whole output against the oracle."""
    c = Case(orc, seed=workloads.seed_of(0, 0), K=4096, N=4096, M=1)
    y = host_bf16_as_f64(gemv(c.device()))
    ref, ref_abs = c.reference(orc)
    check_close(y, ref, ref_abs, 0.0, depth(c.K), "4096x4096 M=1", xs_abs(c.x, c.sc))


FULL = ([(1, i, K, N, M, False) for i, (_, K, N) in enumerate(workloads.LLAMA3_8B) for M in (1, 4, 8, 16)]
        + [(3, i, K, N, M, True) for i, (_, K, N) in enumerate(workloads.LLAMA2_13B) for M in (1, 16)]
        + [(4, i, K, N, 1, False) for i, (_, K, N) in enumerate(workloads.LLAMA2_70B)])


@pytest.mark.parametrize("cfg,i,K,N,M,csr", FULL, ids=[f"c{c}_{K}x{N}_M{M}" for c, _, K, N, M, _ in FULL])
def test_gemv_full_shapes_sampled(orc, cfg, i, K, N, M, csr):
    c = Case(orc, seed=workloads.seed_of(cfg, i), K=K, N=N, M=M, csr=csr)
    y = host_bf16_as_f64(gemv(c.device()))
    m, n = c.sample(seed=cfg * 10 + i)
    ref, ref_abs = c.reference_at(orc, m, n)
    check_close(y[m, n], ref, ref_abs, 0.0, depth(K), f"{K}x{N} M={M}", xs_abs(c.x, c.sc, m, n))


def test_bounded_wait_times_out_and_context_survives(orc):
    """A wait that can never complete gives up after its limit, reports TIMEOUT through the
    device status word, and leaves the context usable for the next GEMV."""
    import time
    t0 = time.perf_counter()
    w4.selftest_timeout(2_000_000)  # 2 ms
    with pytest.raises(w4.W4A16Error) as e:
        w4.check_device_status()
    assert e.value.code == w4.ERR_TIMEOUT
    assert time.perf_counter() - t0 < 5.0
    w4.check_device_status()  # cleared
    c = Case(orc, seed=77, K=1024, N=256, M=3)
    d = c.device()
    y = host_bf16_as_f64(w4.w4a16_gemv(d["x"], d["qweight"], d["scales"], d["zeros"]))
    w4.check_device_status()
    ref, ref_abs = c.reference(orc)
    check_close(y, ref, ref_abs, 0.0, depth(c.K), "after timeout", xs_abs(c.x, c.sc))
    with pytest.raises(w4.W4A16Error):
        w4.selftest_timeout(-1)


@pytest.mark.parametrize("schedule", SCHEDULES, ids=["stream_k", "cluster"])
def test_gemv_maximum_k(orc, schedule):
    """K = 2^20, the GEMV's largest K (2048 units per row block), on random packed weights:
    every output against the oracle."""
    K, N, M = 1 << 20, 128, 2
    rng = np.random.default_rng(20)
    qw = rng.integers(0, 2 ** 32, size=(N, K // 8), dtype=np.uint64).astype(np.uint32)
    sc = (rng.uniform(0.002, 0.02, size=(K // 128, N)).astype(np.float16)).view(np.uint16)
    z = rng.integers(0, 2 ** 32, size=(K // 128, N // 8), dtype=np.uint64).astype(np.uint32)
    x = workloads.uniform_bf16(21, (M, K))
    y = w4.w4a16_gemv_ex(dev_bf16(x), dev_bits(qw, torch.int32), dev_bits(sc, torch.int16), dev_bits(z, torch.int32),
                         schedule=schedule)
    w4.check_device_status()
    ref, ref_abs = orc.linear(x, qw, sc, z, N, with_abs=True)
    check_close(host_bf16_as_f64(y), ref, ref_abs, 0.0, depth(K), f"K=2^20 schedule={schedule}", xs_abs(x, sc))
