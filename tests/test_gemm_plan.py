"""The prefill GEMM's launch plan (host arithmetic, no GPU): token tile by M, split-K only for
grids of under two waves, runs of whole 128-k slices with no empty split, the partial-tile
bytes the workspace must hold, the caps, and the choices measured on B200."""
import itertools

import pytest

import w4a16_gemm_awq_b200 as w4

MIB = 1 << 20


def tiles_of(M, N, bn):
    return (N // 128) * ((M + bn - 1) // bn)


@pytest.mark.parametrize("M,N,K,sms", list(itertools.product(
    [17, 32, 33, 64, 65, 128, 129, 300, 512, 1024, 2048, 8192],
    [128, 256, 1024, 4096, 28672],
    [1024, 4096, 8192, 28672],
    [132, 148])))
def test_plan_invariants(M, N, K, sms):
    bn, splits, per, pbytes = w4.gemm_plan(M, N, K, sms)
    assert bn == (32 if M <= 32 else 64 if M <= 64 else 128 if M <= 128 else 256)
    nslices = K // 128
    tiles = tiles_of(M, N, bn)
    assert 1 <= splits <= 8
    assert splits * per >= nslices and (splits - 1) * per < nslices  # every split has work
    if splits == 1:
        assert per == nslices and pbytes == 0
    else:
        assert tiles < 2 * sms                      # only grids of under two waves split
        assert pbytes == tiles * splits * 128 * bn * 4 <= 64 * MIB
        assert per >= 4
        if bn == 256:
            assert tiles * splits <= sms            # wide tiles: one wave only


def test_plan_choices_measured_on_b200():
    # Llama-2-70B layers at M = 64 split (1.9x and 2.5x faster than unsplit)
    assert w4.gemm_plan(64, 8192, 8192, 148)[1] > 1
    assert w4.gemm_plan(64, 8192, 28672, 148)[1] > 1
    # 14336 x 4096 and 4096 x 4096 at M = 512: two splits in one wave
    assert w4.gemm_plan(512, 4096, 14336, 148)[1] == 2
    assert w4.gemm_plan(512, 4096, 4096, 148)[1] == 2
    # a second wave of wide split CTAs lost: these stay unsplit
    assert w4.gemm_plan(2048, 4096, 4096, 148)[1] == 1
    assert w4.gemm_plan(512, 6144, 4096, 148)[1] == 1
    assert w4.gemm_plan(1024, 5120, 5120, 148)[1] == 1
    # large grids never split
    assert w4.gemm_plan(4096, 8192, 8192, 148)[1] == 1
    assert w4.gemm_plan(64, 57344, 8192, 148)[1] == 1


def test_plan_rejects_bad_sizes():
    for args in [(0, 256, 1024, 148), (64, 100, 1024, 148), (64, 256, 1000, 148)]:
        with pytest.raises(w4.W4A16Error) as e:
            w4.gemm_plan(*args)
        assert e.value.code == w4.ERR_SHAPE
    with pytest.raises(w4.W4A16Error) as e:
        w4.gemm_plan(64, 256, 1024, 0)
    assert e.value.code == w4.ERR_VALUE
