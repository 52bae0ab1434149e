"""The prefill launch's plan (CTA tile and split of K over a cluster),
computed on the host through w4_prefill_plan with given counts of resident
CTAs: no GPU needed."""
import ctypes
import itertools
import random

import pytest

import weight_only_int4_quantize_b200 as w4

# CTAs that run at once per tile shape (256x256, 128x256, 256x128, 128x128)
# and cluster size 1..4 on a B200: 148 SMs, one CTA per SM; clusters of 3 and
# 4 CTAs fit about 135 and 132 (a cluster stays inside one GPC).
B200 = [[148, 148, 135, 132]] * 4

# (N, K), M -> (tile rows, tile cols, K split): the fastest configuration, or
# one within 3 % of it, of a B200 sweep that timed every tile shape and split
# on these linears (27B-scale 5120 -> 17408, 17408 -> 5120, 5120 -> 10240;
# Llama-2-7B 4096 -> 4096, 4096 -> 11008, 11008 -> 4096; weights rotated over
# copies larger than twice L2).
SWEPT = [
    ((17408, 5120), 64, (128, 256, 2)),
    ((17408, 5120), 256, (256, 128, 1)),
    ((17408, 5120), 512, (256, 256, 1)),
    ((5120, 17408), 64, (128, 128, 3)),
    ((5120, 17408), 512, (256, 128, 3)),
    ((5120, 17408), 1024, (256, 128, 4)),
    ((5120, 17408), 2048, (256, 128, 2)),
    ((10240, 5120), 64, (128, 256, 3)),
    ((10240, 5120), 256, (256, 128, 3)),
    ((4096, 4096), 128, (128, 128, 4)),
    ((4096, 4096), 512, (256, 128, 2)),
    ((11008, 4096), 128, (128, 256, 3)),
    ((11008, 4096), 512, (256, 256, 1)),
    ((4096, 11008), 512, (256, 128, 2)),
]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    import os
    if not os.path.exists(w4.LIB_PATH):
        from weight_only_int4_quantize_b200 import build
        build.build()
    return w4.lib()


@pytest.mark.parametrize("shape,m,plan", SWEPT)
def test_plan_matches_swept_fastest(shape, m, plan):
    assert w4.prefill_plan([shape], m, B200) == plan


def test_grouped_plans():
    trio = [(17408, 5120), (5120, 17408), (10240, 5120)]
    llama = [(4096, 4096)] * 4 + [(11008, 4096)] * 2 + [(4096, 11008)]
    assert w4.prefill_plan(trio, 2048, B200) == (256, 256, 1)
    assert w4.prefill_plan(llama, 512, B200) == (256, 256, 1)
    assert w4.prefill_plan(llama, 2048, B200) == (256, 256, 1)
    # few rows: the group is split over clusters of 128-row tiles
    assert w4.prefill_plan(llama, 128, B200) == (128, 256, 2)


def _random_group(rng):
    n = rng.randint(1, 16)
    return [(rng.randint(1, 40000), 128 * rng.randint(1, 256)) for _ in range(n)]


def test_plans_respect_the_kernel_limits():
    """256-row tiles only when M fills them; a split leaves every CTA at least
    two 64-deep k-blocks and never applies to 256 x 256 tiles (their fp32
    partial tile does not fit the stage buffers)."""
    rng = random.Random(5)
    for _ in range(2000):
        shapes = _random_group(rng)
        m = rng.choice([1, 7, 33, 64, 100, 255, 256, 300, 512, 1000, 2048, 4096, 9000])
        rows, cols, ks = w4.prefill_plan(shapes, m, B200)
        assert rows in (128, 256) and cols in (128, 256) and 1 <= ks <= 4
        if rows == 256:
            assert m >= 256
        if ks > 1:
            assert min(k for _, k in shapes) // 64 >= 2 * ks
            assert (rows, cols) != (256, 256)


def test_plan_ignores_item_order():
    rng = random.Random(6)
    for _ in range(200):
        shapes = _random_group(rng)[:5]
        m = rng.choice([64, 512, 2048])
        plans = {w4.prefill_plan(list(p), m, B200) for p in itertools.permutations(shapes)}
        assert len(plans) == 1


def test_no_split_without_room_for_clusters():
    """With one resident CTA per cluster size > 1, a split only adds waves."""
    lone = [[148, 1, 1, 1]] * 4
    rng = random.Random(7)
    for _ in range(500):
        shapes = _random_group(rng)
        m = rng.choice([1, 64, 512, 4096])
        assert w4.prefill_plan(shapes, m, lone)[2] == 1


def test_plan_validation(_lib):
    f = _lib.w4_prefill_plan
    n1 = (ctypes.c_int64 * 17)(*([4096] * 17))
    k1 = (ctypes.c_int64 * 17)(*([4096] * 17))
    res = (ctypes.c_int * 16)(*([148] * 16))
    out = [ctypes.c_int() for _ in range(3)]
    o = [ctypes.byref(v) for v in out]
    assert f(n1, k1, 1, 64, res, *o) == 0
    assert f(None, k1, 1, 64, res, *o) == 1
    assert f(n1, k1, 1, 64, res, None, o[1], o[2]) == 1
    assert f(n1, k1, 0, 64, res, *o) == 1
    assert f(n1, k1, 17, 64, res, *o) == 1
    assert f(n1, k1, 1, 0, res, *o) == 2
    bad_k = (ctypes.c_int64 * 1)(100)
    assert f(n1, bad_k, 1, 64, res, *o) == 2
    bad_n = (ctypes.c_int64 * 1)(0)
    assert f(bad_n, k1, 1, 64, res, *o) == 2
    zero = (ctypes.c_int * 16)(*([148] * 15 + [0]))
    assert f(n1, k1, 1, 64, zero, *o) == 1
    with pytest.raises(ValueError):
        w4.prefill_plan([(4096, 4096)], 64, [[148] * 4] * 3)


def test_device_counts_need_a_device(_lib):
    """Without given counts the plan asks the current device; with no usable
    device the call returns W4_ERR_CUDA and launches nothing."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    n1 = (ctypes.c_int64 * 1)(4096)
    out = [ctypes.c_int() for _ in range(3)]
    assert _lib.w4_prefill_plan(n1, n1, 1, 64, None, *[ctypes.byref(v) for v in out]) == 6
