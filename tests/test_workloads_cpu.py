"""The seeded synthetic inputs follow the stated recipe: bf16 values drawn
repeatably from their seeds, max(1, round(frac·K)) outlier input channels
scaled by mult and shared by x and its calibration draw, W ~ N(0, 0.02²),
bias ~ N(0, 0.01²), no outliers in the AWQ conditioning vector, and the
five workloads at their stated shapes."""
import numpy as np
import pytest

import workloads as wl


def _is_bf16(a):
    return np.array_equal(a, wl.to_bf16(a))


def test_draws_are_repeatable_bf16_and_shaped():
    c = wl.small_case(128, 512, 256, 32, seed=5)
    a, b = wl.draw_svdq(c), wl.draw_svdq(c)
    for k in a:
        assert np.array_equal(a[k], b[k]) and _is_bf16(a[k]), k
    assert a["x"].shape == (128, 512) and a["x_cal"].shape == (256, 512)
    assert a["W"].shape == (256, 512) and a["bias"].shape == (256,)
    # x and its calibration draw are different draws
    assert not np.array_equal(a["x"][:128], a["x_cal"][:128])
    # another seed, other values
    assert not np.array_equal(a["W"], wl.draw_svdq(wl.small_case(128, 512, 256, 32, seed=6))["W"])


@pytest.mark.parametrize("frac,mult", [(0.01, 20.0), (0.02, 30.0)])
def test_outlier_channels_follow_the_recipe(frac, mult):
    K = 1024
    c = wl.small_case(512, K, 64, 32, seed=9, frac=frac, mult=mult)
    d = wl.draw_svdq(c)
    ch = wl.outlier_channels(K, frac, 9)
    assert len(ch) == max(1, round(frac * K)) and len(set(ch.tolist())) == len(ch)
    mask = np.zeros(K, bool)
    mask[ch] = True
    for x in (d["x"], d["x_cal"]):          # the same channels in both draws
        std = x.std(axis=0)
        assert np.all(np.abs(std[mask] / mult - 1) < 0.15)
        assert np.all(np.abs(std[~mask] - 1) < 0.15)
    assert len(wl.outlier_channels(64, 0.001, 0)) == 1   # at least one channel


def test_weight_and_bias_spreads():
    W, b = wl.draw_linear(512, 512, seed=3)
    assert abs(W.std() / 0.02 - 1) < 0.01 and abs(W.mean()) < 1e-4
    assert abs(b.std() / 0.01 - 1) < 0.1


def test_awq_conditioning_vector_has_no_outliers():
    d = wl.draw_awq(wl.AwqCase("t", 8, 512, 64))
    assert d["x"].shape == (8, 512) and d["x_cal"].shape == (256, 512)
    std = d["x_cal"].std(axis=0)
    assert np.all(np.abs(std - 1) < 0.25)


def test_the_five_workloads_have_their_stated_shapes():
    shape = lambda c: (c.M, c.K, c.N, c.r)  # noqa: E731
    assert shape(wl.TINY) == (256, 512, 512, 32)
    assert shape(wl.ATTN) == (4096, 3072, 3072, 32) and wl.HEADLINE is wl.ATTN
    assert shape(wl.MLP_UP) == (4096, 3072, 12288, 32)
    assert shape(wl.MLP_DOWN) == (4096, 12288, 3072, 32)
    assert sorted(wl.QKV) == [16, 32, 64, 128]
    for r, c in wl.QKV.items():
        assert shape(c) == (4608, 3072, 9216, r) and (c.outlier_frac, c.outlier_mult) == (0.02, 30.0)
    assert sorted(wl.AWQ) == [1, 2, 8]
    for m, c in wl.AWQ.items():
        assert (c.M, c.K, c.N, c.group) == (m, 3072, 18432, 64)
