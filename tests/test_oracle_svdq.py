"""Pins for oracle/svdq.py and oracle/prep.py against closed forms,
brute force, special cases and the pages' qualitative claim."""
import numpy as np
import pytest

import workloads
from oracle import codecs, prep, svdq


def _rng(s=0):
    return np.random.default_rng(s)


# ------------------------------------------------------- quantization ----
def test_block_round_trip_of_representable_values():
    # x = e2m1 value · 2^e with one group exponent; gs a power of two:
    # the group amax is 6·2^e, so t = 2^e·gs/ (6/6) is exactly representable
    rng = _rng(1)
    M, K = 8, 64
    codes = rng.integers(0, 16, (M, K)).astype(np.uint8)
    codes[:, ::16] = 7                     # every group holds ±6 → amax = 6·2^e
    e = rng.integers(-3, 4, (M, K // 16))
    x = codecs.e2m1_decode(codes) * np.repeat(2.0 ** e, 16, axis=1)
    gs = np.float32(4.0)
    got_codes, got_sf = svdq.nvfp4_quantize(x.astype(np.float32), gs)
    assert np.array_equal(got_codes & 0x7, codes & 0x7)
    assert np.array_equal(codecs.e4m3_decode(got_sf), 2.0 ** e * 4.0)
    assert np.array_equal(svdq.nvfp4_dequantize(got_codes, got_sf, gs), x)


def _nvfp4_groups_by_hand():
    from tests._golden import rows
    groups, cur = [], None
    for r in rows("nvfp4_groups_by_hand.txt"):
        if r[0] == "case":
            kv = dict(t.split("=", 1) for t in r[2:])
            cur = dict(name=r[1], gs=np.float32(kv["gs"]), sf=int(kv["sf"], 16), x=[], codes=[])
            groups.append(cur)
        else:
            cur["x"].append(np.float32(r[0]))
            cur["codes"].append(int(r[1], 16))
    return groups


@pytest.mark.parametrize("g", _nvfp4_groups_by_hand(), ids=lambda g: g["name"])
def test_quantize_matches_hand_quantized_groups(g):
    # groups off the representable grid (a block scale between E4M3 points,
    # elements between E2M1 points, saturation of both, a scale rounding to
    # zero), so that a misplaced tensor scale (t = a/(6·gs), inv = d/gs), a
    # dropped rounding step or a lost sign changes the bytes
    x = np.zeros((1, 16), np.float32)
    n = len(g["x"])
    x[0, :n] = g["x"]
    codes, sf = svdq.nvfp4_quantize(x, g["gs"])
    assert int(sf[0, 0]) == g["sf"]
    assert codes[0, :n].tolist() == g["codes"]
    assert np.all(codes[0, n:] == 0)


def test_quantization_error_within_format_bound():
    rng = _rng(2)
    x = workloads.to_bf16(rng.standard_normal((64, 256)).astype(np.float32) * 3)
    q = svdq.quantize_act(x, None)
    deq = svdq.nvfp4_dequantize(q["codes"], q["sf"], q["gs"])
    d = codecs.e4m3_decode(q["sf"])
    step = np.repeat(d / np.float64(q["gs"]), 16, axis=1)   # one E2M1 unit, in x units
    v = np.abs(x.astype(np.float64)) / step                 # magnitude in E2M1 units
    half_gap = np.where(v < 2, 0.25, np.where(v < 4, 0.5, 1.0))
    bound = half_gap * step + np.maximum(v - 6, 0) * step + 1e-6 * step
    assert np.all(np.abs(deq - x) <= bound)


def test_tensor_scale_puts_the_amax_group_at_448():
    x = workloads.to_bf16(_rng(3).standard_normal((32, 128)).astype(np.float32))
    q = svdq.quantize_act(x, None)
    assert q["gs"] == np.float32(2688) / np.float32(np.abs(x).max())
    assert (q["sf"] == 0x7E).sum() >= 1
    assert codecs.e4m3_decode(q["sf"]).max() == 448.0


def test_zero_groups_give_zero_scale_and_signed_zero_codes():
    x = np.zeros((2, 32), np.float32)
    x[0, :16] = -0.0
    x[1, 16:] = 1.0
    q = svdq.quantize_act(x, None)
    assert q["sf"][0].tolist() == [0, 0] and q["sf"][1, 0] == 0
    assert np.all(q["codes"][0, :16] == 8) and np.all(q["codes"][0, 16:] == 0)
    assert np.all(q["codes"][1, 16:] == 7)   # 1.0 · 2688 / 448 → 6
    assert svdq.tensor_scale(0.0) == 1.0


def test_all_zero_tensor_scale_is_one():
    q = svdq.quantize_act(np.zeros((4, 16), np.float32), None)
    assert q["gs"] == 1.0 and not q["sf"].any() and not q["codes"].any()


def test_unit_smoothing_equals_no_smoothing_and_smoothing_divides():
    x = workloads.to_bf16(_rng(4).standard_normal((16, 64)).astype(np.float32))
    a = svdq.quantize_act(x, None, np.float32(100))
    b = svdq.quantize_act(x, np.ones(64, np.float32), np.float32(100))
    assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["sf"], b["sf"])
    s = np.full(64, 2.0, np.float32)              # power of two: exact halving
    c = svdq.quantize_act(x, s, np.float32(100))
    assert np.array_equal(c["xh"], x / 2)


# --------------------------------------------------------- contractions ----
def _brute_y(ca, sfa, gsa, xl, cw, sfw, gsw, L2t, bias):
    M, K = ca.shape
    N = cw.shape[0]
    y = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                a = codecs.e2m1_decode(ca[m, k]) * codecs.e4m3_decode(sfa[m, k // 16]) / float(gsa)
                w = codecs.e2m1_decode(cw[n, k]) * codecs.e4m3_decode(sfw[n, k // 16]) / float(gsw)
                acc += a * w
            for j in range(xl.shape[1]):
                acc += float(xl[m, j]) * float(L2t[n, j])
            y[m, n] = acc + float(bias[n])
    return y


def test_svdq_linear_equals_triple_loop_on_tiny_shapes():
    rng = _rng(6)
    M, K, N, r = 3, 32, 5, 2
    ca = rng.integers(0, 16, (M, K)).astype(np.uint8)
    cw = rng.integers(0, 16, (N, K)).astype(np.uint8)
    sfa = rng.integers(0, 0x7F, (M, K // 16)).astype(np.uint8)
    sfw = rng.integers(0, 0x7F, (N, K // 16)).astype(np.uint8)
    xl = rng.standard_normal((M, r))
    L2t = rng.standard_normal((N, r))
    bias = rng.standard_normal(N)
    ref = _brute_y(ca, sfa, 3.0, xl, cw, sfw, 5.0, L2t, bias)
    got = svdq.svdq_linear(ca, sfa, np.float32(3), xl, cw, sfw, np.float32(5), L2t, bias)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_gelu_tanh_special_values_and_identities():
    g = svdq.gelu_tanh
    assert g(0.0) == 0.0
    # tanh is odd, so g(v) - g(-v) = v exactly in real arithmetic
    v = np.linspace(-9, 9, 361)
    np.testing.assert_allclose(g(v) - g(-v), v, rtol=0, atol=1e-13)
    # saturated tails: the identity above and the zero tail
    assert abs(g(30.0) - 30.0) < 1e-12 and abs(g(-30.0)) < 1e-12
    # slope 1/2 at the origin, from the series g(v) = v/2 + c·v²/2 + O(v⁴), c = √(2/π)
    h = 1e-6
    assert abs((g(h) - g(-h)) / (2 * h) - 0.5) < 1e-9
    assert abs((g(h) + g(-h)) / (h * h) - np.sqrt(2 / np.pi)) < 1e-5


def test_gelu_tanh_is_the_tanh_form_and_close_to_exact_gelu():
    import math
    import torch
    v = np.linspace(-8, 8, 2001)
    lib = torch.nn.functional.gelu(torch.from_numpy(v), approximate="tanh").numpy()
    np.testing.assert_allclose(svdq.gelu_tanh(v), lib, rtol=1e-14, atol=1e-15)
    exact = np.array([0.5 * t * (1 + math.erf(t / math.sqrt(2))) for t in v])
    err = np.abs(svdq.gelu_tanh(v) - exact)
    assert err.max() < 1e-3 and err.max() > 1e-5  # an approximation of Φ, not Φ itself


def test_gelu_is_applied_after_the_bias():
    rng = _rng(9)
    M, K, N, r = 2, 32, 3, 1
    ca = rng.integers(0, 16, (M, K)).astype(np.uint8)
    cw = rng.integers(0, 16, (N, K)).astype(np.uint8)
    sfa = rng.integers(0, 0x7F, (M, K // 16)).astype(np.uint8)
    sfw = rng.integers(0, 0x7F, (N, K // 16)).astype(np.uint8)
    xl, L2t, bias = rng.standard_normal((M, r)), rng.standard_normal((N, r)), rng.standard_normal(N) * 5
    pre = _brute_y(ca, sfa, 3.0, xl, cw, sfw, 5.0, L2t, bias)
    got = svdq.svdq_linear(ca, sfa, np.float32(3), xl, cw, sfw, np.float32(5), L2t, bias, act="gelu")
    import math
    want = np.vectorize(lambda t: 0.5 * t * (1 + math.tanh(math.sqrt(2 / math.pi) * (t + 0.044715 * t ** 3))))(pre)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
    with pytest.raises(ValueError):
        svdq.svdq_linear(ca, sfa, np.float32(3), xl, cw, sfw, np.float32(5), L2t, bias, act="relu")


def test_lora_down_equals_loop_over_k():
    rng = _rng(7)
    x = workloads.to_bf16(rng.standard_normal((3, 48)).astype(np.float32))
    s = (rng.uniform(0.5, 3.0, 48)).astype(np.float32)
    L1t = workloads.to_bf16(rng.standard_normal((4, 48)).astype(np.float32))
    got = svdq.lora_down(x, s, L1t)
    for m in range(3):
        for j in range(4):
            acc = 0.0
            for k in range(48):
                xh = np.float32(np.float32(x[m, k]) * np.float32(np.float32(1) / s[k]))
                acc += float(codecs.bf16_round(np.array([xh]))[0]) * float(L1t[j, k])
            assert got[m, j] == pytest.approx(acc, rel=1e-12, abs=1e-12)


def test_zero_residual_leaves_only_the_low_rank_branch():
    # W = rank-2 matrix exactly representable by the bf16 factors → R = 0
    rng = _rng(8)
    K, N, r, M = 64, 32, 2, 16
    L1t = workloads.to_bf16(rng.standard_normal((r, K)).astype(np.float32))
    L2t = workloads.to_bf16(rng.standard_normal((N, r)).astype(np.float32))
    bias = workloads.to_bf16(rng.standard_normal(N).astype(np.float32) * 0.01)
    R = np.zeros((N, K), np.float32)
    gs_w = svdq.tensor_scale(0.0)
    cw, sfw = svdq.nvfp4_quantize(R, gs_w)
    x = workloads.to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    q = svdq.quantize_act(x, None)
    xl = svdq.lora_down(x, None, L1t)
    y = svdq.svdq_linear(q["codes"], q["sf"], q["gs"], xl, cw, sfw, gs_w, L2t, bias)
    expect = codecs.bf16_round(x).astype(np.float64) @ L1t.T.astype(np.float64) @ L2t.T.astype(np.float64) + bias
    np.testing.assert_allclose(y, expect, rtol=1e-12, atol=1e-12)
    assert gs_w == 1.0 and not sfw.any()


def test_rank_zero_is_plain_nvfp4_gemm():
    case = workloads.small_case(64, 128, 48, 0, seed=9)
    d = workloads.draw_svdq(case)
    layer = prep.prepare_svdq_layer(d["x_cal"], d["W"], d["bias"], 0)
    out = svdq.svdq_forward(d["x"], layer)
    A = svdq.nvfp4_dequantize(out["codes"], out["sf"], out["gs"])
    W = svdq.nvfp4_dequantize(layer["codes_w"], layer["sf_w"], layer["gs_w"])
    np.testing.assert_allclose(out["y"], A @ W.T + d["bias"], rtol=1e-12, atol=1e-12)
    # and with no low-rank branch the residual is the whole smoothed weight
    np.testing.assert_allclose(layer["R"], d["W"].astype(np.float64) * layer["s"].astype(np.float64)[None, :], rtol=1e-12)


def test_prepared_layer_reconstructs_the_weight():
    case = workloads.small_case(64, 128, 64, 16, seed=10)
    d = workloads.draw_svdq(case)
    L = prep.prepare_svdq_layer(d["x_cal"], d["W"], d["bias"], 16)
    recon = (L["L2t"].astype(np.float64) @ L["L1t"].astype(np.float64) + L["R"]) / L["s"][None, :]
    np.testing.assert_allclose(recon, d["W"], rtol=1e-10, atol=1e-12)
    # the low-rank factors are the leading singular directions of Ŵ
    What = d["W"] * L["s"][None, :]
    sv = np.linalg.svd(What, compute_uv=False)
    assert np.linalg.norm(L["R"]) == pytest.approx(np.sqrt((sv[16:] ** 2).sum()), rel=2e-2)


def test_smoothing_factor_definition():
    x = np.array([[1.0, -8.0], [2.0, 0.5]], np.float32)
    W = np.array([[0.5, 0.02], [-0.25, 0.01]], np.float32)
    s = prep.smoothing_factors(x, W)
    np.testing.assert_allclose(s, [np.sqrt(2 / 0.5), np.sqrt(8 / 0.02)], rtol=1e-6)


def test_smoothing_balances_activation_and_weight_ranges():
    # the α = 0.5 balance the smoothing is chosen for: after x̂ = x·diag(1/s)
    # and Ŵ = W·diag(s), every input channel's activation max equals its
    # weight max (both sqrt(max|x_k| · max|W_k|)), and the product is unchanged
    rng = _rng(17)
    x = rng.standard_normal((64, 48)) * rng.uniform(0.1, 30.0, 48)[None, :]
    W = rng.standard_normal((40, 48)) * rng.uniform(0.001, 0.5, 48)[None, :]
    s = prep.smoothing_factors(x, W).astype(np.float64)
    xmax = np.abs(x / s[None, :]).max(axis=0)
    wmax = np.abs(W * s[None, :]).max(axis=0)
    np.testing.assert_allclose(xmax, wmax, rtol=1e-6)
    np.testing.assert_allclose((x / s[None, :]) @ (W * s[None, :]).T, x @ W.T, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("frac,mult", [(0.01, 20.0), (0.02, 30.0)])
def test_svd_branch_lowers_error_on_outlier_inputs(frac, mult):
    # the pages' central claim: plain W4A4 is hurt by outliers; SVDQuant's
    # low-rank branch absorbs them and lowers the error of the 4-bit layer
    case = workloads.SvdqCase("outlier", 256, 1024, 256, 32, frac, mult, seed=11)
    d = workloads.draw_svdq(case)
    exact = d["x"].astype(np.float64) @ d["W"].T.astype(np.float64) + d["bias"]
    err = {}
    for r in (0, 32):
        L = prep.prepare_svdq_layer(d["x_cal"], d["W"], d["bias"], r)
        y = svdq.svdq_forward(d["x"], L)["y"]
        err[r] = np.linalg.norm(y - exact) / np.linalg.norm(exact)
    # and the un-smoothed plain W4A4 layer is the worst of all
    L0 = prep.prepare_svdq_layer(d["x_cal"], d["W"], d["bias"], 0, smooth=False)
    e_plain = np.linalg.norm(svdq.svdq_forward(d["x"], L0)["y"] - exact) / np.linalg.norm(exact)
    assert err[32] < 0.8 * err[0], err
    assert err[32] < e_plain


def test_inv_smooth_is_the_correctly_rounded_reciprocal():
    # 1/s in fp64 is exact enough that one rounding to fp32 gives RN32(1/s):
    # for a 24-bit s, 1/s is never within 2^-49 of an fp32 midpoint
    s = _rng(21).uniform(1e-3, 1e3, 200000).astype(np.float32)
    got = svdq.inv_smooth(s, s.size)
    want = (1.0 / s.astype(np.float64)).astype(np.float32)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    assert np.array_equal(svdq.inv_smooth(None, 7), np.ones(7, np.float32))


def test_act_tensor_scale_puts_the_largest_group_at_448():
    rng = _rng(22)
    x = codecs.bf16_round((rng.standard_normal((96, 128)) * 3).astype(np.float32))
    s = rng.uniform(0.5, 2.0, 128).astype(np.float32)
    gs = svdq.act_tensor_scale(x, s)
    q = svdq.quantize_act(x, s, gs)
    assert codecs.e4m3_decode(q["sf"]).max() == 448.0   # the E4M3 maximum, exactly
    assert svdq.act_tensor_scale(np.zeros((4, 64), np.float32), None) == 1.0


def test_low_rank_factors_meet_the_eckart_young_bound():
    # any rank-r matrix leaves at least the tail singular energy; the bf16
    # factors may add at most their own rounding to it
    rng = _rng(23)
    N, K, r = 60, 40, 8
    signal = rng.standard_normal((N, r)) @ rng.standard_normal((r, K))
    What = signal + 1e-3 * rng.standard_normal((N, K))
    L1t, L2t = prep.low_rank_factors(What, r)
    assert L1t.shape == (r, K) and L2t.shape == (N, r)
    resid = np.linalg.norm(What - L2t.astype(np.float64) @ L1t.astype(np.float64))
    sig = np.linalg.svd(What, compute_uv=False)
    tail = np.sqrt(np.sum(sig[r:] ** 2))
    assert tail * (1 - 1e-12) <= resid <= tail + 8e-3 * np.linalg.norm(What)
    z1, z2 = prep.low_rank_factors(What, 0)
    assert z1.shape == (0, K) and z2.shape == (N, 0)


def test_svd_of_smoothed_reconstructs_the_transposed_weight():
    What = _rng(24).standard_normal((30, 20))
    U, S, Vt = prep.svd_of_smoothed(What)
    np.testing.assert_allclose((U * S[None, :]) @ Vt, What.T, atol=1e-12)
    np.testing.assert_allclose(U.T @ U, np.eye(U.shape[1]), atol=1e-12)
    assert np.all(np.diff(S) <= 0)


def test_awq_scales_follow_the_square_root_of_channel_means():
    rng = _rng(25)
    x = rng.standard_normal((128, 64)) * rng.uniform(0.01, 10.0, 64)[None, :]
    a = prep.awq_scales(x)
    m = np.abs(x).mean(axis=0)
    ratio = a / np.sqrt(m)
    np.testing.assert_allclose(ratio, ratio[0], rtol=1e-12)   # a_k ∝ mean|x_k|^(1/2)
    assert a.max() * a.min() == pytest.approx(1.0, rel=1e-12)


def test_bf16_bit_helpers_match_torch():
    import torch
    x = (_rng(26).standard_normal(20000) * 100).astype(np.float32)
    t = torch.from_numpy(x).to(torch.bfloat16)
    assert np.array_equal(codecs.bf16_bits(x), t.view(torch.int16).numpy().view(np.uint16))
    assert np.array_equal(codecs.bf16_from_bits(codecs.bf16_bits(x)), t.float().numpy())
