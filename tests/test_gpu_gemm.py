"""svdq_w4a4_linear (block-scaled tcgen05 FP4 GEMM + fused low-rank
up-projection + bias) against the oracle, through the C ABI.

Bar: max|err| <= 2e-2·rms(ref) and ||err||_F <= 5e-3·||ref||_F, ref = the
oracle's fp64 y from the same codes, scales and down-projection.  The FP4
products are exact in the tensor core, so the error is the fp32
accumulation order, the bf16 rounding of bf16(xl·gs_a·gs_w) in the low-rank
MMA (2^-9 relative on that term) and the bf16 output rounding (2^-9).

Two input routes are covered: (a) the oracle's activation codes and
down-projection fed straight to the GEMM (tests the GEMM alone), and
(b) the CUDA quantize call feeding the GEMM (the whole layer), compared with
the oracle's whole layer.  At full sizes the oracle evaluates a sample of
rows (every row of y is independent given the static activation scale).
"""
import functools

import numpy as np
import pytest
import torch

import workloads
from oracle import prep, svdq as osv
from tests._gpu import (assert_gelu_close, assert_gemm_close, bf16, f32, needs_gpu, prepared, u8,
                        weights_from_layer)

import svdquant_w4a4_gemm_b200 as sv

pytestmark = [pytest.mark.gpu, needs_gpu]


def _gemm_on_oracle_inputs(case, smooth=True, with_bias=True, act=None, bias=None):
    d, L = prepared(case, smooth=smooth, with_bias=with_bias)
    if bias is not None:
        L = dict(L, bias=bias)
    out = osv.svdq_forward(d["x"], L, act=act)
    w = weights_from_layer(L)
    r = case.r
    lora = f32(out["xl"]) if r else None
    y = sv.w4a4_linear(u8(out["packed"]), u8(out["sf_swizzled"]), f32([out["gs"]]), lora, w, act=act)
    torch.cuda.synchronize()
    if act is not None:
        return y, out["y"], osv.svdq_forward(d["x"], L)["y"]
    return y, out["y"]


# (M, K, N, r): BN=192 (N = 384) and BN=128 tiles, ragged M, ragged N tile, K not a
# multiple of 256 (short last stage), every rank
SMALL = [
    (128, 256, 256, 0),
    (128, 256, 128, 0),
    (128, 512, 256, 32),
    (256, 512, 512, 32),     # the tiny workload's shape
    (200, 512, 384, 16),
    (77, 320, 400, 64),
    (300, 1024, 256, 128),
    (129, 64, 16, 32),
]


@pytest.mark.parametrize("M,K,N,r", SMALL)
def test_gemm_small_oracle_inputs(M, K, N, r):
    case = workloads.small_case(M, K, N, r, seed=M * 7 + N + r)
    y, ref = _gemm_on_oracle_inputs(case)
    assert_gemm_close(y, ref, f"M{M} K{K} N{N} r{r}")


def test_gemm_no_bias_no_smoothing():
    case = workloads.small_case(256, 512, 256, 32, seed=3)
    y, ref = _gemm_on_oracle_inputs(case, smooth=False, with_bias=False)
    assert_gemm_close(y, ref, "no bias, no smoothing")


def test_zero_residual_gives_low_rank_branch_only():
    M, K, N, r = 128, 256, 256, 32
    rng = np.random.default_rng(1)
    L1t = workloads.to_bf16(rng.standard_normal((r, K)).astype(np.float32) * 0.1)
    L2t = workloads.to_bf16(rng.standard_normal((N, r)).astype(np.float32) * 0.1)
    x = workloads.to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    gs_w = osv.tensor_scale(0.0)
    cw, sfw = osv.nvfp4_quantize(np.zeros((N, K), np.float32), gs_w)
    from oracle import codecs
    L = dict(packed_w=codecs.pack_nibbles(cw), sf_w_swizzled=codecs.swizzle_scales(sfw), gs_w=gs_w,
             L1t=L1t, L2t=L2t, s=None, bias=None)
    q = osv.quantize_act(x, None)
    xl = osv.lora_down(x, None, L1t)
    y = sv.w4a4_linear(u8(q["packed"]), u8(q["sf_swizzled"]), f32([q["gs"]]), f32(xl), weights_from_layer(L))
    ref = osv.svdq_linear(q["codes"], q["sf"], q["gs"], xl, cw, sfw, gs_w, L2t, None)
    assert_gemm_close(y, ref, "R = 0")


# GELU(tanh) in the epilogue: both tile widths, a ragged M and N tail
@pytest.mark.parametrize("M,K,N,r", [(256, 512, 512, 32), (200, 512, 384, 16), (77, 320, 400, 64)])
def test_gemm_gelu_small(M, K, N, r):
    case = workloads.small_case(M, K, N, r, seed=M * 5 + N + r)
    y, ref, pre = _gemm_on_oracle_inputs(case, act="gelu")
    assert_gelu_close(y, ref, pre, f"GELU M{M} K{K} N{N} r{r}")


def test_gemm_gelu_saturating_range():
    # a bias ramp over [-12, 12] pushes the pre-activations through the
    # negative tail (GELU -> 0), the bend near 0 and the linear regime
    M, K, N, r = 256, 512, 384, 32
    case = workloads.small_case(M, K, N, r, seed=41)
    ramp = workloads.to_bf16(np.linspace(-12.0, 12.0, N).astype(np.float32))
    y, ref, pre = _gemm_on_oracle_inputs(case, act="gelu", bias=ramp)
    assert_gelu_close(y, ref, pre, "GELU over [-12, 12]")
    yn = y.float().cpu().numpy()
    assert (yn[:, :N // 8] <= 0).all() and (yn[:, :N // 8] > -0.2).all()  # far negative: tiny, non-positive


def test_whole_layer_tiny_workload():
    case = workloads.TINY
    d, L = prepared(case)
    gs = osv.act_tensor_scale(d["x"], L["s"])
    y = sv.svdq_linear(bf16(d["x"]), weights_from_layer(L), f32([gs]))
    torch.cuda.synchronize()
    ref = osv.svdq_forward(d["x"], L, gs)["y"]
    assert_gemm_close(y, ref, "tiny whole layer")


def test_whole_layer_dynamic_scale():
    case = workloads.small_case(333, 768, 256, 32, seed=12)
    d, L = prepared(case)
    y = sv.svdq_linear(bf16(d["x"]), weights_from_layer(L), None)
    torch.cuda.synchronize()
    ref = osv.svdq_forward(d["x"], L, None)["y"]
    assert_gemm_close(y, ref, "dynamic-scale whole layer")


# ------------------------------------------------------------ full sizes ----
_SVD = {}


@functools.lru_cache(maxsize=8)
def _full(case_name, r):
    case = {c.name: c for c in [workloads.ATTN, workloads.MLP_UP, *workloads.QKV.values()]}.get(case_name)
    if case is None:
        raise KeyError(case_name)
    d = workloads.draw_svdq(case)
    cache = _SVD.setdefault((case.seed, case.N, case.K), {})
    L = prep.prepare_svdq_layer(d["x_cal"], d["W"], d["bias"], r, svd_cache=cache)
    return d, L


def _whole_layer_sampled(d, L, x=None, step=16, act=None):
    x = d["x"] if x is None else x
    gs = osv.act_tensor_scale(x, L["s"])
    y = sv.svdq_linear(bf16(x), weights_from_layer(L), f32([gs]), act=act)
    torch.cuda.synchronize()
    rows = np.arange(0, x.shape[0], step)
    ref = osv.svdq_forward(x[rows], L, gs, act=act)["y"]
    if act is not None:
        return y[torch.from_numpy(rows).cuda()], ref, osv.svdq_forward(x[rows], L, gs)["y"]
    return y[torch.from_numpy(rows).cuda()], ref


def test_attn_projection_full_size():
    d, L = _full(workloads.ATTN.name, 32)
    y, ref = _whole_layer_sampled(d, L)
    assert_gemm_close(y, ref, "attn full")


def test_mlp_up_full_size():
    d, L = _full(workloads.MLP_UP.name, 32)
    y, ref = _whole_layer_sampled(d, L, step=32)
    assert_gemm_close(y, ref, "mlp up full")


def test_mlp_up_gelu_full_size():
    # the MLP up-projection as a DiT block runs it: GELU(tanh) fused into the epilogue
    d, L = _full(workloads.MLP_UP.name, 32)
    y, ref, pre = _whole_layer_sampled(d, L, step=32, act="gelu")
    assert_gelu_close(y, ref, pre, "mlp up + GELU full")


def test_mlp_down_full_size():
    case = workloads.MLP_DOWN
    d = workloads.draw_svdq(case)
    x = workloads.mlp_down_input()
    # calibrate the smoothing on the down-projection's own input distribution
    L = prep.prepare_svdq_layer(x[:256], d["W"], d["bias"], case.r)
    y, ref = _whole_layer_sampled(d, L, x=x, step=32)
    assert_gemm_close(y, ref, "mlp down full")


@pytest.mark.parametrize("r", [16, 32, 64, 128])
def test_fused_qkv_rank_sweep_full_size(r):
    d, L = _full(workloads.QKV[r].name, r)
    y, ref = _whole_layer_sampled(d, L, step=32)
    assert_gemm_close(y, ref, f"qkv r={r}")


def _random_operands(M, K, N, r, seed):
    """Oracle-quantized random operands (no SVD) for shapes with many tiles."""
    from oracle import codecs
    rng = np.random.default_rng(seed)
    x = workloads.to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    q = osv.quantize_act(x, None)
    R = rng.standard_normal((N, K)).astype(np.float32) * 0.05
    gs_w = osv.tensor_scale(np.abs(R).max())
    cw, sfw = osv.nvfp4_quantize(R, gs_w)
    L1t = workloads.to_bf16(rng.standard_normal((r, K)).astype(np.float32) * 0.05)
    L2t = workloads.to_bf16(rng.standard_normal((N, r)).astype(np.float32) * 0.2)
    bias = workloads.to_bf16(rng.standard_normal(N).astype(np.float32) * 0.01)
    xl = osv.lora_down(x, None, L1t)
    L = dict(packed_w=codecs.pack_nibbles(cw), sf_w_swizzled=codecs.swizzle_scales(sfw), gs_w=gs_w,
             L1t=L1t, L2t=L2t, s=None, bias=bias)
    return q, xl, cw, sfw, gs_w, L


@pytest.mark.parametrize("M,K,N,r", [(512, 1536, 20480, 32), (256, 3072, 10240, 64), (384, 2048, 9984, 128)])
def test_gemm_many_tiles_per_cta(M, K, N, r):
    # more output tiles than SMs, and more K steps than ring slots: every CTA
    # walks several tiles and the ring wraps inside each tile
    q, xl, cw, sfw, gs_w, L = _random_operands(M, K, N, r, seed=M + N)
    y = sv.w4a4_linear(u8(q["packed"]), u8(q["sf_swizzled"]), f32([q["gs"]]), f32(xl), weights_from_layer(L))
    torch.cuda.synchronize()
    cols = np.sort(np.random.default_rng(0).choice(N, 768, replace=False))
    ref = osv.svdq_linear(q["codes"], q["sf"], q["gs"], xl, cw[cols], sfw[cols], gs_w, L["L2t"][cols],
                          L["bias"][cols])
    assert_gemm_close(y[:, torch.from_numpy(cols).cuda()], ref, f"many tiles M{M} K{K} N{N} r{r}")


# ------------------------------------------------ split outputs (fused QKV) --
def _split_case(M, K, N, r, parts, seed, pad=0):
    case = workloads.small_case(M, K, N, r, seed=seed)
    d, L = prepared(case)
    out = osv.svdq_forward(d["x"], L)
    w = weights_from_layer(L)
    lora = f32(out["xl"]) if r else None
    args = (u8(out["packed"]), u8(out["sf_swizzled"]), f32([out["gs"]]), lora, w)
    n_part = N // parts
    ys = None
    if pad:  # each part a column slice of a wider buffer: ldy = n_part + pad
        big = [torch.full((M, n_part + pad), 7.0, dtype=torch.bfloat16, device="cuda") for _ in range(parts)]
        ys = [b[:, :n_part] for b in big]
    got = sv.w4a4_linear_split(*args, parts=parts, ys=ys)
    fused = sv.w4a4_linear(*args)
    torch.cuda.synchronize()
    if pad:
        for b in big:  # the padding columns are never written
            assert (b[:, n_part:].float() == 7.0).all()
    return got, fused, out["y"]


# (M, K, N, r, parts, pad): three parts of 128 (tile width 128 although N
# is a multiple of 192), three of 384 (192), two of 256 (128), ragged M, a
# padded leading dimension
SPLIT = [
    (200, 512, 384, 32, 3, 0),
    (256, 512, 1152, 16, 3, 0),
    (77, 320, 512, 64, 2, 24),
    (129, 256, 768, 32, 3, 8),
]


@pytest.mark.parametrize("M,K,N,r,parts,pad", SPLIT)
def test_split_outputs_small(M, K, N, r, parts, pad):
    got, fused, ref = _split_case(M, K, N, r, parts, seed=M + N + parts, pad=pad)
    n_part = N // parts
    # the output bar holds for y, which the parts store side by side (a part's
    # own rms can be too small a yardstick: on a 129 x 256 part the bf16
    # rounding of the exact result alone reaches 2.01e-2 of it)
    assert_gemm_close(torch.cat(got, dim=1), ref, f"parts of M{M} K{K} N{N} r{r}")
    same_tile = (n_part % 192 == 0) == (N % 192 == 0)
    for i, y in enumerate(got):
        cols = slice(i * n_part, (i + 1) * n_part)
        if same_tile:  # same tiling as the single-output call: the same bits
            assert torch.equal(y, fused[:, cols]), f"part {i} differs from the single-output call"


def test_fused_qkv_split_full_size():
    # the fused QKV projection: one quantized activation, one GEMM over
    # [W_q; W_k; W_v], Q, K and V stored in their own [M, 3072] tensors
    d, L = _full(workloads.QKV[32].name, 32)
    x = d["x"]
    gs = osv.act_tensor_scale(x, L["s"])
    w = weights_from_layer(L)
    q, sf, lora, gso = sv.quantize_act(bf16(x), w.smooth, w.L1t, f32([gs]))
    qkv = sv.w4a4_linear_split(q, sf, gso, lora, w, parts=3)
    fused = sv.w4a4_linear(q, sf, gso, lora, w)
    torch.cuda.synchronize()
    n_part = w.N // 3
    for i in range(3):
        assert torch.equal(qkv[i], fused[:, i * n_part:(i + 1) * n_part])
    rows = np.arange(0, x.shape[0], 64)
    ref = osv.svdq_forward(x[rows], L, gs)["y"]
    idx = torch.from_numpy(rows).cuda()
    assert_gemm_close(torch.cat([t[idx] for t in qkv], dim=1), ref, "qkv parts")


def test_split_with_gelu_matches_single_output():
    case = workloads.small_case(256, 512, 1152, 32, seed=77)
    d, L = prepared(case)
    out = osv.svdq_forward(d["x"], L)
    w = weights_from_layer(L)
    args = (u8(out["packed"]), u8(out["sf_swizzled"]), f32([out["gs"]]), f32(out["xl"]), w)
    parts = sv.w4a4_linear_split(*args, parts=3, act="gelu")
    whole = sv.w4a4_linear(*args, act="gelu")
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(parts, dim=1), whole)


def test_fused_prep_stacks_the_projections():
    from svdquant_w4a4_gemm_b200 import prep as dprep
    g = torch.Generator(device="cuda").manual_seed(3)
    Ws = [(torch.randn(n, 256, device="cuda", generator=g) * 0.02).to(torch.bfloat16) for n in (128, 128, 256)]
    bs = [torch.randn(128, device="cuda", generator=g).to(torch.bfloat16), None,
          torch.randn(256, device="cuda", generator=g).to(torch.bfloat16)]
    xc = torch.randn(64, 256, device="cuda", generator=g).to(torch.bfloat16)
    # r = 0: no SVD, so the stacked layer must match the concatenation bit for bit
    fused = dprep.prepare_svdq_fused(Ws, bs, xc, 0)
    whole = dprep.prepare_svdq(torch.cat(Ws), torch.cat([bs[0], torch.zeros(128, dtype=torch.bfloat16,
                                                                              device="cuda"), bs[2]]), xc, 0)
    ranked = dprep.prepare_svdq_fused(Ws, bs, xc, 16)
    torch.cuda.synchronize()
    assert fused.N == 512 and ranked.N == 512 and ranked.rank == 16
    for a, b in ((fused.q_w, whole.q_w), (fused.sf_w, whole.sf_w), (fused.bias, whole.bias),
                 (fused.smooth, whole.smooth)):
        assert torch.equal(a, b)
