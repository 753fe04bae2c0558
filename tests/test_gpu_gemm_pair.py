"""The W4A4 GEMM on SM pairs (256 x 192 or 256 x 128 tiles, tcgen05
cta_group::2; svdq_set_gemm_pairs(1), for M > 128) against the oracle,
through the C ABI, and against the one-SM kernel on the same inputs.

The bar is the GEMM bar of tests/test_gpu_gemm.py.  The shapes single out
what is new in the pair kernel: each SM's tensor memory must hold its own
128 rows' A scales and the B scales of all 192 columns (tile column offsets
0 and 64 inside a 128-row scale block), a pair whose second CTA lies wholly
or partly past M, a short last K step, several tiles per cluster, and the
low-rank operand of both SMs feeding one MMA.
"""
import numpy as np
import pytest
import torch

import workloads
from oracle import svdq as osv
from tests._gpu import assert_gemm_close, f32, needs_gpu, prepared, u8, weights_from_layer
from tests.test_gpu_gemm import _random_operands

import svdquant_w4a4_gemm_b200 as sv

pytestmark = [pytest.mark.gpu, needs_gpu]


# (M, K, N, r): first the simplest pair tile (one FP4 step, no low-rank
# step), then the low-rank branch, the second CTA past M (M = 384: two pairs,
# the last CTA holds no rows), ragged M inside the second CTA with a short
# last K step, several tiles along N (tile offsets 64 mod 128), every rank,
# M = 129 (one row in the second CTA, K = one 64-block), and 256 x 128 tiles
# (N a multiple of 128, not of 192)
PAIR = [
    (256, 256, 192, 0),
    (256, 512, 192, 32),
    (384, 1024, 384, 16),
    (200, 320, 576, 64),
    (640, 2048, 960, 128),
    (129, 64, 192, 32),
    (384, 512, 256, 32),
    (300, 1024, 640, 64),
]


def _run(case, pairs):
    d, L = prepared(case)
    out = osv.svdq_forward(d["x"], L)
    w = weights_from_layer(L)
    lora = f32(out["xl"]) if case.r else None
    prev = sv.set_gemm_pairs(pairs)
    try:
        y = sv.w4a4_linear(u8(out["packed"]), u8(out["sf_swizzled"]), f32([out["gs"]]), lora, w)
        torch.cuda.synchronize()
    finally:
        sv.set_gemm_pairs(prev)
    sv.check_device_errors()
    return y, out["y"]


@pytest.mark.parametrize("M,K,N,r", PAIR)
def test_pair_gemm_small(M, K, N, r):
    y, ref = _run(workloads.small_case(M, K, N, r, seed=M + K + N + r), True)
    assert_gemm_close(y, ref, f"pair M{M} K{K} N{N} r{r}")


@pytest.mark.parametrize("M,K,N,r", PAIR[1:4])
def test_pair_and_single_sm_kernels_agree(M, K, N, r):
    case = workloads.small_case(M, K, N, r, seed=M + K + N + r)
    y2, ref = _run(case, True)
    y1, _ = _run(case, False)
    assert_gemm_close(y1, ref, "one-SM kernel")
    assert_gemm_close(y2, ref, "pair kernel")
    # both round the same fp32 sums to bf16; only the summation order inside
    # the tensor core may differ
    diff = (y1.float() - y2.float()).abs().max().item()
    rms = float(np.sqrt(np.mean(ref ** 2)))
    assert diff <= 2e-2 * rms, diff


@pytest.mark.parametrize("M,K,N,r", [(2048, 1536, 9984, 32), (1152, 3072, 4608, 128), (768, 1024, 5120, 16)])
def test_pair_gemm_many_tiles_per_cluster(M, K, N, r):
    # more pair tiles than clusters and more K steps than ring slots
    q, xl, cw, sfw, gs_w, L = _random_operands(M, K, N, r, seed=M + N + 1)
    prev = sv.set_gemm_pairs(True)
    try:
        y = sv.w4a4_linear(u8(q["packed"]), u8(q["sf_swizzled"]), f32([q["gs"]]), f32(xl),
                           weights_from_layer(L))
        torch.cuda.synchronize()
    finally:
        sv.set_gemm_pairs(prev)
    sv.check_device_errors()
    cols = np.sort(np.random.default_rng(1).choice(N, 768, replace=False))
    ref = osv.svdq_linear(q["codes"], q["sf"], q["gs"], xl, cw[cols], sfw[cols], gs_w, L["L2t"][cols],
                          L["bias"][cols])
    assert_gemm_close(y[:, torch.from_numpy(cols).cuda()], ref, f"pair many tiles M{M} K{K} N{N} r{r}")


def test_pair_gemm_wait_times_out_cleanly_and_context_survives():
    """The host-side fault hook: both CTAs' producers skip the first ring
    slot, so the stagers' and the MMA thread's bounded waits run out; every
    role gives up, the pair still meets at its cluster barrier, frees its
    tensor memory and exits.  The next call is correct."""
    case = workloads.small_case(256, 512, 384, 32, seed=23)
    d, L = prepared(case)
    out = osv.svdq_forward(d["x"], L)
    w = weights_from_layer(L)
    args = (u8(out["packed"]), u8(out["sf_swizzled"]), f32([out["gs"]]), f32(out["xl"]), w)
    sv.check_device_errors()
    prev_p = sv.set_gemm_pairs(True)
    prev_t = sv.set_wait_timeout_ns(50_000_000)   # 50 ms
    prev_f = sv.lib().svdq_debug_set_fault(1)
    try:
        sv.w4a4_linear(*args)
        with pytest.raises(sv.SvdqError) as e:
            sv.check_device_errors()
        assert e.value.status == sv.DEVICE_TIMEOUT
    finally:
        sv.lib().svdq_debug_set_fault(prev_f)
        sv.set_wait_timeout_ns(prev_t)
    try:
        sv.check_device_errors()
        y = sv.w4a4_linear(*args)
        torch.cuda.synchronize()
    finally:
        sv.set_gemm_pairs(prev_p)
    assert_gemm_close(y, out["y"], "pair kernel after a timed-out launch")
