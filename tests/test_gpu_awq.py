"""awq_w4a16_linear against the oracle, through the C ABI.

Bar: max|err| <= 2e-2·rms(ref) and ||err||_F <= 5e-3·||ref||_F with the
oracle's fp64 y.  The kernel keeps q − z exact, splits x̂ into bf16 hi + lo
(~16 significant bits), accumulates in fp32 and rounds y to bf16 (2^-9
relative), so the bf16 output rounding dominates the error.
"""
import numpy as np
import pytest
import torch

import workloads
from oracle import awq as oawq, prep
from tests._gpu import assert_gemm_close, bf16, f16, f32, needs_gpu

import svdquant_w4a4_gemm_b200 as sv

pytestmark = [pytest.mark.gpu, needs_gpu]


def _run(case, with_bias=True, with_ainv=True):
    d = workloads.draw_awq(case)
    L = prep.prepare_awq_layer(d["x_cal"], d["W"], d["bias"])
    ainv = L["act_scale_inv"] if with_ainv else None
    bias = L["bias"] if with_bias else None
    qw = torch.from_numpy(L["qweight"].view(np.int32)).cuda()
    y = sv.awq_w4a16_linear(bf16(d["x"]), None if ainv is None else f32(ainv), qw, f16(L["sc"]),
                            f16(L["z"]), None if bias is None else bf16(bias))
    torch.cuda.synchronize()
    ref = oawq.awq_linear(d["x"], ainv, L["q"], L["sc"], L["z"], bias)
    return y, ref


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8])
def test_awq_small(M):
    case = workloads.AwqCase(f"awq M{M}", M, 512, 256, seed=40 + M)
    y, ref = _run(case)
    assert_gemm_close(y, ref, f"awq M={M}")


def test_awq_no_bias_no_scale():
    case = workloads.AwqCase("awq plain", 3, 1024, 128, seed=7)
    y, ref = _run(case, with_bias=False, with_ainv=False)
    assert_gemm_close(y, ref, "awq plain")


@pytest.mark.parametrize("M", [1, 2, 8])
def test_awq_modulation_full_size(M):
    y, ref = _run(workloads.AWQ[M])
    assert_gemm_close(y, ref, f"awq full M={M}")


def test_awq_zero_weights_give_bias():
    M, K, N = 2, 256, 64
    q = np.full((N, K), 5, np.uint8)
    z = np.full((N, K // 64), 5, np.float16)
    sc = np.full((N, K // 64), 0.01, np.float16)
    x = workloads.to_bf16(np.random.default_rng(0).standard_normal((M, K)).astype(np.float32))
    b = workloads.to_bf16(np.arange(N, dtype=np.float32) * 0.01)
    qw = torch.from_numpy(oawq.pack_int4_words(q).view(np.int32)).cuda()
    y = sv.awq_w4a16_linear(bf16(x), None, qw, f16(sc), f16(z), bf16(b))
    assert np.array_equal(y.float().cpu().numpy(), np.broadcast_to(b, (M, N)))


# (M, K, N): the streaming kernel's edge cases — one 128-byte chunk per row
# (4 groups: warps 4-11 hold no K range), groups not a multiple of 12 (warps
# with 2 and 3 groups), the largest K held in registers (3072: 4 groups per
# warp) with one and with two B tiles, more strips than SMs (several strips
# per CTA and a ring that wraps), fewer strips than SMs, and 16 strips per CTA
# on 148 SMs (the most whose bias is staged)
STREAM = [
    (1, 256, 48),
    (6, 768, 80),
    (8, 3072, 2400),
    (4, 3072, 512),
    (2, 1024, 16),
    (7, 2048, 5984),
    (3, 512, 37888),
]


@pytest.mark.parametrize("M,K,N", STREAM)
def test_awq_stream_shapes(M, K, N):
    y, ref = _run(workloads.AwqCase(f"awq M{M} K{K} N{N}", M, K, N, seed=M + K + N))
    assert_gemm_close(y, ref, f"awq M={M} K={K} N={N}")
    sv.check_device_errors()


def test_awq_unaligned_scales_and_large_k_take_the_other_kernel():
    """Scales and zeros at a 2-byte offset (the bulk copies of the streaming
    kernel need 16-byte alignment), K not a multiple of 256 (its TMA box takes
    whole 128-byte chunks of a row), K above what it holds in registers
    (4096 and 5120: more than 4 groups per warp) and more than 16 strips of
    16 rows per SM go through the register-streaming kernel; all give the
    oracle's result."""
    for M, K, N, shift in ((3, 1024, 256, True), (5, 320, 64, False), (4, 4096, 512, False),
                           (8, 5120, 128, False), (2, 256, 16 * 17 * 148, False)):
        case = workloads.AwqCase(f"awq M{M} K{K}", M, K, N, seed=K + N)
        d = workloads.draw_awq(case)
        L = prep.prepare_awq_layer(d["x_cal"], d["W"], d["bias"])
        qw = torch.from_numpy(L["qweight"].view(np.int32)).cuda()
        sc, z = f16(L["sc"]), f16(L["z"])
        if shift:  # the same values, starting 2 bytes into a larger buffer
            big_s = torch.empty(sc.numel() + 1, dtype=sc.dtype, device=sc.device)
            big_z = torch.empty(z.numel() + 1, dtype=z.dtype, device=z.device)
            big_s[1:] = sc.flatten()
            big_z[1:] = z.flatten()
            sc, z = big_s[1:].view_as(sc), big_z[1:].view_as(z)
        y = sv.awq_w4a16_linear(bf16(d["x"]), f32(L["act_scale_inv"]), qw, sc, z, bf16(L["bias"]))
        torch.cuda.synchronize()
        ref = oawq.awq_linear(d["x"], L["act_scale_inv"], L["q"], L["sc"], L["z"], L["bias"])
        assert_gemm_close(y, ref, f"awq other kernel M={M} K={K}")
    sv.check_device_errors()
