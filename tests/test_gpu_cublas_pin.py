"""The NVFP4 encoding that crosses the boundary, pinned against an
independent implementation: cuBLASLt's block-scaled FP4 GEMM, reached
through torch's ``scaled_mm`` (E2M1 codes as ``float4_e2m1fn_x2``, E4M3
block scales as ``float8_e4m3fn`` with one scale per 16 elements in the
128x4 tiled layout).

The oracle writes packed codes (even k in the low nibble) and swizzled
scales by its own formula, the quantize kernel is bit-exact with it, and the
GEMM kernel reads the same arrangement, so a mistake shared by all three (a
transposed 32x4 order inside a tile, swapped nibbles) would pass every
parity test.  cuBLASLt reads the format as NVIDIA defines it; if it
reproduces the oracle's fp64 product from the oracle's bytes, and the
library's GEMM reproduces cuBLASLt from the quantize kernel's bytes, the
layout and the nibble order are the format's.  The pages name NVFP4 as the
Blackwell precision (blog.margrop.com "技术细节 §3", hardware table) but not
its byte layout, which is NVIDIA's (cuBLAS documentation, "1D Block Scaling
Factors Layout").
"""
import dataclasses

import numpy as np
import pytest
import torch

import workloads
from oracle import prep, svdq as osv
from tests._gpu import assert_gemm_close, bf16, f32, needs_gpu, u8, weights_from_layer

import svdquant_w4a4_gemm_b200 as sv

pytestmark = [pytest.mark.gpu, needs_gpu]


def _scale_view(buf, rows, K):
    rp, cp = -(-rows // 128) * 128, -(-(K // 16) // 4) * 4
    return buf.view(torch.float8_e4m3fn).reshape(rp, cp)


def cublas_nvfp4(qa, sfa, qw, sfw, M, N, K):
    """e2m1(A)·dec(sfa) · (e2m1(W)·dec(sfw))ᵀ by cuBLASLt, [M, N] (no tensor
    scales), in fp32 if cuBLASLt writes fp32 for this kind, else bf16.
    Tries torch's scaled_mm API, then the older ``_scaled_mm`` form; returns
    (y, which)."""
    a = qa.view(torch.float4_e2m1fn_x2)
    b = qw.view(torch.float4_e2m1fn_x2).t()          # [K/2, N], column-major
    sa, sb = _scale_view(sfa, M, K), _scale_view(sfw, N, K)
    errors = []
    F = torch.nn.functional
    for dt in (torch.float32, torch.bfloat16):
        try:
            y = F.scaled_mm(a, b, sa, F.ScalingType.BlockWise1x16, sb, F.ScalingType.BlockWise1x16,
                            swizzle_a=F.SwizzleType.SWIZZLE_32_4_4, swizzle_b=F.SwizzleType.SWIZZLE_32_4_4,
                            output_dtype=dt)
            return y, f"F.scaled_mm -> {dt}"
        except Exception as e:  # noqa: BLE001 - report every attempt if none works
            errors.append(f"F.scaled_mm {dt}: {e}")
        try:
            y = torch._scaled_mm(a, b, sa, sb, out_dtype=dt)
            return y, f"torch._scaled_mm -> {dt}"
        except Exception as e:  # noqa: BLE001
            errors.append(f"torch._scaled_mm {dt}: {e}")
    pytest.fail("no cuBLASLt NVFP4 entry in this torch: " + " | ".join(s[:300] for s in errors))


CASES = [dataclasses.replace(workloads.TINY, name="tiny M256 K512 N512 r0", r=0),
         workloads.SvdqCase("pin M384 K1024 N256 r0", 384, 1024, 256, 0, seed=7)]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c.name)
def test_oracle_bytes_read_by_cublaslt_give_the_oracle_product(case):
    """The oracle's packed codes and swizzled scales of both operands, read
    by cuBLASLt, give the oracle's own fp64 product dec(A)·dec(W)ᵀ (before
    the tensor scales) within the output bar."""
    d = workloads.draw_svdq(case)
    L = prep.prepare_svdq_layer(d["x_cal"], d["W"], None, 0)
    q = osv.quantize_act(d["x"], L["s"])
    M, N, K = case.M, case.N, case.K
    y, which = cublas_nvfp4(u8(q["packed"]), u8(q["sf_swizzled"]), u8(L["packed_w"]),
                            u8(L["sf_w_swizzled"]), M, N, K)
    ref = osv.svdq_linear(q["codes"], q["sf"], 1.0, None, L["codes_w"], L["sf_w"], 1.0, None, None)
    assert_gemm_close(y, ref, f"cuBLASLt ({which}) on the oracle's bytes")


@pytest.mark.parametrize("case", CASES, ids=lambda c: c.name)
def test_library_gemm_matches_cublaslt_on_the_quantize_kernels_bytes(case):
    """The quantize kernel's codes and scales with the oracle's weight bytes:
    the library's W4A4 GEMM at r = 0 without bias equals cuBLASLt's result
    times α = 1/(gs_a·gs_w) within the output bar.  Both are tensor-core sums
    of the same products, but with their own K order and internal
    accumulation (measured: up to ~7e-3·rms apart element-wise, far above
    two bf16 roundings), so the elements are held to the GEMM bar, not to a
    rounding bound; a wrong layout or nibble order gives errors of order the
    output's rms and fails it."""
    d = workloads.draw_svdq(case)
    L = prep.prepare_svdq_layer(d["x_cal"], d["W"], None, 0)
    w = weights_from_layer(L)
    gs_a = np.float32(osv.act_tensor_scale(d["x"], L["s"]))
    qa, sfa, _, gs = sv.quantize_act(bf16(d["x"]), w.smooth, None, f32([gs_a]))
    y_lib = sv.w4a4_linear(qa, sfa, gs, None, w)
    M, N, K = case.M, case.N, case.K
    y_cb, which = cublas_nvfp4(qa, sfa, w.q_w, w.sf_w, M, N, K)
    alpha = 1.0 / (np.float64(gs_a) * np.float64(L["gs_w"]))
    ref = y_cb.double().cpu().numpy() * alpha
    assert_gemm_close(y_lib, ref, f"library GEMM vs cuBLASLt ({which})")
    torch.cuda.synchronize()
    sv.check_device_errors()
