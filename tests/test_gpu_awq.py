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
