"""The Python binding's own argument checks: dtypes, strides and names that
the C ABI cannot see raise ValueError before any library call, and keep
doing so under ``python -O`` (they are not asserts).  CPU tensors, no GPU."""
import os
import subprocess
import sys

import pytest
import torch

import svdquant_w4a4_gemm_b200 as sv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BF16 = torch.bfloat16


def _weights(N=384, K=64):
    return sv.SvdqWeights(q_w=torch.zeros(N, K // 2, dtype=torch.uint8),
                          sf_w=torch.zeros(sv.scale_bytes(N, K), dtype=torch.uint8),
                          gs_w=torch.ones(1), L1t=torch.zeros(0, K, dtype=BF16),
                          L2t=torch.zeros(N, 0, dtype=BF16), smooth=None, bias=None)


def test_quantize_rejects_wrong_dtype_rank_and_column_stride():
    with pytest.raises(ValueError, match="bf16"):
        sv.quantize_act(torch.zeros(4, 64))
    with pytest.raises(ValueError, match="column stride"):
        sv.quantize_act(torch.zeros(64, 4, dtype=BF16).t())
    with pytest.raises(ValueError, match="2-D"):
        sv.quantize_act_dynamic(torch.zeros(4, 64, 2, dtype=BF16))


def test_dynamic_quantize_rejects_a_short_workspace():
    x = torch.zeros(4, 64, dtype=BF16)
    with pytest.raises(ValueError, match="workspace"):
        sv.quantize_act_dynamic(x, workspace=torch.zeros(sv.QUANTIZE_WORKSPACE_BYTES - 1, dtype=torch.uint8))


def test_linear_rejects_an_unknown_activation_and_mismatched_outputs():
    w = _weights()
    q = torch.zeros(4, 32, dtype=torch.uint8)
    with pytest.raises(ValueError, match="act="):
        sv.w4a4_linear(q, None, None, None, w, act="relu")
    with pytest.raises(ValueError, match="act="):
        sv.w4a4_linear_split(q, None, None, None, w, parts=3, act="silu")
    two = [torch.zeros(4, 128, dtype=BF16) for _ in range(2)]
    with pytest.raises(ValueError, match="parts"):
        sv.w4a4_linear_split(q, None, None, None, w, parts=3, ys=two)
    mixed = [torch.zeros(4, 128, dtype=BF16), torch.zeros(4, 136, dtype=BF16)[:, :128],
             torch.zeros(4, 128, dtype=BF16)]
    with pytest.raises(ValueError, match="leading dimension"):
        sv.w4a4_linear_split(q, None, None, None, w, parts=3, ys=mixed)


def test_awq_rejects_a_non_contiguous_activation():
    with pytest.raises(ValueError, match="contiguous bf16"):
        sv.awq_w4a16_linear(torch.zeros(64, 2, dtype=BF16).t(), None, None, None, None)


def test_checks_hold_under_python_O():
    code = ("import torch, svdquant_w4a4_gemm_b200 as sv\n"
            "try:\n"
            "    sv.quantize_act(torch.zeros(4, 64))\n"
            "except ValueError:\n"
            "    print('ValueError')\n")
    p = subprocess.run([sys.executable, "-O", "-c", code], cwd=ROOT, capture_output=True, text=True,
                       timeout=300)
    assert p.returncode == 0, p.stderr[-2000:]
    assert p.stdout.strip() == "ValueError"
