"""Helpers shared by the GPU parity tests: moving oracle arrays to the
device, building the library's weight bundle from an oracle-prepared layer,
and the tolerances (all derived in the test docstrings)."""
import functools

import numpy as np
import pytest
import torch

import workloads
from oracle import prep

import svdquant_w4a4_gemm_b200 as sv

needs_gpu = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")

DEV = "cuda"


def bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(DEV).to(torch.bfloat16)


def f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(DEV)


def u8(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).to(DEV)


def f16(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float16)).to(DEV)


def weights_from_layer(L):
    return sv.SvdqWeights(
        q_w=u8(L["packed_w"]), sf_w=u8(L["sf_w_swizzled"]), gs_w=f32([L["gs_w"]]),
        L1t=bf16(L["L1t"]), L2t=bf16(L["L2t"]),
        smooth=None if L["s"] is None else f32(L["s"]),
        bias=None if L["bias"] is None else bf16(L["bias"]))


@functools.lru_cache(maxsize=16)
def prepared(case, smooth=True, with_bias=True):
    """Raw draws + oracle-prepared layer for a workload case (cached)."""
    d = workloads.draw_svdq(case)
    L = prep.prepare_svdq_layer(d["x_cal"], d["W"], d["bias"] if with_bias else None, case.r,
                                smooth=smooth)
    return d, L


def assert_gemm_close(y_gpu, y_ref, what=""):
    """The output bar: max|err| <= 2e-2·rms(ref) and ||err||_F <= 5e-3·||ref||_F."""
    y = y_gpu.float().cpu().numpy().astype(np.float64)
    err = y - y_ref
    rms = np.sqrt(np.mean(y_ref ** 2))
    rel_f = np.linalg.norm(err) / np.linalg.norm(y_ref)
    mx = np.abs(err).max() / rms
    assert np.isfinite(y).all(), f"{what}: non-finite outputs"
    assert mx <= 2e-2 and rel_f <= 5e-3, f"{what}: max|err|/rms={mx:.3e} relF={rel_f:.3e}"
    return mx, rel_f


GELU_MAX_SLOPE = 1.129  # max |d/dv GELU_tanh(v)|, reached near v = 1.42


def assert_gelu_close(y_gpu, y_ref, y_pre, what=""):
    """The output bar through GELU: the epilogue's error before the activation
    meets the plain bar, and GELU scales an error by at most its maximal slope,
    so max|err| <= 1.129 · 2e-2 · rms(pre-activation); the Frobenius bar stays
    relative to the GELU output itself, ||err||_F <= 5e-3·||ref||_F."""
    y = y_gpu.float().cpu().numpy().astype(np.float64)
    err = y - y_ref
    rms_pre = np.sqrt(np.mean(np.asarray(y_pre, dtype=np.float64) ** 2))
    rel_f = np.linalg.norm(err) / np.linalg.norm(y_ref)
    mx = np.abs(err).max() / rms_pre
    assert np.isfinite(y).all(), f"{what}: non-finite outputs"
    assert mx <= GELU_MAX_SLOPE * 2e-2 and rel_f <= 5e-3, \
        f"{what}: max|err|/rms(pre)={mx:.3e} relF={rel_f:.3e}"
    return mx, rel_f


def describe_byte_mismatch(got, ref):
    bad = np.nonzero(got != ref)[0]
    return f"{len(bad)} of {ref.size} bytes differ; first at {bad[:8].tolist()}: " \
           f"got {got[bad[:8]].tolist()} want {ref[bad[:8]].tolist()}"
