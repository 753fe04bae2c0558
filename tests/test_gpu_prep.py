"""The library's on-device weight preparation (prep.py) against the oracle's
CPU preparation.

The two cannot agree bit for bit: the device takes a randomized SVD in fp32
(the oracle the exact one in fp64), rounds the residual to bf16 before
quantizing it with the library's own quantize call, and reduces the AWQ
channel means in another order.  A randomized SVD does not return the exact
top-r factors where the spectrum has no gap (the Gaussian bulk behind the
outlier directions): any r directions of a flat tail are equally good.  So
the device prep is held to what it must deliver:
- smoothing factors equal to the oracle's within fp32 rounding;
- a rank-r branch as good as the exact truncated SVD: its residual
  ||Ŵ − L2ᵀ·L1ᵀ||_F within 1 % of the oracle's (Eckart-Young optimal up
  to the bf16 rounding of the factors), and the same leading singular
  values (the outlier directions, which do have a gap) within 1 %;
- a layer as good as the oracle-prepared one: run through the same kernels,
  its error against the exact fp64 linear x·Wᵀ + b is within 10 % (+1e-3)
  of the oracle-prepared layer's error;
- AWQ: the same per-channel activation scale and, through the W4A16 kernel,
  the same accuracy against the exact linear.
"""
import numpy as np
import pytest
import torch

import workloads
from oracle import prep as oprep
from tests._gpu import bf16, f16, f32, needs_gpu, weights_from_layer

import svdquant_w4a4_gemm_b200 as sv
from svdquant_w4a4_gemm_b200 import prep as dprep

pytestmark = [pytest.mark.gpu, needs_gpu]


def _rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return np.linalg.norm(a - b) / np.linalg.norm(b)


@pytest.mark.parametrize("case", [workloads.TINY, workloads.small_case(384, 1024, 768, 64, seed=31)],
                         ids=["tiny", "r64"])
def test_device_svdq_prep_is_as_good_as_the_oracle_prep(case):
    d = workloads.draw_svdq(case)
    Lo = oprep.prepare_svdq_layer(d["x_cal"], d["W"], d["bias"], case.r)
    wd = dprep.prepare_svdq(bf16(d["W"]), bf16(d["bias"]), bf16(d["x_cal"]), case.r)
    wo = weights_from_layer(Lo)
    x = bf16(d["x"])
    y_dev = sv.svdq_linear(x, wd, None)
    y_orc = sv.svdq_linear(x, wo, None)
    torch.cuda.synchronize()
    sv.check_device_errors()
    s_dev = wd.smooth.cpu().numpy().astype(np.float64)
    assert np.abs(s_dev / Lo["s"].astype(np.float64) - 1).max() <= 1e-6
    P_dev = (wd.L2t.float() @ wd.L1t.float()).cpu().numpy().astype(np.float64)
    P_orc = Lo["L2t"].astype(np.float64) @ Lo["L1t"].astype(np.float64)
    What = np.asarray(d["W"], np.float64) * Lo["s"].astype(np.float64)[None, :]
    res_dev = np.linalg.norm(What - P_dev)
    res_orc = np.linalg.norm(What - P_orc)
    assert res_dev <= 1.01 * res_orc, (res_dev, res_orc)
    n_out = len(workloads.outlier_channels(case.K, case.outlier_frac, case.seed))
    sv_dev = np.linalg.svd(P_dev, compute_uv=False)[:n_out]
    sv_orc = np.linalg.svd(P_orc, compute_uv=False)[:n_out]
    assert np.abs(sv_dev / sv_orc - 1).max() <= 1e-2, (sv_dev, sv_orc)
    y_exact = d["x"].astype(np.float64) @ np.asarray(d["W"], np.float64).T + np.asarray(d["bias"], np.float64)
    e_dev = _rel(y_dev.float().cpu().numpy(), y_exact)
    e_orc = _rel(y_orc.float().cpu().numpy(), y_exact)
    assert e_orc < 0.1, e_orc
    assert e_dev <= 1.1 * e_orc + 1e-3, (e_dev, e_orc)


def test_device_awq_prep_is_as_good_as_the_oracle_prep():
    ac = workloads.AwqCase("prep", 4, 1024, 512, seed=9)
    da = workloads.draw_awq(ac)
    LA = oprep.prepare_awq_layer(da["x_cal"], da["W"], da["bias"])
    ainv, qw, sc, z = dprep.prepare_awq(bf16(da["W"]), bf16(da["x_cal"]))
    x = bf16(da["x"])
    b = bf16(da["bias"])
    y_dev = sv.awq_w4a16_linear(x, ainv, qw, sc, z, b)
    y_orc = sv.awq_w4a16_linear(x, f32(LA["act_scale_inv"]), torch.from_numpy(LA["qweight"].view(np.int32)).cuda(),
                                f16(LA["sc"]), f16(LA["z"]), b)
    torch.cuda.synchronize()
    assert np.abs(ainv.cpu().numpy().astype(np.float64) / LA["act_scale_inv"] - 1).max() <= 1e-5
    y_exact = da["x"].astype(np.float64) @ np.asarray(da["W"], np.float64).T + np.asarray(da["bias"], np.float64)
    e_dev = _rel(y_dev.float().cpu().numpy(), y_exact)
    e_orc = _rel(y_orc.float().cpu().numpy(), y_exact)
    assert e_orc < 0.1, e_orc
    assert e_dev <= 1.1 * e_orc + 1e-3, (e_dev, e_orc)
