"""Offline weight preparation (the calibration step), on the CPU.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The pages describe this as the job of the quantization toolkit
(diffuse-compressor: inspect → calibrate/quantize → package; blog.margrop.com
"5. 自己量化一个模型", keryc.com "Cuantizando tus propios modelos"), with the
defaults rank 32 and precision nvfp4 (``--rank 32``; "nvfp4_r32").  The
tests use it to turn seeded raw draws into the prepared operands that both
the CUDA library and the oracle receive, so SVD round-off can never break
parity.  Readings (the pages give no formulas):

* smoothing s_k = sqrt(max_m|x_mk| / max_n|W_nk|), numerator and
  denominator clamped to ≥ 1e-5 (the SmoothQuant α = 0.5 form);
* truncated SVD of Ŵ = W·diag(s) in fp64; L1 = U_r·diag(√σ),
  L2 = diag(√σ)·V_rᵀ, each rounded to bf16 (the split of Σ does not change
  the product);
* the residual is taken against the bf16-rounded factors:
  R = Ŵ − fp64(L1)·fp64(L2);
* gs_w = 2688 / amax(fp32(R)), then R is quantized with the same NVFP4
  codec as the activations (groups of 16 along K).
* AWQ: a_k = mean_m(|x_cal[m,k]|)^0.5, normalised by sqrt(max a · min a),
  folded into the weight before int4 quantization.
"""

import numpy as np

from . import codecs, svdq, awq


def smoothing_factors(x, W, eps=1e-5):
    xmax = np.maximum(np.abs(np.asarray(x, dtype=np.float64)).max(axis=0), eps)
    wmax = np.maximum(np.abs(np.asarray(W, dtype=np.float64)).max(axis=0), eps)
    return np.sqrt(xmax / wmax).astype(np.float32)


def svd_of_smoothed(What):
    """Thin SVD of Whatᵀ (K×N) = U Σ Vᵀ in fp64."""
    return np.linalg.svd(np.asarray(What, dtype=np.float64).T, full_matrices=False)


def low_rank_factors(What, r, svd=None):
    """Truncated SVD of What [N, K] (nn.Linear layout, y = x·Whatᵀ).

    Returns (L1t [r, K], L2t [N, r]) as float32 arrays holding bf16 values:
    x·Whatᵀ ≈ (x·L1)·L2 with L1 = L1tᵀ (K×r) and L2 = L2tᵀ (r×N).
    ``svd`` may pass a precomputed ``svd_of_smoothed(What)``.
    """
    N, K = What.shape
    if r == 0:
        return np.zeros((0, K), np.float32), np.zeros((N, 0), np.float32)
    # Whatᵀ (K×N) = U Σ Vᵀ  ->  L1 = U_r √Σ (K×r), L2 = √Σ V_rᵀ (r×N)
    U, S, Vt = svd if svd is not None else svd_of_smoothed(What)
    root = np.sqrt(S[:r])
    L1 = U[:, :r] * root[None, :]
    L2 = root[:, None] * Vt[:r, :]
    return codecs.bf16_round(L1.T.astype(np.float32)), codecs.bf16_round(L2.T.astype(np.float32))


def prepare_svdq_layer(x_cal, W, bias, r, smooth=True, svd_cache=None):
    """Everything the W4A4 linear needs, from raw bf16 W [N, K] and x_cal.

    ``svd_cache``: optional dict; the SVD of the smoothed weight is stored in
    it under key "svd" and reused (for sweeping r over one weight)."""
    W = np.asarray(W, dtype=np.float64)
    N, K = W.shape
    s = smoothing_factors(x_cal, W) if smooth else None
    What = W * (s.astype(np.float64)[None, :] if s is not None else 1.0)
    svd = None
    if svd_cache is not None and r > 0:
        if "svd" not in svd_cache:
            svd_cache["svd"] = svd_of_smoothed(What)
        svd = svd_cache["svd"]
    L1t, L2t = low_rank_factors(What, r, svd)
    R = What - L2t.astype(np.float64) @ L1t.astype(np.float64)   # N×K
    R32 = R.astype(np.float32)
    gs_w = svdq.tensor_scale(np.abs(R32).max())
    codes_w, sf_w = svdq.nvfp4_quantize(R32, gs_w)
    return dict(s=s, L1t=L1t, L2t=L2t, R=R, gs_w=np.float32(gs_w), codes_w=codes_w,
                sf_w=sf_w, packed_w=codecs.pack_nibbles(codes_w),
                sf_w_swizzled=codecs.swizzle_scales(sf_w),
                bias=None if bias is None else np.asarray(bias, np.float32), W=W)


def awq_scales(x_cal, alpha=0.5):
    a = np.abs(np.asarray(x_cal, dtype=np.float64)).mean(axis=0) ** alpha
    a = np.maximum(a, 1e-8)
    return a / np.sqrt(a.max() * a.min())


def prepare_awq_layer(x_cal, W, bias, group=awq.GROUP):
    a = awq_scales(x_cal)
    Wt = np.asarray(W, dtype=np.float64) * a[None, :]
    q, sc, z = awq.int4_quantize(Wt, group)
    return dict(a=a, act_scale_inv=(1.0 / a).astype(np.float32), q=q, sc=sc, z=z,
                qweight=awq.pack_int4_words(q),
                bias=None if bias is None else np.asarray(bias, np.float32), W=W)
