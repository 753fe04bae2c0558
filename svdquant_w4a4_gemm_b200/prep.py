"""Offline weight preparation on the device (what the pages' quantization
toolkit does before a checkpoint is packaged: calibrate, smooth, split off
the low-rank branch, quantize the residual; blog.margrop.com "5. 自己量化一个
模型"; keryc.com "Cuantizando tus propios modelos").  Not on the hot path.

* smoothing s_k = sqrt(max_m|x_cal[m,k]| / max_n|W[n,k]|) (clamped >= 1e-5);
* rank-r truncated SVD of Ŵ = W·diag(s) (fp32 on the device) by a
  randomized range finder (Halko, Martinsson and Tropp 2011, "Finding
  structure with randomness", Algorithms 4.4 and 5.1: a seeded Gaussian
  sketch with oversampling, a few power iterations re-orthonormalized by QR,
  then the SVD of the small projected matrix); Σ split evenly:
  L1 = U_r·√Σ, L2 = √Σ·V_rᵀ, stored bf16 as L1ᵀ [r, K] and L2ᵀ [N, r];
* residual R = Ŵ − L2ᵀ·L1ᵀ, gs_w = 2688 / max|R|, and R is NVFP4-quantized
  by this library's own ``svdq_quantize_act`` (R rounded to bf16 first);
* AWQ: a_k = mean_m|x_cal[m,k]|^0.5 / sqrt(max a · min a), W̃ = W·diag(a),
  asymmetric int4 per (row, group of 64) with fp16 scale and zero.
"""
import torch

from . import SvdqWeights, quantize_act


def randomized_svd(A, r, oversample=16, power_iters=4, seed=0):
    """Top-r singular triplets of A [K, N] (fp32): (U [K, r], S [r], Vh [r, N]).

    Sketch Y = A·Ω with Ω [N, r + p] Gaussian (seeded, so the prep is
    repeatable), q power iterations Y ← A·(Aᵀ·Y) with a QR after each
    product (keeps the small singular directions from drowning in
    round-off), Q = qr(Y), then the exact SVD of B = Qᵀ·A [(r + p), N] and
    U = Q·U_B.  The range error shrinks like (σ_{r+p+1}/σ_r)^(2q+1), so a
    spectrum with a clear gap after the outlier directions is found to fp32
    accuracy, and a flat tail to a residual within a fraction of a percent of
    the Eckart-Young optimum."""
    K, N = A.shape
    k = min(r + oversample, K, N)
    g = torch.Generator(device=A.device)
    g.manual_seed(seed)
    omega = torch.randn(N, k, generator=g, device=A.device, dtype=A.dtype)
    Q, _ = torch.linalg.qr(A @ omega)
    for _ in range(power_iters):
        Z, _ = torch.linalg.qr(A.T @ Q)
        Q, _ = torch.linalg.qr(A @ Z)
    Ub, S, Vh = torch.linalg.svd(Q.T @ A, full_matrices=False)
    return (Q @ Ub)[:, :r], S[:r], Vh[:r, :]


def prepare_svdq(W, bias, x_cal, r, smooth=True):
    """W [N, K] bf16, bias [N] bf16 or None, x_cal [*, K] bf16 -> SvdqWeights."""
    dev = W.device
    Wf = W.float()
    N, K = Wf.shape
    s = None
    if smooth:
        xmax = x_cal.float().abs().amax(dim=0).clamp_min(1e-5)
        wmax = Wf.abs().amax(dim=0).clamp_min(1e-5)
        s = (xmax / wmax).sqrt()
    What = Wf * (s[None, :] if s is not None else 1.0)
    if r > 0:
        U, S, Vh = randomized_svd(What.T.contiguous(), r)
        root = S[:r].sqrt()
        L1t = (U[:, :r] * root[None, :]).T.contiguous().to(torch.bfloat16)
        L2t = (root[:, None] * Vh[:r, :]).T.contiguous().to(torch.bfloat16)
        R = What - L2t.float() @ L1t.float()
    else:
        L1t = torch.zeros(0, K, dtype=torch.bfloat16, device=dev)
        L2t = torch.zeros(N, 0, dtype=torch.bfloat16, device=dev)
        R = What
    amax = R.abs().max()
    gs_w = torch.where(amax > 0, 2688.0 / amax, torch.ones_like(amax)).reshape(1).float()
    q_w, sf_w, _, _ = quantize_act(R.to(torch.bfloat16).contiguous(), None, None, gs_w)
    return SvdqWeights(q_w=q_w, sf_w=sf_w, gs_w=gs_w, L1t=L1t, L2t=L2t,
                       smooth=None if s is None else s.contiguous(),
                       bias=None if bias is None else bias.contiguous())


def prepare_svdq_fused(Ws, biases, x_cal, r, smooth=True):
    """One prepared layer for projections that read the same input (Q, K and V
    of an attention block): their weights stacked along N, [W_0; W_1; ...],
    smoothed, decomposed and quantized together, so one activation
    quantization serves all of them.  The output columns of part i are
    [Σ_{j<i} N_j, Σ_{j<=i} N_j); ``w4a4_linear_split`` stores them apart."""
    W = torch.cat(list(Ws), dim=0)
    bias = None
    if any(b is not None for b in biases):
        bias = torch.cat([b if b is not None else torch.zeros(Wi.shape[0], dtype=W.dtype, device=W.device)
                          for Wi, b in zip(Ws, biases)])
    return prepare_svdq(W, bias, x_cal, r, smooth=smooth)


def prepare_awq(W, x_cal, group=64):
    """W [N, K] bf16, x_cal [*, K] -> (act_scale_inv [K] fp32, qweight [N, K/8] int32,
    scales [N, K/64] fp16, zeros [N, K/64] fp16)."""
    a = x_cal.float().abs().mean(dim=0).clamp_min(1e-8).sqrt()
    a = a / (a.max() * a.min()).sqrt()
    Wt = W.float() * a[None, :]
    N, K = Wt.shape
    g = Wt.reshape(N, K // group, group)
    mn, mx = g.amin(dim=-1), g.amax(dim=-1)
    sc = ((mx - mn) / 15.0).half()
    sc = torch.where((mx == mn) | (sc == 0), torch.ones_like(sc), sc)
    z = (-mn / sc.float()).round().clamp(0, 15).half()
    q = ((g / sc.float()[..., None]).round() + z.float()[..., None]).clamp(0, 15).to(torch.int64)
    q = q.reshape(N, K // 8, 8)
    shifts = (4 * torch.arange(8, device=W.device, dtype=torch.int64))
    words = (q << shifts).sum(dim=-1)                     # < 2^32, exact in int64
    words = torch.where(words >= 2 ** 31, words - 2 ** 32, words).to(torch.int32)
    return (1.0 / a).float().contiguous(), words.contiguous(), sc.contiguous(), z.contiguous()
