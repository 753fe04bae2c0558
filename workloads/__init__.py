"""Seeded synthetic workloads shared by the tests, the bench and the oracle.

This module holds NO arithmetic of the method (no smoothing, SVD or
quantization): only shapes and seeded random draws of the raw layer
operands, rounded to their storage dtype (bf16).  Both the CUDA side and
the oracle side start from these arrays.

The shapes stand in for the diffusion-transformer layers that the pages
benchmark (ERNIE-Image-Turbo at 1024x1024; "Bringing Nunchaku 4-bit
Diffusion Inference to Diffusers", benchmark section): a 1024x1024 image in
a 2x2-patch latent gives 4096 image tokens; the hidden size 3072 and MLP
ratio 4 are those of common DiT blocks.  The real weights and prompts are
not available, so the values are Gaussian with a few outlier channels, the
structure the pages give as the reason W4A4 is hard (blog.margrop.com
"技术细节 §1": large outliers in activations and weights).

Draw recipe (numpy PCG64, fp32 draws, then bf16 round-to-nearest-even):
* x ~ N(0, 1) [M, K]; ``max(1, round(frac·K))`` input channels chosen by a
  seeded permutation are multiplied by ``mult`` before rounding;
* W ~ N(0, 0.02²) [N, K] (nn.Linear layout); bias ~ N(0, 0.01²) [N];
* a separate calibration draw x_cal (256 rows, same outlier channels).
"""

from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class SvdqCase:
    name: str
    M: int
    K: int
    N: int
    r: int
    outlier_frac: float = 0.01
    outlier_mult: float = 20.0
    seed: int = 0


@dataclass(frozen=True)
class AwqCase:
    name: str
    M: int
    K: int
    N: int
    group: int = 64
    seed: int = 4


# The five workloads.  Seeds: the tiny case uses 0; the others use their
# index (1..4); the MLP down-projection adds 100 to its index.
TINY = SvdqCase("tiny M256 K512 N512 r32", 256, 512, 512, 32, seed=0)
ATTN = SvdqCase("attn-proj M4096 K3072 N3072 r32", 4096, 3072, 3072, 32, seed=1)
MLP_UP = SvdqCase("mlp-up M4096 K3072 N12288 r32", 4096, 3072, 12288, 32, seed=2)
MLP_DOWN = SvdqCase("mlp-down M4096 K12288 N3072 r32", 4096, 12288, 3072, 32, seed=102)
QKV = {r: SvdqCase(f"fused-qkv M4608 K3072 N9216 r{r}", 4608, 3072, 9216, r,
                   outlier_frac=0.02, outlier_mult=30.0, seed=3) for r in (16, 32, 64, 128)}
AWQ = {m: AwqCase(f"awq-mod M{m} K3072 N18432 g64", m, 3072, 18432) for m in (1, 2, 8)}

HEADLINE = ATTN


def to_bf16(a):
    """fp32 array -> fp32 array holding the nearest bf16 values."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def outlier_channels(K, frac, seed):
    rng = np.random.Generator(np.random.PCG64(seed + 7919))
    n = max(1, int(round(frac * K)))
    return np.sort(rng.permutation(K)[:n])


def draw_activations(M, K, frac, mult, seed, stream=0):
    rng = np.random.Generator(np.random.PCG64([seed, stream]))
    x = rng.standard_normal((M, K), dtype=np.float32)
    if frac > 0:
        x[:, outlier_channels(K, frac, seed)] *= np.float32(mult)
    return to_bf16(x)


def draw_linear(N, K, seed):
    rng = np.random.Generator(np.random.PCG64([seed, 1]))
    W = rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02)
    b = rng.standard_normal((N,), dtype=np.float32) * np.float32(0.01)
    return to_bf16(W), to_bf16(b)


def draw_svdq(case, M=None):
    """Raw operands of one W4A4 layer: x [M,K], x_cal [256,K], W [N,K], bias [N]."""
    M = case.M if M is None else M
    x = draw_activations(M, case.K, case.outlier_frac, case.outlier_mult, case.seed, 0)
    x_cal = draw_activations(256, case.K, case.outlier_frac, case.outlier_mult, case.seed, 2)
    W, b = draw_linear(case.N, case.K, case.seed)
    return dict(x=x, x_cal=x_cal, W=W, bias=b)


def draw_awq(case):
    """Raw operands of one W4A16 layer (no outliers in the conditioning vector)."""
    x = draw_activations(case.M, case.K, 0.0, 1.0, case.seed, 10 + case.M)
    x_cal = draw_activations(256, case.K, 0.0, 1.0, case.seed, 2)
    W, b = draw_linear(case.N, case.K, case.seed)
    return dict(x=x, x_cal=x_cal, W=W, bias=b)


def small_case(M, K, N, r, seed=0, frac=0.01, mult=20.0):
    return SvdqCase(f"M{M} K{K} N{N} r{r}", M, K, N, r, frac, mult, seed)


def mlp_down_input(up_case=None):
    """Input of the MLP down-projection: bf16(GELU_tanh(x·W_upᵀ + b_up)).

    A realistic activation distribution for the down-projection workload,
    computed from the raw (unquantized) up-projection draws in fp32 on the
    CPU, so it depends on neither the CUDA library nor the oracle.
    """
    up_case = MLP_UP if up_case is None else up_case
    d = draw_svdq(up_case)
    x = torch.from_numpy(d["x"])
    W = torch.from_numpy(d["W"])
    b = torch.from_numpy(d["bias"])
    h = torch.nn.functional.gelu(x @ W.T + b, approximate="tanh")
    return h.to(torch.bfloat16).to(torch.float32).numpy()
