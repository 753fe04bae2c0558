"""The device weight prep's randomized SVD (Halko, Martinsson and Tropp
2011, "Finding structure with randomness": a Gaussian range finder with
power iterations, then the SVD of the small projected matrix), pinned on
the CPU against matrices whose singular values are known by construction:
the claims of its docstring, each checked against the exact answer."""
import numpy as np
import pytest
import torch

from svdquant_w4a4_gemm_b200.prep import randomized_svd


def _matrix(K, N, sigma, seed):
    # A = U·diag(sigma)·Vᵀ with Haar-random orthonormal U [K, n], V [N, n]
    rng = np.random.default_rng(seed)
    n = len(sigma)
    U, _ = np.linalg.qr(rng.standard_normal((K, n)))
    V, _ = np.linalg.qr(rng.standard_normal((N, n)))
    return (U * sigma[None, :]) @ V.T, U, V


def _tail(sigma, r):
    return float(np.sqrt(np.sum(sigma[r:] ** 2)))


@pytest.mark.parametrize("r", [8, 32])
def test_a_spectrum_with_a_gap_is_recovered_to_fp32_accuracy(r):
    # r outlier directions well above a decaying tail (the SVDQuant case:
    # smoothing moves the activation outliers into a few weight directions)
    K, N = 384, 256
    sigma = np.concatenate([np.linspace(40.0, 20.0, r), 0.5 * 0.97 ** np.arange(N - r)])
    A, U, V = _matrix(K, N, sigma, seed=r)
    Ur, S, Vh = randomized_svd(torch.from_numpy(A).float(), r)
    Ur, S, Vh = Ur.double().numpy(), S.double().numpy(), Vh.double().numpy()
    np.testing.assert_allclose(S, sigma[:r], rtol=2e-5)
    # the same subspace: the top singular vectors up to sign
    np.testing.assert_allclose(np.abs(np.sum(Ur * U[:, :r], axis=0)), 1.0, atol=1e-4)
    np.testing.assert_allclose(np.abs(np.sum(Vh.T * V[:, :r], axis=0)), 1.0, atol=1e-4)
    np.testing.assert_allclose(Ur.T @ Ur, np.eye(r), atol=1e-5)
    # the rank-r residual is the Eckart-Young optimum (the tail energy)
    res = np.linalg.norm(A - (Ur * S[None, :]) @ Vh)
    assert res == pytest.approx(_tail(sigma, r), rel=1e-3)


def test_a_flat_tail_stays_within_a_fraction_of_a_percent_of_the_optimum():
    # no gap at all: singular values decay slowly across the whole spectrum
    K, N, r = 384, 256, 32
    sigma = 1.0 / np.sqrt(1.0 + np.arange(N))
    A, _, _ = _matrix(K, N, sigma, seed=7)
    Ur, S, Vh = (t.double().numpy() for t in randomized_svd(torch.from_numpy(A).float(), r))
    res = np.linalg.norm(A - (Ur * S[None, :]) @ Vh)
    opt = _tail(sigma, r)
    assert opt <= res * (1 + 1e-5)          # never below the optimum
    # within 0.2 % of it (one or two power iterations alone leave 1.9 % and 0.4 %)
    assert res <= opt * 1.002


def test_the_prep_is_repeatable():
    A = torch.from_numpy(_matrix(128, 96, np.linspace(5.0, 0.1, 96), seed=3)[0]).float()
    a = randomized_svd(A, 16)
    b = randomized_svd(A, 16)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_awq_prep_packs_and_quantizes_as_the_header_states():
    # nibble j of word w holds q[n, 8w + j] (an int32 view of the uint32
    # word, so words with the top nibble >= 8 are negative), zero points are
    # integers, and (q - z)·sc is within half a step of W·diag(a) (no code of
    # this draw meets the clamp to [0, 15], which could cost a step); the codes
    # are the oracle's int4 quantizer's on the same scaled weights, except
    # where fp32 and fp64 land on opposite sides of a rounding midpoint
    from oracle import awq as oawq
    from svdquant_w4a4_gemm_b200.prep import prepare_awq
    rng = np.random.default_rng(11)
    N, K = 48, 256
    W = torch.from_numpy((rng.standard_normal((N, K)) * 0.05).astype(np.float32)).to(torch.bfloat16)
    x_cal = torch.from_numpy(rng.standard_normal((64, K)).astype(np.float32)).to(torch.bfloat16)
    ainv, words, sc, z = prepare_awq(W, x_cal)
    assert words.dtype == torch.int32 and words.shape == (N, K // 8) and bool((words < 0).any())
    q = oawq.unpack_int4_words(words.numpy().view(np.uint32), K).astype(np.float64)
    zf, scf = z.double().numpy(), sc.double().numpy()
    assert np.all(zf == np.rint(zf)) and zf.min() >= 0 and zf.max() <= 15
    a = 1.0 / ainv.double().numpy()
    target = W.double().numpy() * a[None, :]
    deq = oawq.int4_dequantize(q.astype(np.uint8), sc.numpy(), z.numpy())
    step = np.repeat(scf, 64, axis=1)
    assert np.all(np.abs(deq - target) <= 0.5 * step * 1.01 + 1e-7)
    q_ref, _, _ = oawq.int4_quantize(W.float().numpy().astype(np.float64) * (1.0 / ainv.numpy()).astype(np.float64))
    assert np.mean(q_ref == q) > 0.999
