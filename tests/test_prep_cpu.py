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
