"""Pins for smoothing (Stage 2) and the SVD split (Stage 3) of the oracle:
closed forms, the Eckart-Young identity, orthonormality, an independent
power iteration, and a scalar-loop residual."""
import numpy as np

import workloads
from oracle import formats as F
from oracle import svdquant as S


def test_lambda_closed_form():
    X = np.array([[1.0, -4.0, 0.0], [2.0, 0.5, 0.0]], np.float32)
    W = np.array([[0.5, -1.0], [0.25, 0.0625], [3.0, 1.0]], np.float32)
    lam = S.smoothing_factors(X, W)
    # channel 0: sqrt(2 / 1); channel 1: sqrt(4 / 0.25) = 4; channel 2: X max is 0 -> 1
    assert lam.dtype == np.float32
    assert lam[0] == np.float32(np.sqrt(2.0)) and lam[1] == 4.0 and lam[2] == 1.0
    inv = S.inverse_lambda(lam)
    assert inv[1] == 0.25 and inv[0] == np.float32(1.0) / np.float32(np.sqrt(2.0))


def test_migration_preserves_product():
    """X^ W^ = X W: lambda divides X's columns and multiplies W's rows."""
    L = workloads.draw_layer("t", "nvfp4", 64, 128, 96, 8, seed=21, n_out=4)
    lam = S.smoothing_factors(L.X, L.W)
    Xh = S.smooth_activation(L.X, S.inverse_lambda(lam)).astype(np.float64)
    _, _, _, What = S.svd_split(L.W, lam, 8)
    ref = L.X.astype(np.float64) @ L.W.astype(np.float64)
    assert np.max(np.abs(Xh @ What - ref)) <= 1e-6 * np.max(np.abs(ref))
    # migration moves part of the outliers into the weight: with x20 activation
    # and x5 weight outliers, strength 0.5 gives lambda twice as large on the
    # outlier channels, so their peak-to-median ratio halves
    ax = np.abs(L.X).max(0)
    axh = np.abs(Xh).max(0)
    r0, r1 = ax.max() / np.median(ax), axh.max() / np.median(axh)
    assert r0 > 10 and 0.4 < r1 / r0 < 0.6


def test_eckart_young_and_orthonormality():
    L = workloads.draw_layer("t", "nvfp4", 64, 96, 160, 12, seed=22, n_out=4)
    lam = S.smoothing_factors(L.X, L.W)
    U, sig, Vt, What = S.svd_split(L.W, lam, 12)
    r = 12
    approx = (U * sig[:r]) @ Vt
    tail = np.sum(sig[r:] ** 2)
    err2 = np.sum((What - approx) ** 2)
    assert abs(err2 - tail) <= 1e-10 * np.sum(What ** 2)
    assert abs(np.sum(What ** 2) - np.sum(sig ** 2)) <= 1e-10 * np.sum(What ** 2)
    assert np.allclose(U.T @ U, np.eye(r), atol=1e-12)
    assert np.allclose(Vt @ Vt.T, np.eye(r), atol=1e-12)
    assert np.all(np.diff(sig) <= 0)
    # sign convention
    piv = np.argmax(np.abs(Vt), axis=1)
    assert np.all(Vt[np.arange(r), piv] > 0)


def test_top_singular_value_matches_power_iteration():
    L = workloads.draw_layer("t", "nvfp4", 32, 64, 80, 4, seed=23, n_out=3)
    lam = S.smoothing_factors(L.X, L.W)
    U, sig, Vt, What = S.svd_split(L.W, lam, 4)
    v = np.ones(What.shape[1])
    for _ in range(2000):
        v = What.T @ (What @ v)
        v /= np.linalg.norm(v)
    s1 = np.linalg.norm(What @ v)
    assert abs(s1 - sig[0]) <= 1e-9 * sig[0]
    assert abs(abs(v @ Vt[0]) - 1) <= 1e-6


def test_folded_factors_are_rounded_scaled_svd():
    L = workloads.draw_layer("t", "nvfp4", 48, 64, 64, 8, seed=24, n_out=3)
    lam = S.smoothing_factors(L.X, L.W)
    U, sig, Vt, _ = S.svd_split(L.W, lam, 8)
    L1f, L2, _ = S.svd_factors(L.W, lam, 8)
    L1 = U * sig[:8]
    want = L1 / lam.astype(np.float64)[:, None]
    # each L1f entry is the bf16 value nearest to lambda^-1 U Sigma
    assert np.all(np.abs(L1f - want) <= np.abs(want) * 2.0 ** -8 + 1e-300)
    assert np.array_equal(L1f, F.bf16_round(L1f))
    assert np.all(np.abs(L2 - Vt) <= np.abs(Vt) * 2.0 ** -8)


def _residual_loops(W, lam, L1f, L2):
    K, N = W.shape
    R = np.zeros((K, N), np.float32)
    for k in range(K):
        lk = float(lam[k])
        for n in range(N):
            s = 0.0
            for i in range(L1f.shape[1]):
                s = s + float(L1f[k, i]) * float(L2[i, n])
            R[k, n] = np.float32(lk * float(W[k, n]) - lk * s)
    return R


def test_residual_matches_scalar_loops_bit_for_bit():
    L = workloads.draw_layer("t", "nvfp4", 16, 16, 24, 4, seed=25, n_out=2)
    lam = S.smoothing_factors(L.X, L.W)
    L1f, L2, _ = S.svd_factors(L.W, lam, 4)
    R = S.residual(L.W, lam, L1f, L2)
    assert np.array_equal(R, _residual_loops(L.W, lam, L1f, L2))


def test_residual_norm_is_tail_energy():
    """||R||_F differs from sqrt(sum_{i>r} sigma_i^2) by at most the distance
    between the rounded and the exact rank-r product (triangle inequality)."""
    L = workloads.draw_layer("t", "nvfp4", 64, 128, 192, 16, seed=26, n_out=4)
    lam = S.smoothing_factors(L.X, L.W)
    U, sig, Vt, What = S.svd_split(L.W, lam, 16)
    L1f, L2, _ = S.svd_factors(L.W, lam, 16)
    R = S.residual(L.W, lam, L1f, L2).astype(np.float64)
    exact_lr = (U * sig[:16]) @ Vt
    rounded_lr = lam.astype(np.float64)[:, None] * (L1f @ L2)
    slack = np.linalg.norm(rounded_lr - exact_lr) + 1e-6 * np.linalg.norm(What)
    assert abs(np.linalg.norm(R) - np.sqrt(np.sum(sig[16:] ** 2))) <= slack
    # and the residual rebuilds W^ with the rounded factors
    assert np.max(np.abs(R + rounded_lr - What)) <= 1e-6 * np.max(np.abs(What))
