"""Pins of the randomized-SVD oracle (oracle/rsvd.py): the counter-based
generator against its published known-answer vectors, exact recovery of a
matrix whose rank fits the sketch, near-optimality (Eckart-Young) on a
decaying spectrum and on the synthetic workload, orthonormal factors, and
the sign convention of the exact split."""
import numpy as np

import workloads
from conftest import read_golden
from oracle import rsvd as R
from oracle import svdquant as S


def test_philox_known_answers():
    for row in read_golden("philox4x32_10_kat.txt"):
        v = [int(x, 16) for x in row]
        out = R.philox4x32_10(np.array([v[:4]], np.uint64), v[4:6])[0]
        assert [int(x) for x in out] == v[6:10]


def test_rademacher_signs_follow_the_stream():
    X = R.rademacher(5, 7, seed=123)
    words = R.philox4x32_10(np.array([[b, 0, 0, 0] for b in range(9)], np.uint64), (123, 0)).reshape(-1)
    assert np.array_equal(X.reshape(-1), np.where(words[:35] >> 31 == 0, 1.0, -1.0))
    big = R.rademacher(200, 50)
    assert set(np.unique(big)) == {-1.0, 1.0} and abs(big.mean()) < 0.02


def _orth(rng, n, k):
    return np.linalg.qr(rng.standard_normal((n, k)))[0]


def test_exact_recovery_when_the_rank_fits_the_sketch():
    rng = np.random.default_rng(0)
    K, N, k = 300, 200, 20
    sig = np.linspace(5.0, 1.0, k)
    A = _orth(rng, K, k) @ np.diag(sig) @ _orth(rng, N, k).T
    U, s, Vt = R.randomized_svd(A, k)
    assert np.allclose(s[:k], sig, rtol=1e-12, atol=0)
    assert np.allclose(U @ np.diag(s[:k]) @ Vt, A, rtol=0, atol=1e-12 * np.abs(A).max())
    assert np.allclose(U.T @ U, np.eye(k), atol=1e-13) and np.allclose(Vt @ Vt.T, np.eye(k), atol=1e-13)


def test_near_optimal_on_a_decaying_spectrum():
    rng = np.random.default_rng(1)
    K, N, r = 256, 384, 16
    sig = 2.0 ** (-0.5 * np.arange(K))
    A = _orth(rng, K, K) @ np.diag(sig) @ _orth(rng, N, K).T
    U, s, Vt = R.randomized_svd(A, r)
    err = np.linalg.norm(A - U @ np.diag(s[:r]) @ Vt)
    opt = np.sqrt(np.sum(sig[r:] ** 2))            # Eckart-Young
    assert opt * (1 - 1e-12) <= err <= opt * (1 + 1e-9)
    assert np.allclose(s[:r], sig[:r], rtol=1e-9)


def test_signs_and_near_optimality_on_the_synthetic_layer():
    L = workloads.draw_layer("rsvd", "nvfp4", 64, 256, 384, 32, seed=7, n_out=4)
    lam = S.smoothing_factors(L.X, L.W)
    What = np.asarray(lam, np.float64)[:, None] * np.asarray(L.W, np.float64)
    U, s, Vt = R.randomized_svd(What, 32)
    piv = np.argmax(np.abs(Vt), axis=1)
    assert np.all(Vt[np.arange(32), piv] > 0)
    sv = np.linalg.svd(What, compute_uv=False)
    err = np.linalg.norm(What - U @ np.diag(s[:32]) @ Vt)
    opt = np.sqrt(np.sum(sv[32:] ** 2))
    assert err <= opt * 1.02
    # the outlier-driven leading values are found to high accuracy
    assert np.allclose(s[:4], sv[:4], rtol=1e-8)


def test_folded_factors_rebuild_the_smoothed_weight():
    """With W of exact rank r and power-of-two lambda (exact scaling), the
    folded factors rebuild diag(lambda) W through diag(lambda) L1f L2 up to
    their bf16 rounding: the fold divides U_r Sigma_r by lambda, once."""
    from oracle import formats as F
    rng = np.random.default_rng(3)
    K, N, k = 128, 96, 8
    W = _orth(rng, K, k) @ np.diag(np.linspace(3.0, 0.5, k)) @ _orth(rng, N, k).T
    lam = (2.0 ** rng.integers(-3, 4, size=K)).astype(np.float32)
    L1f, L2, sigma = R.randomized_factors(W, lam, k)
    assert np.array_equal(F.bf16_round(L1f), L1f) and np.array_equal(F.bf16_round(L2), L2)
    target = lam.astype(np.float64)[:, None] * W
    rebuilt = lam.astype(np.float64)[:, None] * (L1f @ L2)
    assert np.linalg.norm(rebuilt - target) <= 2.0 ** -7 * np.linalg.norm(target)
    # and the singular values are those of diag(lambda) W
    assert np.allclose(sigma[:k], np.linalg.svd(target, compute_uv=False)[:k], rtol=1e-10)
