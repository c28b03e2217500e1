"""Plain CPU oracle of the randomized truncated SVD used to split W^ on the
device (float64 numpy).

TEST INFRASTRUCTURE ONLY: only tests/, __graft_entry__.smoke() and the CPU
baseline leg of bench.py may import this module.  It shares no code with
the CUDA path.

The pages fix only that W^ = diag(lambda) W is split by an SVD into a rank-r
16-bit branch L1 L2 and a residual (SVDQuant overview figure, Stage 3,
"svdq-int4-flux.1-dev" model card).  The exact truncated SVD (svdquant.svd_split)
is that definition.  For preparing weights on the GPU without a dense SVD
this build uses the randomized range finder with subspace iteration of
Halko, Martinsson and Tropp, "Finding structure with randomness" (SIAM
Review 53(2), 2011): Algorithm 4.4 (randomized subspace iteration) followed
by Algorithm 5.1 (direct SVD of the small projected matrix), in the steps
and order below.  Readings (choices of this build):
  * test matrix: Rademacher (+1/-1) entries, N x l with l = min(r + 8, K, N)
    (oversampling p = 8); entry (n, j) is the top bit of 32-bit word
    e = n l + j of a Philox4x32-10 stream (Salmon, Moraes, Dror and Shaw,
    "Parallel random numbers: as easy as 1, 2, 3", SC 2011): block e / 4,
    counter (block mod 2^32, block / 2^32, 0, 0), key (seed mod 2^32,
    seed / 2^32), word e mod 4; bit 0 -> +1, bit 1 -> -1;
  * q = 3 subspace iterations, every orthonormalization a CholeskyQR2 (two
    passes of G = Y^T Y, G = R^T R, Y <- Y R^-1); a Gram matrix that is not
    numerically positive definite (a sketch of lower rank than its width) is
    factored with the shift 2^-40 trace(G) on its diagonal;
  * the small SVD through the symmetric eigenproblem of T = Z^T Z with
    Z = W^T Q (so B = Q^T W^ = Z^T): T = P diag(e) P^T, eigenvalues in
    descending order, sigma = sqrt(max(e, 0)), U = Q P, V = Z P / sigma;
  * signs as in svdquant.svd_split: each right singular vector's
    largest-magnitude entry positive (first index wins a tie).
"""
from __future__ import annotations

import numpy as np

from . import formats as F

PHILOX_M = (0xD2511F53, 0xCD9E8D57)
PHILOX_W = (0x9E3779B9, 0xBB67AE85)
MASK32 = 0xFFFFFFFF
OVERSAMPLE = 8
POWER_ITERS = 3
DEFAULT_SEED = 0x5EED


def philox4x32_10(ctr, key) -> np.ndarray:
    """Philox4x32-10 on an array of counters (n, 4) with one key (2,).
    Returns (n, 4) uint32."""
    c = [np.asarray(ctr, np.uint64)[:, i] & MASK32 for i in range(4)]
    k0, k1 = int(key[0]) & MASK32, int(key[1]) & MASK32
    for r in range(10):
        if r:
            k0, k1 = (k0 + PHILOX_W[0]) & MASK32, (k1 + PHILOX_W[1]) & MASK32
        p0 = c[0] * np.uint64(PHILOX_M[0])
        p1 = c[2] * np.uint64(PHILOX_M[1])
        hi0, lo0 = p0 >> np.uint64(32), p0 & np.uint64(MASK32)
        hi1, lo1 = p1 >> np.uint64(32), p1 & np.uint64(MASK32)
        c = [hi1 ^ c[1] ^ np.uint64(k0), lo1, hi0 ^ c[3] ^ np.uint64(k1), lo0]
    return np.stack(c, axis=1).astype(np.uint32)


def rademacher(rows: int, cols: int, seed: int = DEFAULT_SEED) -> np.ndarray:
    """(rows, cols) float64 of +-1 from the Philox stream (see the header)."""
    n_words = rows * cols
    blocks = (n_words + 3) // 4
    b = np.arange(blocks, dtype=np.uint64)
    ctr = np.stack([b & np.uint64(MASK32), b >> np.uint64(32), np.zeros_like(b), np.zeros_like(b)], axis=1)
    words = philox4x32_10(ctr, (seed & MASK32, (seed >> 32) & MASK32)).reshape(-1)[:n_words]
    return np.where((words >> np.uint32(31)) == 0, 1.0, -1.0).reshape(rows, cols)


def cholesky_upper(G) -> np.ndarray:
    """R upper triangular with G = R^T R.  If G is not numerically positive
    definite (a sketch of lower rank than its width), the factorization is
    taken of G + s I with s = 2^-40 trace(G) (s = 1 when G = 0) instead."""
    G = np.asarray(G, np.float64)
    try:
        return np.linalg.cholesky(G).T
    except np.linalg.LinAlgError:
        tr = float(np.trace(G))
        shift = tr * 2.0 ** -40 if tr > 0 else 1.0
        return np.linalg.cholesky(G + shift * np.eye(G.shape[0])).T


def cholqr2(Y) -> np.ndarray:
    """Orthonormal columns spanning Y (tall): two passes of Cholesky QR."""
    Q = np.asarray(Y, np.float64)
    for _ in range(2):
        R = cholesky_upper(Q.T @ Q)                # G = R^T R, R upper triangular
        Q = np.linalg.solve(R.T, Q.T).T            # Q R^-1
    return Q


def randomized_svd(What, rank: int, seed: int = DEFAULT_SEED, p: int = OVERSAMPLE, q: int = POWER_ITERS):
    """Rank-`rank` factors of W^ (K, N): (U_r (K, r), sigma (l,), V_r^T (r, N))."""
    What = np.asarray(What, np.float64)
    K, N = What.shape
    l = min(rank + p, K, N)
    Q = cholqr2(What @ rademacher(N, l, seed))
    for _ in range(q):
        Z = cholqr2(What.T @ Q)
        Q = cholqr2(What @ Z)
    Z = What.T @ Q                                 # B^T, B = Q^T W^
    e, P = np.linalg.eigh(Z.T @ Z)
    order = np.argsort(-e, kind="stable")
    e, P = e[order], P[:, order]
    sigma = np.sqrt(np.maximum(e, 0.0))
    U = Q @ P
    V = (Z @ P) / np.where(sigma > 0, sigma, 1.0)[None, :]
    U, V = U[:, :rank], V[:, :rank]
    piv = np.argmax(np.abs(V), axis=0)
    sgn = np.where(V[piv, np.arange(rank)] < 0, -1.0, 1.0)
    return U * sgn[None, :], sigma, (V * sgn[None, :]).T


def randomized_factors(W, lam, rank: int, seed: int = DEFAULT_SEED):
    """The 16-bit factors from the randomized split, folded like
    svdquant.svd_factors: L1f = bf16(diag(lambda)^-1 U_r Sigma_r),
    L2 = bf16(V_r^T).  Returns (L1f, L2, sigma)."""
    W = np.asarray(W, np.float64)
    lam64 = np.asarray(lam, np.float32).astype(np.float64)
    U, sigma, Vt = randomized_svd(lam64[:, None] * W, rank, seed)
    L1f = F.bf16_round(U * sigma[None, :rank] / lam64[:, None])
    L2 = F.bf16_round(Vt)
    return L1f, L2, sigma
