"""GPU parity of the device's low-rank split (svdq_lowrank_factors, and
svdq_prepare_weights without caller factors) against oracle/rsvd.py on the
same inputs and the same Philox sketch.

Bar: the estimated singular values within 1e-9 relative; the bf16 factors
L1f and L2 within one bf16 ulp of the oracle's element by element (both sides
round float64 values that differ only by summation order); the layer built
from the device split within the layer tolerance of the oracle's layer built
from the oracle split."""
import numpy as np
import pytest
import torch

import workloads
from oracle import formats as F
from oracle import rsvd as R
from oracle import svdquant as S
from svdq_harness import assert_y, bf16_np, dev_bf16, dev_f32, lr_slack

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from rank_gemm_b200 import binding
    return binding


def _ulp(v):
    return np.exp2(np.floor(np.log2(np.maximum(np.abs(v), 1e-30))) - 7)


def split_check(B, L, rank):
    lam = S.smoothing_factors(L.X, L.W)
    K, N = L.W.shape
    L1f = torch.empty(K, rank, dtype=torch.bfloat16, device="cuda")
    L2 = torch.empty(rank, N, dtype=torch.bfloat16, device="cuda")
    sig = np.array(B.svdq_lowrank_factors(K, N, rank, dev_bf16(L.W.T), dev_f32(lam), L1f, L2))
    o1, o2, osig = R.randomized_factors(L.W, lam, rank)
    assert np.allclose(sig, osig, rtol=1e-9, atol=1e-12 * osig[0])
    g1, g2 = bf16_np(L1f), bf16_np(L2)
    d1, d2 = np.abs(g1 - o1), np.abs(g2 - o2)
    assert np.all(d1 <= _ulp(o1) * (1 + 1e-9)) and np.all(d2 <= _ulp(o2) * (1 + 1e-9))
    return lam, dict(sig0=float(sig[0]), n_l1f_ulp=int(np.sum(d1 > 0)), n_l2_ulp=int(np.sum(d2 > 0)))


def test_split_matches_oracle_small(B):
    L = workloads.draw_layer("rsvd_small", "nvfp4", 64, 256, 384, 32, seed=60, n_out=4)
    print(split_check(B, L, 32)[1])


def test_split_rank_near_the_dimension(B):
    # l = min(r + 8, K, N) = K: the sketch spans the whole column space
    L = workloads.draw_layer("rsvd_full", "nvfp4", 32, 128, 160, 16, seed=61, n_out=2)
    print(split_check(B, L, 124)[1])


def test_prepare_without_factors_builds_the_layer(B):
    L = workloads.draw_layer("rsvd_layer", "nvfp4", 128, 512, 384, 32, seed=62, n_out=4)
    lam = S.smoothing_factors(L.X, L.W)
    act = S.act_tensor_scale(L.X, S.inverse_lambda(lam))
    h = B.svdq_prepare_weights("nvfp4", L.K, L.N, 32, dev_bf16(L.W.T), dev_f32(lam), None, None, dev_bf16(L.bias),
                               act_scale=float(act))
    try:
        o1, o2, _ = R.randomized_factors(L.W, lam, 32)
        pw = S.prepare("nvfp4", L.W, lam, o1, o2, L.bias, act)
        Y = torch.empty(L.M, L.N, dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(B.svdq_linear_workspace_bytes(h, L.M), dtype=torch.uint8, device="cuda")
        B.svdq_linear(h, L.M, dev_bf16(L.X), B.SVDQ_EPI_NONE, Y, ws)
        torch.cuda.synchronize()
        print(assert_y(bf16_np(Y), S.forward(pw, L.X)["Y"], slack=lr_slack(L.X, pw)))
    finally:
        B.svdq_free_weights(h)


def test_split_rejects_bad_rank(B):
    W = torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda")
    lam = torch.ones(64, device="cuda")
    out = torch.empty(64 * 65, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(B.SvdqError) as e:
        B.svdq_lowrank_factors(64, 64, 65, W, lam, out, out)
    assert e.value.status == 2


@pytest.mark.slow
def test_split_qkv_full(B):
    L = workloads.qkv()
    print("QKV split:", split_check(B, L, 32)[1])
