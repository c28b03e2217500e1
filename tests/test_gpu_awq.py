"""GPU parity of the AWQ W4A16 layer (svdq_awq_*) against oracle/awq.py.

Bar: codes, binary16 scales, zero points, 1/s and bias bit-exact; Y within
one bf16 ulp of the oracle plus the float32 dot-product bound
2 K u (sum_k |x'_k w^_k| + |b|) (u = 2^-24): the kernel accumulates in
float32 in its own order, the oracle in float64."""
import numpy as np
import pytest
import torch

import workloads
from oracle import awq as A
from oracle import formats as F
from svdq_harness import bf16_np, dev_bf16, dev_f32, read_device, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from rank_gemm_b200 import binding
    return binding


class Awq:
    def __init__(self, B, L):
        self.B, self.L = B, L
        self.aw = A.prepare(L.W, L.bias, L.s)
        self.d_W = dev_bf16(L.W.T)
        self.d_b = dev_bf16(L.bias)
        self.d_s = dev_f32(L.s) if L.s is not None else None
        self.h = B.svdq_awq_prepare(L.K, L.N, self.d_W, self.d_s, self.d_b)
        self.info = B.svdq_awq_view(self.h)

    def close(self):
        if self.h:
            self.B.svdq_awq_free(self.h)
            self.h = None

    def weights(self):
        i, K, N = self.info, self.L.K, self.L.N
        raw = read_device(i.code, (K // 32) * i.N_pad * 16).reshape(K // 32, i.N_pad, 16)
        code = np.empty((K, i.N_pad), np.uint8)
        for b in range(16):
            # byte b is byte b % 4 of word b // 4, i.e. nibble positions
            # p = 2 (b % 4) (low) and p + 1 (high); position p holds
            # k = 8 (b // 4) + i with p = i // 2 + 4 (i % 2)
            order = [0, 2, 4, 6, 1, 3, 5, 7]
            code[8 * (b // 4) + order[2 * (b % 4)]::32, :] = raw[:, :, b] & 0xF
            code[8 * (b // 4) + order[2 * (b % 4) + 1]::32, :] = raw[:, :, b] >> 4
        scale = read_device(i.scale, (K // 64) * i.N_pad * 2).view(np.float16).reshape(K // 64, i.N_pad)
        zero = read_device(i.zero, (K // 64) * i.N_pad).reshape(K // 64, i.N_pad)
        inv_s = read_device(i.inv_s, K * 4).view(np.float32)
        bias = read_device(i.bias, i.N_pad * 4).view(np.float32)
        return code, scale, zero, inv_s, bias

    def linear(self, X):
        M = X.shape[0]
        Y = torch.empty(M, self.L.N, dtype=torch.bfloat16, device="cuda")
        self.B.svdq_awq_linear(self.h, M, dev_bf16(X), Y)
        torch.cuda.synchronize()
        return bf16_np(Y)


def check_weights(g):
    code, scale, zero, inv_s, bias = g.weights()
    aw, N = g.aw, g.L.N
    assert np.array_equal(code[:, :N], aw.code)
    assert np.array_equal(scale[:, :N].astype(np.float32), aw.scale)
    assert np.array_equal(zero[:, :N], aw.zero)
    assert np.array_equal(inv_s, aw.inv_s)
    assert np.array_equal(bias[:N], g.L.bias.astype(np.float32))
    # pad features contribute nothing
    assert np.all(code[:, N:] == 0) and np.all(scale[:, N:] == 0) and np.all(zero[:, N:] == 0)


def check_y(g, X, rows=None):
    Y = g.linear(X)
    Xs = X if rows is None else X[rows]
    Yg = Y if rows is None else Y[rows]
    o = A.forward(g.aw, Xs)
    Wq = A.dequantize(g.aw)
    S = np.abs(o["Xp"]) @ np.abs(Wq) + np.abs(g.aw.bias)[None, :]
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(o["Y"]), 1e-30))) - 7)
    bound = ulp * (1 + 1e-9) + 2.0 * g.L.K * 2.0 ** -24 * S
    err = np.abs(Yg - o["Y"])
    assert np.all(err <= bound), dict(max_err=float(err.max()), worst=float(np.max(err / bound)))
    return dict(max_err=float(err.max()), n_beyond_ulp=int(np.sum(err > ulp * (1 + 1e-9))))


@pytest.mark.parametrize("M,K,N,scale", [(1, 128, 40, False), (3, 192, 96, True), (5, 256, 70, True),
                                         (9, 64, 33, False)])
def test_awq_small_parity(B, M, K, N, scale):
    L = workloads.draw_awq_layer("awq_small", M, K, N, seed=40 + M, with_scale=scale)
    g = Awq(B, L)
    try:
        check_weights(g)
        print((M, K, N), check_y(g, L.X))
    finally:
        g.close()


def test_awq_large_k_single_row_blocks(B):
    # K = 12288: one activation row per pass over the weights (48 KB of staged x')
    L = workloads.draw_awq_layer("awq_bigk", 3, 12288, 64, seed=50, with_scale=True)
    g = Awq(B, L)
    try:
        check_weights(g)
        print(check_y(g, L.X))
    finally:
        g.close()


def test_awq_repeatable_and_empty(B):
    L = workloads.draw_awq_layer("awq_rep", 4, 256, 96, seed=51)
    g = Awq(B, L)
    try:
        assert np.array_equal(g.linear(L.X), g.linear(L.X))
        B.svdq_awq_linear(g.h, 0, dev_bf16(L.X[:0]), torch.empty(0, L.N, dtype=torch.bfloat16, device="cuda"))
    finally:
        g.close()


def test_awq_rejects_bad_shapes(B):
    W = torch.zeros(8, 100, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(B.SvdqError) as e:
        B.svdq_awq_prepare(100, 8, W)
    assert e.value.status == 2


@pytest.mark.slow
@pytest.mark.parametrize("M", [1, 4])
def test_awq_adaln_full(B, M):
    L = workloads.awq_adaln(M)
    g = Awq(B, L)
    try:
        check_weights(g)
        print("adaLN M=%d:" % M, check_y(g, L.X))
    finally:
        g.close()
