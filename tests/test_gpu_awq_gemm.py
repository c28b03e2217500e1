"""GPU parity of the tensor-core W4A16 layer (svdq_awq_gemm) against the
oracle's 16-bit-operand form (oracle/awq.py forward_16bit).

Bar: Y within one bf16 ulp of the oracle plus the float32 dot-product bound
2 K u (sum_k |x'16_k w^16_k| + |b|) (u = 2^-24): the operands are the same
bf16 values on both sides (each dequantized weight rounded once), the sum is
float32 in the tensor core's order on the GPU and float64 in the oracle (the
bar of the AWQ layer family, as for the GEMV; the report also counts the
elements over 1e-2 rms(Y), the SVDQuant layer's bar, which bf16 outputs one
ulp apart at a rounding boundary can exceed)."""
import numpy as np
import pytest
import torch

import workloads
from oracle import awq as A
from svdq_harness import bf16_np, dev_bf16, dev_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from rank_gemm_b200 import binding
    return binding


class AwqGemm:
    def __init__(self, B, L):
        self.B, self.L = B, L
        self.aw = A.prepare(L.W, L.bias, L.s)
        self.h = B.svdq_awq_prepare(L.K, L.N, dev_bf16(L.W.T), dev_f32(L.s) if L.s is not None else None,
                                    dev_bf16(L.bias))

    def close(self):
        if self.h:
            self.B.svdq_awq_free(self.h)
            self.h = None

    def gemm(self, Xd, M):
        Y = torch.full((M, self.L.N), float("nan"), dtype=torch.bfloat16, device="cuda")
        self.B.svdq_awq_gemm(self.h, M, Xd, Y)
        torch.cuda.synchronize()
        return Y


def check_y16(g, Y_gpu, X, rows=None):
    Xs = X if rows is None else X[rows]
    ref = A.forward_16bit(g.aw, Xs)
    S = np.abs(ref["Xp16"]) @ np.abs(ref["W16"]) + np.abs(g.aw.bias)[None, :]
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref["Y"]), 1e-30))) - 7)
    bound = ulp * (1 + 1e-9) + 2.0 * g.L.K * 2.0 ** -24 * S
    err = np.abs(Y_gpu - ref["Y"])
    assert np.all(err <= bound), dict(max_err=float(err.max()), worst=float(np.max(err / bound)),
                                      where=np.unravel_index(np.argmax(err / bound), err.shape))
    rms = float(np.sqrt(np.mean(ref["Y"] ** 2)))
    return dict(max_err=float(err.max()), max_rel_rms=float(err.max() / rms),
                n_over_rel_1e2=int(np.sum(err > 1e-2 * rms)), n_beyond_ulp=int(np.sum(err > ulp * (1 + 1e-9))))


@pytest.mark.parametrize("M,K,N,scale", [(300, 256, 272, False), (130, 192, 512, True), (1, 64, 16, False),
                                         (257, 1024, 768, True)])
def test_awq_gemm_small_parity(B, M, K, N, scale):
    """Ragged M and N tiles (N % 256 != 0), a single row, with and without an
    AWQ scale (the kernel then rewrites X as bf16(x / s) in place)."""
    L = workloads.draw_awq_layer("awq_gemm_small", M, K, N, seed=70 + M, with_scale=scale)
    g = AwqGemm(B, L)
    try:
        Y = bf16_np(g.gemm(dev_bf16(L.X), M))
        print((M, K, N, scale), check_y16(g, Y, L.X))
        assert B.svdq_poll_device_error() == 0
    finally:
        g.close()


def test_awq_gemm_matches_gemv_within_the_weight_rounding(B):
    """The tensor-core form differs from the float32-weight GEMV only by the
    roundings it names: |Y16 - Y| <= sum_k |x'| |w^16 - w^| + |x'16 - x'| |w^16|
    + two bf16 ulps + both float32 bounds."""
    L = workloads.draw_awq_layer("awq_gemm_vs_gemv", 4, 512, 256, seed=79, with_scale=True)
    g = AwqGemm(B, L)
    try:
        Xd = dev_bf16(L.X)
        Y16 = bf16_np(g.gemm(Xd, L.M))
        Yv = torch.empty(L.M, L.N, dtype=torch.bfloat16, device="cuda")
        B.svdq_awq_linear(g.h, L.M, Xd, Yv)
        torch.cuda.synchronize()
        Yv = bf16_np(Yv)
        o, o16 = A.forward(g.aw, L.X), A.forward_16bit(g.aw, L.X)
        Wq = A.dequantize(g.aw)
        bound = (np.abs(o["Xp"]) @ np.abs(o16["W16"] - Wq) + np.abs(o16["Xp16"] - o["Xp"]) @ np.abs(o16["W16"])
                 + 4.0 * L.K * 2.0 ** -24 * (np.abs(o["Xp"]) @ np.abs(Wq) + np.abs(g.aw.bias)[None, :])
                 + 2.0 * np.exp2(np.floor(np.log2(np.maximum(np.abs(o["Y"]), 1e-30))) - 6))
        assert np.all(np.abs(Y16 - Yv) <= bound)
    finally:
        g.close()


def test_awq_gemm_repeatable_empty_and_shapes(B):
    L = workloads.draw_awq_layer("awq_gemm_rep", 200, 128, 256, seed=80)
    g = AwqGemm(B, L)
    try:
        Xd = dev_bf16(L.X)
        assert torch.equal(g.gemm(Xd, L.M), g.gemm(Xd, L.M))
        B.svdq_awq_gemm(g.h, 0, Xd, torch.empty(0, L.N, dtype=torch.bfloat16, device="cuda"))
    finally:
        g.close()
    L = workloads.draw_awq_layer("awq_gemm_odd_n", 4, 64, 40, seed=81)
    g = AwqGemm(B, L)
    try:
        with pytest.raises(B.SvdqError) as e:     # N % 16 != 0: the 32-byte output rows do not fit
            g.gemm(dev_bf16(L.X), L.M)
        assert e.value.status == 2
    finally:
        g.close()


@pytest.mark.slow
def test_awq_gemm_qkv_full(B):
    """The QKV shape (M=4608, K=3072, N=9216) at the size the bench times; Y on
    193 rows spread over M."""
    L = workloads.awq_qkv()
    g = AwqGemm(B, L)
    try:
        Y = g.gemm(dev_bf16(L.X), L.M)
        rows = np.unique(np.concatenate([np.linspace(0, L.M - 1, 192).astype(np.int64), [L.M - 1]]))
        Yr = bf16_np(Y[torch.from_numpy(rows).cuda()])
        print("QKV W4A16:", check_y16(g, Yr, L.X, rows))
        assert B.svdq_poll_device_error() == 0
    finally:
        g.close()
