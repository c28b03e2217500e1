"""The MLP pair with the cross-layer fusion (svdq_linear_emit_next /
svdq_mlp): the first layer's epilogue writes the second layer's kernel-1
outputs, so its bf16 output never reaches memory.

Bars:
  * against the unfused GPU path on the same handles (a consistency check,
    GPU against GPU): the second layer's codes and replicated scales
    bit-identical; its LR within two bf16 ulps plus twice the float32
    dot-product bound (both sides sum in float32, in different orders);
  * against the all-oracle chain (the oracle's own fc1 output feeds its
    fc2): relative RMS of Y2 <= 1e-2 and worst element <= 0.1 rms, the
    chain bar of test_gpu_full, on its rows (fc1's output differs by a bf16
    ulp here and there, which moves some of fc2's codes across a rounding
    step; over all 4608 rows the unfused chain's worst element is 0.16 rms
    too, at the same place);
  * against the unfused GPU chain on every row: worst element <= 0.05 rms,
    RMS <= 1e-3 (the two differ only in fc2's LR summation order)."""
import numpy as np
import pytest
import torch

import workloads
from oracle import svdquant as S
from svdq_harness import GpuLayer, bf16_np, dev_bf16, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from rank_gemm_b200 import binding
    return binding


def _pair(M, K1, N1, N2, seed, rank2=32, lora2=0):
    g = torch.Generator("cpu").manual_seed(seed)
    fc1 = workloads.draw_layer("mlp_fc1", "nvfp4", M, K1, N1, 32, seed=seed, gelu=True, gen=g)
    W2, b2, _ = workloads.draw_weight_only(N1, N2, workloads.n_outliers(N1), g)
    g1 = GpuLayer("nvfp4", fc1.X, fc1.W, fc1.bias, 32)
    Y1_o = S.forward(g1.pw, fc1.X, gelu=True)["Y"].astype(np.float32)
    A2 = B2 = None
    if lora2:   # a LoRA on fc2 (A: N1 x l, B: l x N2, N(0, 0.01)), appended to its factors
        A2 = (torch.randn(N1, lora2, generator=g) * 0.01).to(torch.bfloat16).float().numpy()
        B2 = (torch.randn(lora2, N2, generator=g) * 0.01).to(torch.bfloat16).float().numpy()
    g2 = GpuLayer("nvfp4", Y1_o, W2, b2, rank2, A2, B2)
    return fc1, g1, g2, Y1_o


def _chain_check(B, g1, g2, X, Y1_o):
    M = X.shape[0]
    Y2 = torch.empty(M, g2.N, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(B.svdq_mlp_workspace_bytes(g1.h, g2.h, M), dtype=torch.uint8, device="cuda")
    B.svdq_mlp(g1.h, g2.h, M, dev_bf16(X), B.SVDQ_EPI_GELU_TANH, B.SVDQ_EPI_NONE, Y2, ws)
    torch.cuda.synchronize()
    Y2_o = S.forward(g2.pw, Y1_o)["Y"]
    d = bf16_np(Y2) - Y2_o
    rms = float(np.sqrt(np.mean(Y2_o ** 2)))
    rel_rms, rel_max = float(np.sqrt(np.mean(d ** 2))) / rms, float(np.max(np.abs(d))) / rms
    assert rel_rms <= 1e-2 and rel_max <= 0.1, (rel_rms, rel_max)
    return rel_rms, rel_max


@pytest.mark.parametrize("M,K1,N1,N2,rank2,lora2", [
    (200, 512, 768, 256, 32, 0),
    # fc2 with a LoRA (r_tot 48) and at the largest rank emit mode takes (64)
    (200, 512, 768, 256, 32, 16),
    (130, 256, 512, 256, 48, 16),
    # 160 tiles on 148 SMs: some CTAs take two, so a tile's partial runs inside
    # the next tile's k-loop; one 256-wide k-tile per tile
    (1280, 256, 4096, 256, 32, 16),
])
def test_emit_matches_the_unfused_gpu_path(B, M, K1, N1, N2, rank2, lora2):
    fc1, g1, g2, _ = _pair(M, K1, N1, N2, seed=70 + rank2 + lora2, rank2=rank2, lora2=lora2)
    try:
        M = fc1.M
        Xd = dev_bf16(fc1.X)
        # unfused: fc1's bf16 output, then fc2's kernel 1 on it
        Y1 = g1.linear(Xd, M, gelu=True)
        q_ref, s_ref, l_ref = g2.kernel1(Y1, M)
        # fused
        q2, s2, l2 = g2.buffers(M)
        ws = torch.empty(B.svdq_linear_emit_next_workspace_bytes(g1.h, g2.h, M), dtype=torch.uint8, device="cuda")
        B.svdq_linear_emit_next(g1.h, g2.h, M, Xd, B.SVDQ_EPI_GELU_TANH, q2, s2, l2, ws)
        torch.cuda.synchronize()
        assert torch.equal(q2, q_ref)
        assert torch.equal(s2, s_ref)
        i = g2.info
        lr = lambda t: to_np(t)[: M * i.r_pad * 2].view(np.uint16).reshape(M, i.r_pad).astype(np.uint32)
        a = (lr(l2) << 16).view(np.float32).astype(np.float64)
        b = (lr(l_ref) << 16).view(np.float32).astype(np.float64)
        Y1f = bf16_np(Y1)
        L1 = np.zeros((g2.K, i.r_pad))
        L1[:, : g2.r_tot] = np.asarray(g2.pw.L1f, np.float64)
        bound = 2.0 * g2.K * 2.0 ** -24 * (np.abs(Y1f) @ np.abs(L1))
        ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(b), 1e-30))) - 7)
        assert np.all(np.abs(a - b) <= 2 * (ulp + bound)), float(np.max(np.abs(a - b) / (ulp + bound)))
        print("LR entries differing:", int(np.sum(a != b)), "of", a.size)
    finally:
        g1.close()
        g2.close()


def test_fused_mlp_chain_small(B):
    fc1, g1, g2, Y1_o = _pair(256, 512, 1024, 512, seed=71)
    try:
        print(_chain_check(B, g1, g2, fc1.X, Y1_o))
    finally:
        g1.close()
        g2.close()


def test_pair_checks(B):
    fc1, g1, g2, _ = _pair(64, 256, 512, 256, seed=72)
    try:
        with pytest.raises(B.SvdqError) as e:   # w2's K must be w1's N (fc1 twice: 512 != 256)
            B.svdq_mlp(g1.h, g1.h, 64, dev_bf16(fc1.X), 1, 0, torch.empty(64, 512, dtype=torch.bfloat16, device="cuda"),
                       torch.empty(1 << 20, dtype=torch.uint8, device="cuda"))
        assert e.value.status == 2
        assert B.svdq_mlp_workspace_bytes(g1.h, g1.h, 64) == 0
    finally:
        g1.close()
        g2.close()


@pytest.mark.slow
def test_fused_mlp_full(B):
    # the full MLP pair: against the all-oracle chain on the rows test_gpu_full
    # samples (its chain bar), and against the unfused GPU chain on every row
    # (they differ only through fc2's LR summation order)
    fc1, (W2, b2, _) = workloads.mlp_pair()
    g1 = GpuLayer(fc1.fmt, fc1.X, fc1.W, fc1.bias, fc1.rank)
    try:
        Y1_o = S.forward(g1.pw, fc1.X, gelu=True)["Y"].astype(np.float32)
        g2 = GpuLayer("nvfp4", Y1_o, W2, b2, 32)
        try:
            M = fc1.M
            Xd = dev_bf16(fc1.X)
            Y2 = torch.empty(M, g2.N, dtype=torch.bfloat16, device="cuda")
            ws = torch.empty(B.svdq_mlp_workspace_bytes(g1.h, g2.h, M), dtype=torch.uint8, device="cuda")
            B.svdq_mlp(g1.h, g2.h, M, Xd, B.SVDQ_EPI_GELU_TANH, B.SVDQ_EPI_NONE, Y2, ws)
            Y2u = g2.linear(g1.linear(Xd, M, gelu=True), M)
            torch.cuda.synchronize()
            rows = np.unique(np.concatenate([np.linspace(0, M - 1, 192).astype(np.int64), [M - 1]]))
            Y2_o = S.forward(g2.pw, Y1_o[rows])["Y"]
            rms = float(np.sqrt(np.mean(Y2_o ** 2)))
            d = bf16_np(Y2)[rows] - Y2_o
            rel_rms, rel_max = float(np.sqrt(np.mean(d ** 2))) / rms, float(np.max(np.abs(d))) / rms
            du = np.abs(bf16_np(Y2) - bf16_np(Y2u))
            print("fused MLP full: chain rel_rms %.3e rel_max %.3e; fused vs unfused max %.3e rms"
                  % (rel_rms, rel_max, du.max() / rms))
            assert rel_rms <= 1e-2 and rel_max <= 0.1
            assert du.max() <= 0.05 * rms and float(np.sqrt(np.mean(du ** 2))) <= 1e-3 * rms
        finally:
            g2.close()
    finally:
        g1.close()
