"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Bar: codes and block scales bit-exact; the smoothing factors, tensor scales
and the residual's codes bit-exact; LR within one bf16 ulp plus the float32
dot-product error bound 2 K u sum|x l| (bit-exact on dyadic inputs); Y within max|dY| <= 1e-2 rms(Y_oracle) (an element above
that only if it is within one bf16 ulp of the oracle's value)."""
import numpy as np
import pytest
import torch

import workloads
from oracle import formats as F
from oracle import svdquant as S
from svdq_harness import (GpuLayer, assert_y, bf16_np, dev_bf16, dev_f32, lr_check, lr_slack, rup, to_np,
                           y_check)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from rank_gemm_b200 import binding
    return binding


def _full_check(L, gelu=False, lora=False):
    g = GpuLayer(L.fmt, L.X, L.W, L.bias, L.rank,
                 L.lora_A if lora else None, L.lora_B if lora else None)
    try:
        pw = g.pw
        # weight side: residual codes, scales and tensor scale bit-exact
        qR, sR, s_tR = g.weight_codes()
        assert s_tR == pw.s_tR
        assert np.array_equal(qR, pw.qR)
        assert np.array_equal(np.asarray(sR).view(np.uint8) if sR.dtype != np.uint8 else sR,
                              np.asarray(pw.sR).view(np.uint8))
        # kernel 1
        M = L.M
        Xd = dev_bf16(L.X)
        qX, sX, LR = g.kernel1(Xd, M)
        q, s, lr, lr_pad = g.decode_act(qX, sX, LR, M)
        oq, osc = S.quantize_activation(pw, L.X)
        assert np.array_equal(q, oq)
        assert np.array_equal(np.asarray(s).view(np.uint8), np.asarray(osc).view(np.uint8))
        lrc = lr_check(lr, L.X, pw.L1f)
        assert lrc["ok"], lrc
        assert np.all(lr_pad == 0)
        # whole layer
        Y = bf16_np(g.linear(Xd, M, gelu=gelu))
        Y_o = S.forward(pw, L.X, gelu=gelu)["Y"]
        return assert_y(Y, Y_o, slack=lr_slack(L.X, pw, gelu))
    finally:
        g.close()


def test_calibrate_matches_oracle_bit_exact(B):
    L = workloads.small()
    Xd, Wd = dev_bf16(L.X), dev_bf16(L.W.T)
    lam = torch.empty(L.K, dtype=torch.float32, device="cuda")
    act = torch.empty(1, dtype=torch.float32, device="cuda")
    ws = torch.empty(B.svdq_calibrate_workspace_bytes(L.K), dtype=torch.uint8, device="cuda")
    B.svdq_calibrate(L.M, L.K, L.N, Xd, Wd, 0.5, lam, act, ws)
    torch.cuda.synchronize()
    lam_o = S.smoothing_factors(L.X, L.W)
    assert np.array_equal(to_np(lam), lam_o)
    assert to_np(act)[0] == S.act_tensor_scale(L.X, S.inverse_lambda(lam_o))


def test_small_config_full_parity(B):
    r = _full_check(workloads.small())
    print("small:", r)


def test_ragged_shapes_parity(B):
    # M not a multiple of 32 or 128, K not a multiple of 256, N not a multiple of 256
    L = workloads.draw_layer("ragged", "nvfp4", 200, 320, 272, 32, seed=11, n_out=3)
    print("ragged:", _full_check(L))


def test_gelu_epilogue(B):
    L = workloads.draw_layer("gelu", "nvfp4", 160, 512, 384, 32, seed=12, n_out=4, gelu=True)
    print("gelu:", _full_check(L, gelu=True))


def test_lora_appended(B):
    L = workloads.draw_layer("lora", "nvfp4", 256, 512, 512, 16, seed=13, n_out=4, lora_rank=16)
    print("lora:", _full_check(L, lora=True))


def test_tiny_and_empty_m(B):
    L = workloads.draw_layer("m1", "nvfp4", 1, 256, 256, 16, seed=14, n_out=2)
    _full_check(L)
    g = GpuLayer(L.fmt, L.X, L.W, L.bias, L.rank)
    try:
        Y = torch.empty(0, L.N, dtype=torch.bfloat16, device="cuda")
        B.svdq_linear(g.h, 0, dev_bf16(L.X[:0]), 0, Y, torch.empty(16, dtype=torch.uint8, device="cuda"))
    finally:
        g.close()


def test_e2m1_rounding_of_every_bf16_value_in_range(B):
    """lambda = 1 and s_t = 0.5 make every group with max 6 use d = 1, so the
    codes are E2M1(x) of every bf16 value in [-6, 6]: ties, negative zero,
    subnormals."""
    pos = np.arange(0, 0x40C1, dtype=np.uint32) << 16
    vals = pos.view(np.float32)
    vals = np.concatenate([vals, -vals]).astype(np.float32)
    K = 1024
    per_row = (K // 16) * 15
    rows = -(-vals.size // per_row)
    body = np.zeros(rows * per_row, np.float32)
    body[: vals.size] = vals
    body = body.reshape(rows, K // 16, 15)
    X = np.concatenate([np.full((rows, K // 16, 1), 6.0, np.float32), body], axis=2).reshape(rows, K)
    rng = np.random.default_rng(0)
    W = (rng.standard_normal((K, 64)) * 0.02).astype(np.float32)
    W = torch.from_numpy(W).bfloat16().float().numpy()
    lam = np.ones(K, np.float32)
    L1f, L2, _ = S.svd_factors(W, lam, 16)
    g = GpuLayer("nvfp4", X, W, np.zeros(64, np.float32), 16, factors=(lam, L1f, L2), act=np.float32(0.5))
    try:
        qX, sX, LR = g.kernel1(dev_bf16(X), rows)
        q, s, _, _ = g.decode_act(qX, sX, LR, rows)
        oq, osc = S.quantize_activation(g.pw, X)
        assert np.all(osc == 0x40)
        bad = np.argwhere(q != oq)
        assert bad.size == 0, [(float(X[i, j]), int(q[i, j]), int(oq[i, j])) for i, j in bad[:8]]
    finally:
        g.close()


def test_lowrank_down_bit_exact_on_dyadic_inputs(B):
    M, K, N, r = 96, 512, 256, 32
    d = workloads.dyadic_layer(M, K, N, r, seed=15)
    X, L1f = d["X"], d["L1f"]
    rng = np.random.default_rng(1)
    W = torch.from_numpy((rng.standard_normal((K, N)) * 0.05).astype(np.float32)).bfloat16().float().numpy()
    L2 = torch.from_numpy((rng.standard_normal((r, N)) * 0.1).astype(np.float32)).bfloat16().float().numpy()
    lam = np.ones(K, np.float32)
    g = GpuLayer("nvfp4", X, W, np.zeros(N, np.float32), r, factors=(lam, L1f, L2))
    try:
        qX, sX, LR = g.kernel1(dev_bf16(X), M)
        _, _, lr, _ = g.decode_act(qX, sX, LR, M)
        exact = X.astype(np.float64) @ L1f.astype(np.float64)
        assert np.array_equal(lr, F.bf16_round(exact))
    finally:
        g.close()


def test_unfused_path_matches_fused(B):
    L = workloads.draw_layer("unfused", "nvfp4", 300, 768, 512, 32, seed=16, n_out=4)
    g = GpuLayer(L.fmt, L.X, L.W, L.bias, L.rank)
    try:
        M, Xd = L.M, dev_bf16(L.X)
        qX, sX, LR = g.kernel1(Xd, M)
        qX2, sX2, LR2 = g.buffers(M)
        B.svdq_quantize_act(g.h, M, Xd, qX2, sX2)
        B.svdq_lowrank_down(g.h, M, Xd, LR2)
        torch.cuda.synchronize()
        a, b = g.decode_act(qX, sX, LR, M), g.decode_act(qX2, sX2, LR2, M)
        for u, v in zip(a, b):
            assert np.array_equal(np.asarray(u), np.asarray(v))
        Yf = bf16_np(g.linear(Xd, M))
        Yu = bf16_np(g.linear(Xd, M, unfused=True))
        Y_o = S.forward(g.pw, L.X)["Y"]
        sl = lr_slack(L.X, g.pw)
        assert_y(Yf, Y_o, slack=sl)
        assert_y(Yu, Y_o, slack=sl, exception="unfused_nvfp4")
        # plain W4A4 GEMM (no low-rank branch): alpha Q(X^) Q(R) + b
        Yp = torch.empty(M, L.N, dtype=torch.bfloat16, device="cuda")
        B.svdq_w4a4_gemm(g.h, M, qX, sX, Yp)
        torch.cuda.synchronize()
        oq, osc = S.quantize_activation(g.pw, L.X)
        Yp_o = S.epilogue(S.main_product(g.pw, oq, osc), g.pw.bias, False)
        assert_y(bf16_np(Yp), Yp_o, exception="plain_w4a4_nvfp4")
    finally:
        g.close()


def test_repeated_runs_are_bitwise_identical(B):
    L = workloads.draw_layer("det", "nvfp4", 512, 1024, 768, 32, seed=17, n_out=5)
    g = GpuLayer(L.fmt, L.X, L.W, L.bias, L.rank)
    try:
        Xd = dev_bf16(L.X)
        ref = g.linear(Xd, L.M).clone()
        for _ in range(10):
            assert torch.equal(g.linear(Xd, L.M), ref)
    finally:
        g.close()


def test_bounded_wait_times_out_and_context_survives(B):
    assert B.svdq_poll_device_error() == 0
    B.svdq_selftest_wait_timeout(20000)          # 20 ms limit on a barrier nobody completes
    assert B.svdq_poll_device_error() == 7       # SVDQ_ERR_TIMEOUT
    assert B.svdq_poll_device_error() == 0       # cleared
    _full_check(workloads.draw_layer("after", "nvfp4", 64, 256, 256, 16, seed=18, n_out=2))


def test_capability_check_rejects_other_devices(B):
    import ctypes
    L = workloads.draw_layer("cc", "nvfp4", 32, 256, 256, 16, seed=19, n_out=2)
    g = GpuLayer(L.fmt, L.X, L.W, L.bias, L.rank)
    try:
        B.svdq_debug_override_cc(9, 0)
        Y = torch.empty(L.M, L.N, dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(B.svdq_linear_workspace_bytes(g.h, L.M), dtype=torch.uint8, device="cuda")
        with pytest.raises(B.SvdqError) as e:
            B.svdq_linear(g.h, L.M, dev_bf16(L.X), 0, Y, ws)
        assert e.value.status == 4
    finally:
        B.svdq_debug_override_cc(-1, 0)
        g.close()


def test_output_alignment_is_checked_before_launch(B):
    """The 4-bit GEMM writes Y in 32-byte row segments: a Y that is 16- but not
    32-byte aligned is refused on the host (status 3) before any launch, and
    a 32-byte aligned one inside the same buffer works."""
    for fmt in ("nvfp4", "int4"):
        L = workloads.draw_layer("align", fmt, 32, 256, 256, 16, seed=20, n_out=2)
        g = GpuLayer(L.fmt, L.X, L.W, L.bias, L.rank)
        try:
            Xd = dev_bf16(L.X)
            buf = torch.empty(L.M * L.N + 32, dtype=torch.bfloat16, device="cuda")
            assert buf.data_ptr() % 32 == 0
            Y16 = buf[8: 8 + L.M * L.N]            # 16 bytes past a 32-byte boundary
            ws = torch.empty(B.svdq_linear_workspace_bytes(g.h, L.M), dtype=torch.uint8, device="cuda")
            calls = [lambda Y: B.svdq_linear(g.h, L.M, Xd, 0, Y, ws),
                     lambda Y: B.svdq_linear_unfused(g.h, L.M, Xd, 0, Y, ws)]
            for call in calls:
                with pytest.raises(B.SvdqError) as e:
                    call(Y16)
                assert e.value.status == 3
            torch.cuda.synchronize()
            assert B.svdq_poll_device_error() == 0
            Y32 = buf[16: 16 + L.M * L.N]
            B.svdq_linear(g.h, L.M, Xd, 0, Y32, ws)
            ref = torch.empty(L.M, L.N, dtype=torch.bfloat16, device="cuda")
            B.svdq_linear(g.h, L.M, Xd, 0, ref, ws)
            assert torch.equal(Y32.view(L.M, L.N), ref)
        finally:
            g.close()


# ------------------------------------------------------------------ INT4 (int8 tensor-core path)
def test_int4_small_parity(B):
    L = workloads.draw_layer("int4", "int4", 200, 512, 384, 32, seed=21, n_out=4)
    print("int4:", _full_check(L))


def test_int4_ragged_gelu_lora(B):
    L = workloads.draw_layer("int4r", "int4", 77, 320, 272, 16, seed=22, n_out=3, gelu=True, lora_rank=16)
    print("int4 ragged:", _full_check(L, gelu=True, lora=True))


def test_int4_unfused_and_plain(B):
    L = workloads.draw_layer("int4u", "int4", 130, 768, 256, 32, seed=23, n_out=4)
    g = GpuLayer(L.fmt, L.X, L.W, L.bias, L.rank)
    try:
        Xd = dev_bf16(L.X)
        Y_o = S.forward(g.pw, L.X)["Y"]
        assert_y(bf16_np(g.linear(Xd, L.M, unfused=True)), Y_o, slack=lr_slack(L.X, g.pw), exception="unfused_int4")
        qX, sX, LR = g.kernel1(Xd, L.M)
        Yp = torch.empty(L.M, L.N, dtype=torch.bfloat16, device="cuda")
        B.svdq_w4a4_gemm(g.h, L.M, qX, sX, Yp)
        torch.cuda.synchronize()
        oq, osc = S.quantize_activation(g.pw, L.X)
        assert_y(bf16_np(Yp), S.epilogue(S.main_product(g.pw, oq, osc), g.pw.bias, False), exception="plain_w4a4_int4")
    finally:
        g.close()
