"""GPU parity of the per-call NVFP4 activation tensor scale (svdq_linear_dynamic)
against the oracle's forward(..., dynamic=True).

Bar: the scale the call chose (s_tX and j, from the record it writes into
the workspace) bit-exact with oracle.dynamic_act_scale; codes and block
scales bit-exact with the oracle's quantization under that scale; LR equal
to the oracle's LR times 2^(k - j) (2^k the prepared alpha) within the usual
LR bound; Y within 1e-2 rms plus the LR slack.  The activations are drawn
from the workload generators and rescaled, so that the batch's amax is far
from the calibration one (the case the per-call scale exists for)."""
import numpy as np
import pytest
import torch

import workloads
from oracle import svdquant as S
from svdq_harness import GpuLayer, assert_y, bf16_np, dev_bf16, lr_check, lr_slack

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from rank_gemm_b200 import binding
    return binding


def _bf16_exact(X):
    """The values a bf16 device copy holds (the oracle sees the same input)."""
    return torch.from_numpy(np.asarray(X, np.float32)).to(torch.bfloat16).float().numpy()


def dynamic_check(g, X, gelu=False, rows=None, exception=None):
    pw, M = g.pw, X.shape[0]
    Xd = dev_bf16(X)
    Y, qX, sX, LR, rec = g.linear_dynamic(Xd, M, gelu=gelu)
    s_t, j = S.dynamic_act_scale(pw, X)
    assert rec[0] == s_t and rec[1] == j and rec[2] == np.float32(2.0 ** j), (rec, s_t, j)
    pwd = S.with_act_scale(pw, s_t)
    q, s, lr, lr_pad = g.decode_act(qX, sX, LR, M)
    oq, osc = S.quantize_activation(pwd, X)
    assert np.array_equal(q, oq)
    assert np.array_equal(np.asarray(s).view(np.uint8), np.asarray(osc).view(np.uint8))
    lrc = lr_check(lr * 2.0 ** (j - pw.alpha_log2), X, pw.L1f)
    assert lrc["ok"], lrc
    assert np.all(lr_pad == 0)
    if rows is None:
        Y_o = S.forward(pw, X, gelu=gelu, dynamic=True)["Y"]
        return Y, j, assert_y(bf16_np(Y), Y_o, slack=lr_slack(X, pw, gelu))
    Y_o = S.forward(pwd, X[rows], gelu=gelu)["Y"]
    Y_g = bf16_np(Y[torch.from_numpy(rows).cuda()])
    return Y, j, assert_y(Y_g, Y_o, slack=lr_slack(X[rows], pw, gelu), exception=exception)


@pytest.mark.parametrize("gain", [1.0 / 256, 1.0, 40.0])
def test_dynamic_scale_small(B, gain):
    L = workloads.small()
    g = GpuLayer(L.fmt, L.X, L.W, L.bias, L.rank)
    try:
        X = _bf16_exact(L.X * gain)
        _, j, r = dynamic_check(g, X)
        print("gain %g: j=%d (prepared k=%d)" % (gain, j, g.pw.alpha_log2), r)
        if gain != 1.0:
            assert j != g.pw.alpha_log2
    finally:
        g.close()


def test_dynamic_ragged_gelu_lora(B):
    L = workloads.draw_layer("dyn", "nvfp4", 200, 320, 272, 16, seed=21, n_out=3, gelu=True, lora_rank=16)
    g = GpuLayer(L.fmt, L.X, L.W, L.bias, L.rank, L.lora_A, L.lora_B)
    try:
        print(dynamic_check(g, _bf16_exact(L.X * 0.01), gelu=True)[2])
    finally:
        g.close()


def test_dynamic_zero_activation(B):
    # amax 0 counts as 2688: j from s_tR alone, every code and scale 0, Y = b
    L = workloads.draw_layer("dynz", "nvfp4", 130, 256, 256, 16, seed=22, n_out=2)
    g = GpuLayer(L.fmt, L.X, L.W, L.bias, L.rank)
    try:
        Y, _, _ = dynamic_check(g, np.zeros_like(L.X))
        assert np.array_equal(bf16_np(Y), np.broadcast_to(_bf16_exact(L.bias)[None, :], Y.shape))
    finally:
        g.close()


def test_dynamic_calls_do_not_share_state(B):
    # a large-amplitude call, then a small one on the same weights: the second
    # must see only its own amax (every amax slot is rewritten by each call)
    L = workloads.draw_layer("dyns", "nvfp4", 256, 512, 256, 32, seed=23, n_out=3)
    g = GpuLayer(L.fmt, L.X, L.W, L.bias, L.rank)
    try:
        _, j1, _ = dynamic_check(g, _bf16_exact(L.X * 100.0))
        _, j2, _ = dynamic_check(g, _bf16_exact(L.X[:70] * 0.01))
        assert j1 > j2
    finally:
        g.close()


def test_dynamic_int4_is_static(B):
    L = workloads.draw_layer("dyni", "int4", 192, 512, 384, 32, seed=24, n_out=3)
    g = GpuLayer(L.fmt, L.X, L.W, L.bias, L.rank)
    try:
        Xd = dev_bf16(L.X)
        Y_dyn = g.linear_dynamic(Xd, L.M)[0]
        Y_st = g.linear(Xd, L.M)
        assert torch.equal(Y_dyn, Y_st)
    finally:
        g.close()


def test_dynamic_workspace_and_empty(B):
    L = workloads.draw_layer("dynw", "nvfp4", 64, 256, 256, 16, seed=25, n_out=2)
    g = GpuLayer(L.fmt, L.X, L.W, L.bias, L.rank)
    try:
        need = B.svdq_linear_dynamic_workspace_bytes(g.h, L.M)
        assert need > B.svdq_linear_workspace_bytes(g.h, L.M)
        Y = torch.empty(L.M, L.N, dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(need - 1, dtype=torch.uint8, device="cuda")
        with pytest.raises(B.SvdqError) as e:
            B.svdq_linear_dynamic(g.h, L.M, dev_bf16(L.X), 0, Y, ws)
        assert e.value.status == 5
        B.svdq_linear_dynamic(g.h, 0, dev_bf16(L.X[:0]), 0, Y[:0], ws)
    finally:
        g.close()


@pytest.mark.slow
def test_dynamic_qkv_full(B):
    # the benchmark's QKV shape, activations drifted 8x above calibration
    L = workloads.qkv()
    g = GpuLayer(L.fmt, L.X, L.W, L.bias, L.rank)
    try:
        X = _bf16_exact(L.X * 8.0)
        rows = np.unique(np.concatenate([np.linspace(0, L.M - 1, 192).astype(np.int64), [L.M - 1]]))
        _, j, r = dynamic_check(g, X, rows=rows, exception="dynamic_qkv_full")
        print("QKV dynamic: j=%d (prepared k=%d)" % (j, g.pw.alpha_log2), r)
    finally:
        g.close()
