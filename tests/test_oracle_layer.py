"""Whole-layer pins for the oracle: reduction to X W + b without quantization,
a scalar-loop brute force of the full W4A4 layer on tiny inputs (both
formats), the LoRA rule, and the pages' qualitative claim."""
import numpy as np
import pytest

import workloads
from oracle import formats as F
from oracle import svdquant as S
from test_oracle_formats import _e2m1_nearest, _e4m3_nearest


def _layer(M, K, N, r, seed, fmt="nvfp4", n_out=3, lora=0):
    L = workloads.draw_layer("t", fmt, M, K, N, r, seed=seed, n_out=n_out, lora_rank=lora)
    return L


# ------------------------------------------------------------ quantization disabled
def check_unquantized_reduces_to_xw(rank_full=True):
    L = _layer(48, 64, 96, 64, seed=31)
    r = min(L.K, L.N) if rank_full else 8
    pw = S.calibrate_and_prepare("nvfp4", L.X, L.W, L.bias, r)
    Y = S.forward(pw, L.X, quantize=False)["Y"]
    ref = L.X.astype(np.float64) @ L.W.astype(np.float64) + L.bias[None, :]
    assert np.max(np.abs(Y - ref)) <= 2e-6 * np.max(np.abs(ref))


def test_unquantized_full_rank_is_xw_plus_b():
    check_unquantized_reduces_to_xw(True)


def test_unquantized_low_rank_is_xw_plus_b():
    check_unquantized_reduces_to_xw(False)


# ------------------------------------------------------------ brute force
def _bf16_nearest(x):
    f = np.array([x], np.float32)
    b = int(f.view(np.uint32)[0] >> 16)
    best = None
    for c in (b - 1, b, b + 1):
        v = float(np.array([c << 16], np.uint32).view(np.float32)[0])
        key = (abs(x - v), c & 1)
        if best is None or key < best[0]:
            best = (key, v)
    return best[1]


def _brute_layer(fmt, X, W, bias, lam, L1f, L2, act_scale, gelu=False):
    f32 = np.float32
    M, K = X.shape
    N = W.shape[1]
    r = L1f.shape[1]
    g = 16 if fmt == "nvfp4" else 64
    inv = [f32(1.0) / f32(l) for l in lam]
    Xh = [[f32(f32(X[m, k]) * inv[k]) for k in range(K)] for m in range(M)]
    R = [[0.0] * K for _ in range(N)]           # R^T: row n, column k
    for k in range(K):
        for n in range(N):
            s = 0.0
            for i in range(r):
                s = s + float(L1f[k, i]) * float(L2[i, n])
            R[n][k] = f32(float(lam[k]) * float(W[k, n]) - float(lam[k]) * s)
    if fmt == "nvfp4":
        amax = max(abs(R[n][k]) for n in range(N) for k in range(K))
        s_tX = f32(act_scale)
        # smallest power of two 2^k >= s_tX amax / 2688, then s_tR = 2^k / s_tX
        target = (float(amax) if amax > 0 else 2688.0) * float(s_tX) / 2688.0
        k = -200
        while 2.0 ** k < target:
            k += 1
        s_tR = f32(f32(2.0 ** k) / s_tX)
    else:
        s_tR = s_tX = f32(1.0)

    def quant_rows(rows, s_t):
        codes, scales, deq = [], [], []
        for row in rows:
            cr, sr, dr = [], [], []
            for j in range(0, K, g):
                blk = row[j:j + g]
                a = f32(max(abs(v) for v in blk))
                if fmt == "nvfp4":
                    sc = _e4m3_nearest(f32(a / f32(f32(6.0) * s_t)))
                    sbv = f32(F.e4m3_decode(np.array([sc]))[0])
                    d = f32(sbv * s_t)
                    iv = f32(0.0) if d == 0 else f32(f32(1.0) / d)
                    for v in blk:
                        c = _e2m1_nearest(f32(v * iv))
                        cr.append(c)
                        dr.append(float(F.e2m1_decode(np.array([c]))[0]) * float(sbv))
                else:
                    sbv = np.float16(f32(a / f32(7.0)))
                    sc = sbv
                    d = f32(sbv)
                    iv = f32(0.0) if d == 0 else f32(f32(1.0) / d)
                    for v in blk:
                        c = int(max(-8, min(7, round(float(f32(v * iv))))))   # round(): half to even
                        cr.append(c)
                        dr.append(c * float(d))
                sr.append(sc)
            codes.append(cr)
            scales.append(sr)
            deq.append(dr)
        return codes, scales, deq

    qX, sX, dX = quant_rows(Xh, s_tX)
    qR, sR, dR = quant_rows(R, s_tR)
    alpha = float(s_tX) * float(s_tR)
    LR = [[_bf16_nearest(sum(float(X[m, k]) * float(L1f[k, i]) for k in range(K))) for i in range(r)]
          for m in range(M)]
    Y = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            main = sum(dX[m][k] * dR[n][k] for k in range(K))
            up = sum(LR[m][i] * float(L2[i, n]) for i in range(r))
            y = alpha * main + up + float(bias[n])
            if gelu:
                y = 0.5 * y * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (y + 0.044715 * y * y * y)))
            Y[m, n] = _bf16_nearest(y)
    return dict(qX=np.array(qX), sX=np.array(sX), qR=np.array(qR), sR=np.array(sR),
                LR=np.array(LR), Y=Y, s_tR=s_tR)


def check_brute_force(fmt, M, K, N, r, seed, gelu=False):
    L = _layer(M, K, N, r, seed, fmt=fmt, n_out=2)
    lam = S.smoothing_factors(L.X, L.W)
    L1f, L2, _ = S.svd_factors(L.W, lam, r)
    act = S.act_tensor_scale(L.X, S.inverse_lambda(lam)) if fmt == "nvfp4" else None
    pw = S.prepare(fmt, L.W, lam, L1f, L2, L.bias, act)
    out = S.forward(pw, L.X, gelu=gelu)
    bf = _brute_layer(fmt, L.X, L.W, L.bias, lam, L1f, L2, act, gelu)
    if fmt == "nvfp4":
        assert np.array_equal(out["qX"], bf["qX"].astype(np.uint8))
        assert np.array_equal(out["sX"], bf["sX"].astype(np.uint8))
        assert np.array_equal(pw.qR, bf["qR"].astype(np.uint8))
        assert np.array_equal(pw.sR, bf["sR"].astype(np.uint8))
        assert pw.s_tR == bf["s_tR"]
    else:
        assert np.array_equal(out["qX"], bf["qX"].astype(np.int8))
        assert np.array_equal(out["sX"].astype(np.float64), bf["sX"].astype(np.float64))
        assert np.array_equal(pw.qR, bf["qR"].astype(np.int8))
        assert np.array_equal(pw.sR.astype(np.float64), bf["sR"].astype(np.float64))
    assert np.array_equal(out["LR"], bf["LR"])
    ulp = np.abs(bf["Y"]) * 2.0 ** -7 + 1e-30
    assert np.all(np.abs(out["Y"] - bf["Y"]) <= ulp)


def test_brute_force_nvfp4_8x16x16():
    check_brute_force("nvfp4", 8, 16, 16, 4, seed=41)


def test_brute_force_nvfp4_gelu_4x32x16():
    check_brute_force("nvfp4", 4, 32, 16, 4, seed=42, gelu=True)


def test_brute_force_int4_4x64x8():
    check_brute_force("int4", 4, 64, 8, 4, seed=43)


# ------------------------------------------------------------ LoRA
def test_lora_leaves_residual_codes_untouched():
    L = _layer(64, 128, 96, 16, seed=51, lora=16)
    lam = S.smoothing_factors(L.X, L.W)
    L1f, L2, _ = S.svd_factors(L.W, lam, 16)
    act = S.act_tensor_scale(L.X, S.inverse_lambda(lam))
    base = S.prepare("nvfp4", L.W, lam, L1f, L2, L.bias, act)
    lora = S.prepare("nvfp4", L.W, lam, L1f, L2, L.bias, act, L.lora_A, L.lora_B)
    assert np.array_equal(base.qR, lora.qR) and np.array_equal(base.sR, lora.sR)
    assert base.s_tR == lora.s_tR
    yb = S.forward(base, L.X)["Y"]
    yl = S.forward(lora, L.X)["Y"]
    want = L.X.astype(np.float64) @ L.lora_A.astype(np.float64) @ L.lora_B.astype(np.float64)
    # the LoRA's contribution passes through the bf16 LR and the bf16 output
    tol = 2.0 ** -7 * (np.abs(yb) + np.abs(yl)) + 1e-2 * np.sqrt(np.mean(want ** 2))
    assert np.all(np.abs((yl - yb) - want) <= tol)


# ------------------------------------------------------------ the pages' claim
def test_low_rank_branch_reduces_quantization_error():
    """Overview figure: migration alone makes the weight hard to quantize;
    the low-rank branch absorbs the outliers.  Error against exact X W:
    SVDQuant < smoothing-only W4A4 < plain W4A4."""
    L = workloads.small()
    ref = L.X.astype(np.float64) @ L.W.astype(np.float64) + L.bias[None, :]

    def err(lam, r):
        L1f, L2, _ = S.svd_factors(L.W, lam, r)
        act = S.act_tensor_scale(L.X, S.inverse_lambda(lam))
        pw = S.prepare("nvfp4", L.W, lam, L1f, L2, L.bias, act)
        Y = S.forward(pw, L.X)["Y"]
        return np.sqrt(np.mean((Y - ref) ** 2)) / np.sqrt(np.mean(ref ** 2))

    lam = S.smoothing_factors(L.X, L.W)
    e_svdq = err(lam, 32)
    e_smooth = err(lam, 0)
    e_plain = err(np.ones(L.K, np.float32), 0)
    assert e_svdq < e_smooth < e_plain, (e_svdq, e_smooth, e_plain)


# ------------------------------------------------------------ the fused GELU (tanh form)
def check_gelu_tanh():
    """gelu_tanh against PyTorch's own float64 tanh-approximation GELU (an
    implementation independent of this oracle) on a dense grid and far
    tails, plus facts that hold for the tanh form only: it is odd-symmetric
    about y/2 (g(y) - g(-y) = y), g(0) = 0, it differs from the erf-form GELU
    by at most 5e-4 but by more than 1e-4 near |y| = 2 (so it is not the erf
    form), and at y = 1 it equals 0.5 (1 + tanh(1.044715 sqrt(2/pi))) written
    with tanh from Python's math module."""
    import math
    import torch
    y = np.concatenate([np.arange(-12.0, 12.0, 1.0 / 64), [-1e3, -40.0, 40.0, 1e3], [0.0]])
    g = S.gelu_tanh(y)
    ref = torch.nn.functional.gelu(torch.from_numpy(y), approximate="tanh").numpy()
    assert np.all(np.abs(g - ref) <= 1e-14 * np.maximum(1.0, np.abs(ref))), np.max(np.abs(g - ref))
    assert S.gelu_tanh(np.array([0.0]))[0] == 0.0
    assert np.all(np.abs(S.gelu_tanh(y) - S.gelu_tanh(-y) - y) <= 1e-13 * np.maximum(1.0, np.abs(y)))
    erf_form = np.array([0.5 * v * (1.0 + math.erf(v / math.sqrt(2.0))) for v in y])
    gap = np.abs(g - erf_form)
    assert gap.max() <= 5e-4 and gap[np.abs(np.abs(y) - 2.0) < 0.5].max() > 1e-4
    one = 0.5 * (1.0 + math.tanh(math.sqrt(2.0 / math.pi) * 1.044715))
    assert abs(S.gelu_tanh(np.array([1.0]))[0] - one) <= 1e-15


def test_gelu_tanh_matches_the_tanh_form():
    check_gelu_tanh()
