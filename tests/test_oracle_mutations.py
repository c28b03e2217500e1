"""Plants plausible mistakes in the oracle (on the CPU, via monkeypatch) and
checks that at least one pin catches each.  This shows the pins are strong
enough to trust the oracle as the parity reference."""
import numpy as np
import pytest

from oracle import formats as F
from oracle import svdquant as S
import test_oracle_formats as TF
import test_oracle_layer as TL
import test_oracle_quant as TQ


def _fails(fn, *a, **k):
    try:
        fn(*a, **k)
    except AssertionError:
        return True
    return False


def test_mutation_e2m1_ties_away_from_zero(monkeypatch):
    def bad(v):
        v = np.asarray(v, np.float64)
        a = np.abs(v)
        mag = ((a >= 0.25).astype(np.int64) + (a >= 0.75) + (a >= 1.25) + (a >= 1.75)
               + (a >= 2.5) + (a >= 3.5) + (a >= 5.0))
        return (mag | (np.signbit(v).astype(np.int64) << 3)).astype(np.uint8)
    monkeypatch.setattr(F, "e2m1_encode", bad)
    assert _fails(TF.check_e2m1_encode_brute_force)


def test_mutation_residual_sign(monkeypatch):
    orig = S.residual

    def bad(W, lam, L1f, L2):
        lam64 = np.asarray(lam, np.float32).astype(np.float64)[:, None]
        return (lam64 * np.asarray(W, np.float64) + lam64 * (np.asarray(L1f) @ np.asarray(L2))).astype(np.float32)
    monkeypatch.setattr(S, "residual", bad)
    assert _fails(TL.check_unquantized_reduces_to_xw, False)
    monkeypatch.setattr(S, "residual", orig)


def test_mutation_lambda_on_wrong_side(monkeypatch):
    monkeypatch.setattr(S, "smooth_activation",
                        lambda X, inv: (np.asarray(X, np.float32) / np.asarray(inv, np.float32)[None, :]).astype(np.float32))
    assert _fails(TL.check_unquantized_reduces_to_xw, False)


def test_mutation_dropped_bias(monkeypatch):
    monkeypatch.setattr(S, "epilogue", lambda y, bias, gelu: F.bf16_round(S.gelu_tanh(y) if gelu else y))
    assert _fails(TL.check_brute_force, "nvfp4", 8, 16, 16, 4, 41)


def test_mutation_missing_tensor_scale(monkeypatch):
    def bad(pw, qX, sX):
        return S.dequantize_nvfp4(qX, sX) @ S.dequantize_nvfp4(pw.qR, pw.sR).T
    monkeypatch.setattr(S, "main_product", bad)
    assert _fails(TL.check_brute_force, "nvfp4", 8, 16, 16, 4, 41)


def test_mutation_transposed_weight_codes(monkeypatch):
    orig = S.prepare

    def bad(*a, **k):
        pw = orig(*a, **k)
        pw.qR = pw.qR.reshape(pw.K, pw.N).T.copy() if pw.K == pw.N else pw.qR[::-1].copy()
        return pw
    monkeypatch.setattr(S, "prepare", bad)
    assert _fails(TL.check_brute_force, "nvfp4", 8, 16, 16, 4, 41)


def test_mutation_int4_scale_without_fp16(monkeypatch):
    monkeypatch.setattr(F, "to_fp16", lambda v: np.asarray(v, np.float32))
    assert _fails(TL.check_brute_force, "int4", 4, 64, 8, 4, 43)


def test_mutation_lowrank_not_rounded(monkeypatch):
    orig = S.lowrank_down
    monkeypatch.setattr(S, "lowrank_down", lambda X, L1f, round_bf16=True: orig(X, L1f, False))
    assert _fails(TL.check_brute_force, "nvfp4", 8, 16, 16, 4, 41)


def test_mutation_act_tensor_scale_divides_by_448(monkeypatch):
    def bad(X, inv_lam):
        a = np.float32(np.max(np.abs(S.smooth_activation(X, inv_lam)))) if np.size(X) else np.float32(0)
        return np.float32(1.0) if a == 0 else np.float32(a / np.float32(448.0))
    monkeypatch.setattr(S, "act_tensor_scale", bad)
    assert _fails(TQ.check_act_tensor_scale_definition)


def test_mutation_act_tensor_scale_amax_over_raw_x(monkeypatch):
    def bad(X, inv_lam):
        a = np.float32(np.max(np.abs(np.asarray(X, np.float32)))) if np.size(X) else np.float32(0)
        return np.float32(1.0) if a == 0 else np.float32(a / S.NVFP4_TENSOR_DIVISOR)
    monkeypatch.setattr(S, "act_tensor_scale", bad)
    assert _fails(TQ.check_act_tensor_scale_definition)


def test_mutation_act_tensor_scale_without_abs(monkeypatch):
    def bad(X, inv_lam):
        a = np.float32(np.max(S.smooth_activation(X, inv_lam))) if np.size(X) else np.float32(0)
        return np.float32(1.0) if a == 0 else np.float32(a / S.NVFP4_TENSOR_DIVISOR)
    monkeypatch.setattr(S, "act_tensor_scale", bad)
    assert _fails(TQ.check_act_tensor_scale_definition)


def test_mutation_gelu_erf_form(monkeypatch):
    import math
    monkeypatch.setattr(S, "gelu_tanh", lambda y: np.array(
        [0.5 * v * (1.0 + math.erf(v / math.sqrt(2.0))) for v in np.asarray(y, np.float64).ravel()]).reshape(np.shape(y)))
    assert _fails(TL.check_gelu_tanh)


def test_mutation_gelu_wrong_cubic_coefficient(monkeypatch):
    def bad(y):
        y = np.asarray(y, np.float64)
        return 0.5 * y * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (y + 0.0447 * y ** 3)))
    monkeypatch.setattr(S, "gelu_tanh", bad)
    assert _fails(TL.check_gelu_tanh)


def test_mutation_gelu_missing_half(monkeypatch):
    def bad(y):
        y = np.asarray(y, np.float64)
        return y * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (y + 0.044715 * y ** 3)))
    monkeypatch.setattr(S, "gelu_tanh", bad)
    assert _fails(TL.check_gelu_tanh)
