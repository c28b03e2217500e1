"""Plants plausible mistakes in the AWQ W4A16 and randomized-split oracles
(on the CPU, via monkeypatch) and checks that at least one of their pins
catches each, as test_oracle_mutations.py does for the W4A4 oracle."""
import numpy as np

from oracle import awq as A
from oracle import formats as F
from oracle import rsvd as R
from oracle import svdquant as S
import test_oracle_awq as TA
import test_oracle_quant as TQ
import test_oracle_rsvd as TR


def _fails(fn, *a, **k):
    try:
        fn(*a, **k)
    except AssertionError:
        return True
    return False


# ---------------------------------------------------------------- AWQ W4A16
def test_mutation_awq_zero_point_subtracted(monkeypatch):
    def bad(Wp):
        Wp = np.asarray(Wp, np.float32)
        K, N = Wp.shape
        G = Wp.reshape(K // A.GROUP, A.GROUP, N)
        lo, hi = G.min(axis=1), G.max(axis=1)
        d = A.fp16_satfinite((np.maximum((hi - lo).astype(np.float32), A.MIN_RANGE) / np.float32(15)).astype(np.float32))
        zero = np.clip(np.rint((-lo / d).astype(np.float32)), 0, 15)
        q = np.rint((G / d[:, None, :]).astype(np.float32)) - zero[:, None, :]
        return np.clip(q, 0, 15).astype(np.uint8).reshape(K, N), d.astype(np.float32), zero.astype(np.uint8)
    monkeypatch.setattr(A, "quantize_groups", bad)
    assert _fails(TA.test_codes_are_the_nearest_grid_point_by_brute_force)


def test_mutation_awq_scale_not_rounded_to_binary16(monkeypatch):
    monkeypatch.setattr(A, "fp16_satfinite", lambda v: np.asarray(v, np.float32))
    assert _fails(TA.test_constant_group_closed_form)


def test_mutation_awq_dequantize_adds_the_zero_point(monkeypatch):
    def bad(aw):
        z = np.repeat(aw.zero.astype(np.float64), A.GROUP, axis=0)
        d = np.repeat(aw.scale.astype(np.float64), A.GROUP, axis=0)
        return (aw.code.astype(np.float64) + z) * d
    monkeypatch.setattr(A, "dequantize", bad)
    assert _fails(TA.test_values_on_the_grid_reconstruct_exactly)


def test_mutation_awq_activation_scaled_the_wrong_way(monkeypatch):
    monkeypatch.setattr(A, "scaled_activation",
                        lambda aw, X: (np.asarray(X, np.float32) * aw.s[None, :]).astype(np.float32))
    assert _fails(TA.test_awq_scaling_keeps_the_product)


def test_mutation_awq_bias_dropped(monkeypatch):
    def bad(aw, X):
        Xp = A.scaled_activation(aw, X).astype(np.float64)
        return dict(Xp=Xp, Y=F.bf16_round(Xp @ A.dequantize(aw)))
    monkeypatch.setattr(A, "forward", bad)
    assert _fails(TA.test_forward_against_exact_rationals)


# ---------------------------------------------------------------- randomized split
def test_mutation_philox_key_schedule(monkeypatch):
    orig = R.philox4x32_10

    def bad(ctr, key):
        return orig(ctr, ((int(key[0]) + 1) & R.MASK32, key[1]))
    monkeypatch.setattr(R, "philox4x32_10", bad)
    assert _fails(TR.test_philox_known_answers)


def test_mutation_rademacher_signs_inverted(monkeypatch):
    orig = R.rademacher
    monkeypatch.setattr(R, "rademacher", lambda rows, cols, seed=R.DEFAULT_SEED: -orig(rows, cols, seed))
    assert _fails(TR.test_rademacher_signs_follow_the_stream)


def test_mutation_no_subspace_iteration(monkeypatch):
    orig = R.randomized_svd
    monkeypatch.setattr(R, "randomized_svd", lambda What, rank, seed=R.DEFAULT_SEED: orig(What, rank, seed, q=0))
    assert _fails(TR.test_near_optimal_on_a_decaying_spectrum)


def test_mutation_right_vectors_not_normalised(monkeypatch):
    orig = R.randomized_svd

    def bad(What, rank, seed=R.DEFAULT_SEED):
        U, s, Vt = orig(What, rank, seed)
        return U, s, Vt * s[:rank, None]                  # Z P without the division by sigma
    monkeypatch.setattr(R, "randomized_svd", bad)
    assert _fails(TR.test_exact_recovery_when_the_rank_fits_the_sketch)


def test_mutation_sign_convention_flipped(monkeypatch):
    orig = R.randomized_svd

    def bad(What, rank, seed=R.DEFAULT_SEED):
        U, s, Vt = orig(What, rank, seed)
        return -U, s, -Vt
    monkeypatch.setattr(R, "randomized_svd", bad)
    assert _fails(TR.test_signs_and_near_optimality_on_the_synthetic_layer)


def test_mutation_lambda_multiplied_into_the_first_factor(monkeypatch):
    def bad(W, lam, rank, seed=R.DEFAULT_SEED):
        W = np.asarray(W, np.float64)
        lam64 = np.asarray(lam, np.float32).astype(np.float64)
        U, sigma, Vt = R.randomized_svd(lam64[:, None] * W, rank, seed)
        return F.bf16_round(U * sigma[None, :rank] * lam64[:, None]), F.bf16_round(Vt), sigma
    monkeypatch.setattr(R, "randomized_factors", bad)
    assert _fails(TR.test_folded_factors_rebuild_the_smoothed_weight)


# ---------------------------------------------------------------- per-call activation tensor scale
def test_mutation_dynamic_scale_exponent_not_smallest(monkeypatch):
    def bad(pw, X):                                    # frexp's exponent taken as is: one power too high at a tie
        Xh = S.smooth_activation(X, pw.inv_lam)
        a = float(np.max(np.abs(Xh))) if np.size(Xh) else 0.0
        x = (a if a > 0 else 2688.0) * float(np.float32(pw.s_tR)) / 2688.0
        j = int(np.frexp(x)[1])
        return np.float32(np.float32(np.ldexp(1.0, j)) / np.float32(pw.s_tR)), j
    monkeypatch.setattr(S, "dynamic_act_scale", bad)
    assert _fails(TQ.test_dynamic_scale_is_tight_at_an_exact_power_of_two)


def test_mutation_dynamic_scale_exponent_rounded_down(monkeypatch):
    def bad(pw, X):                                    # largest j with 2^j <= x: the scale no longer covers the batch
        Xh = S.smooth_activation(X, pw.inv_lam)
        a = float(np.max(np.abs(Xh))) if np.size(Xh) else 0.0
        x = (a if a > 0 else 2688.0) * float(np.float32(pw.s_tR)) / 2688.0
        j = int(np.floor(np.log2(x)))
        return np.float32(np.float32(np.ldexp(1.0, j)) / np.float32(pw.s_tR)), j
    monkeypatch.setattr(S, "dynamic_act_scale", bad)
    assert _fails(TQ.test_dynamic_scale_pairs_to_a_power_of_two_and_covers_the_batch)


def test_mutation_awq_16bit_weights_not_rounded(monkeypatch):
    monkeypatch.setattr(A, "dequantize_16bit", lambda aw: A.dequantize(aw))
    assert _fails(TA.check_forward_16bit_against_exact_rationals, "none")


def test_mutation_awq_16bit_scale_rounded_before_the_product(monkeypatch):
    def bad(aw):
        z = np.repeat(aw.zero.astype(np.float64), A.GROUP, axis=0)
        d = np.repeat(F.bf16_round(aw.scale.astype(np.float64)), A.GROUP, axis=0)
        return F.bf16_round((aw.code.astype(np.float64) - z) * d)
    monkeypatch.setattr(A, "dequantize_16bit", bad)
    assert _fails(TA.check_forward_16bit_against_exact_rationals, "none")


def test_mutation_awq_16bit_activation_scale_dropped(monkeypatch):
    def bad(aw, X):
        Xp16 = F.bf16_round(np.asarray(X, np.float64))
        y = Xp16 @ A.dequantize_16bit(aw) + aw.bias[None, :]
        return dict(Xp16=Xp16, W16=A.dequantize_16bit(aw), Y=F.bf16_round(y))
    monkeypatch.setattr(A, "forward_16bit", bad)
    assert _fails(TA.check_forward_16bit_against_exact_rationals, "random")
