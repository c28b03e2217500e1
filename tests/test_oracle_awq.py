"""Pins of the AWQ W4A16 oracle (oracle/awq.py) against what the pages and
the mathematics fix, independent of the oracle's own formulas: the page's
group size, brute-force nearest-grid codes, exact reconstruction of values
on the grid, the rounding bound, the closed form of a constant group,
invariance under a uniform power-of-two AWQ scale, and the layer output
against exact rational arithmetic on a tiny case."""
from fractions import Fraction

import numpy as np
import pytest

from conftest import read_golden
from oracle import awq as A
from oracle import formats as F


def _page(key):
    for row in read_golden("page_parameters.txt"):
        if row[0] == key:
            return int(row[1])
    raise KeyError(key)


def _rand(shape, seed, scale=0.02):
    rng = np.random.default_rng(seed)
    return F.bf16_round(rng.standard_normal(shape) * scale).astype(np.float32)


def test_group_size_and_bits_are_the_pages():
    assert A.GROUP == _page("awq_w4a16_group_size")
    assert A.MAX_CODE == 2 ** _page("awq_w4a16_weight_bits") - 1


def test_codes_are_the_nearest_grid_point_by_brute_force():
    W = _rand((2 * A.GROUP, 7), 1)
    W[3, 2] = 0.3                       # one outlier stretches its group's range
    code, d, zero = A.quantize_groups(W)
    for g in range(2):
        for n in range(7):
            dd, z = float(d[g, n]), int(zero[g, n])
            for k in range(g * A.GROUP, (g + 1) * A.GROUP):
                t = float(np.float32(np.float32(W[k, n]) / np.float32(dd)))   # the float32 quotient
                # nearest c in 0..15 to t + z; a tie goes to the even (c - z), as round-half-even does
                best = min(range(16), key=lambda c: (abs(t + z - c), (c - z) % 2))
                assert code[k, n] == best, (k, n, t, z)


def test_values_on_the_grid_reconstruct_exactly():
    d0 = 2.0 ** -8                      # exact in binary16
    col = np.array([(j - 5) * d0 for j in range(16)] * 4, np.float32)   # lo = -5 d0, hi = 10 d0
    W = np.stack([col, col[::-1]], axis=1)
    aw = A.prepare(W, np.zeros(2))
    assert np.all(aw.scale == np.float32(d0)) and np.all(aw.zero == 5)
    assert np.array_equal(A.dequantize(aw), W.astype(np.float64))


def test_rounding_error_is_at_most_half_a_step():
    W = _rand((4 * A.GROUP, 33), 2)
    aw = A.prepare(W, np.zeros(33))
    err = np.abs(A.dequantize(aw) - W.astype(np.float64))
    d = np.repeat(aw.scale.astype(np.float64), A.GROUP, axis=0)
    clamped = (aw.code == 0) | (aw.code == A.MAX_CODE)
    # the float32 quotient adds at most 2^-24 relative on |w/d| <= 16
    assert np.all(err[~clamped] <= d[~clamped] * (0.5 + 2.0 ** -19))
    # at the ends of the range the binary16 rounding of the step can push a value one
    # rounding of the scale past the grid: 15 steps of at most 2^-11 relative each
    assert np.all(err <= d * (0.5 + 15 * 2.0 ** -11))


def test_constant_group_closed_form():
    c = np.float32(1e-6)
    W = np.full((A.GROUP, 1), c, np.float32)
    code, d, zero = A.quantize_groups(W)
    # range 0 -> the 1e-5 floor: d = binary16(1e-5 / 15), a subnormal: 11 * 2^-24
    assert d[0, 0] == np.float32(11 * 2.0 ** -24)
    # -c / d = -1.51.. -> rint -2 -> clamped to 0; c / d = 1.51.. -> 2
    assert zero[0, 0] == 0 and np.all(code == 2)
    z = A.quantize_groups(np.zeros((A.GROUP, 1), np.float32))
    assert np.all(z[0] == 0) and z[2][0, 0] == 0


@pytest.mark.parametrize("p", [-3, 4])
def test_uniform_power_of_two_scale_changes_nothing(p):
    W = _rand((3 * A.GROUP, 10), 3)
    X = _rand((4, 3 * A.GROUP), 4, 1.0)
    b = _rand((10,), 5, 0.01)
    a1 = A.prepare(W, b)
    a2 = A.prepare(W, b, s=np.full(3 * A.GROUP, 2.0 ** p, np.float32))
    assert np.array_equal(a1.code, a2.code) and np.array_equal(a1.zero, a2.zero)
    assert np.array_equal(a2.scale, (a1.scale * np.float32(2.0 ** p)).astype(np.float32))
    assert np.array_equal(A.forward(a1, X)["Y"], A.forward(a2, X)["Y"])


def test_awq_scaling_keeps_the_product():
    # X' W' = X W before quantization, for any positive s (up to the two float32 roundings)
    W = _rand((2 * A.GROUP, 6), 6)
    X = _rand((3, 2 * A.GROUP), 7, 1.0)
    s = np.exp(np.random.default_rng(8).uniform(-1, 1, 2 * A.GROUP)).astype(np.float32)
    aw = A.prepare(W, np.zeros(6), s=s)
    lhs = A.scaled_activation(aw, X).astype(np.float64) @ A.scaled_weight(W, s).astype(np.float64)
    rhs = X.astype(np.float64) @ W.astype(np.float64)
    assert np.allclose(lhs, rhs, rtol=0, atol=1e-6 * np.abs(X).sum() * np.abs(W).max())


def test_forward_against_exact_rationals():
    W = _rand((A.GROUP, 3), 9)
    X = _rand((2, A.GROUP), 10, 1.0)
    b = _rand((3,), 11, 0.01)
    aw = A.prepare(W, b)
    Y = A.forward(aw, X)["Y"]
    for m in range(2):
        for n in range(3):
            acc = Fraction(float(b[n]))
            for k in range(A.GROUP):
                wq = (int(aw.code[k, n]) - int(aw.zero[0, n])) * Fraction(float(aw.scale[0, n]))
                acc += Fraction(float(X[m, k])) * wq
            assert Y[m, n] == F.bf16_round(float(acc)), (m, n)


# ------------------------------------------------------------ the 16-bit-operand (tensor-core) form
def _bf16_of_exact(q: Fraction) -> float:
    """The bf16 value nearest to an exact rational (ties to the even
    significand): the two multiples of the binade's step around it."""
    import math
    if q == 0:
        return 0.0
    a = abs(q)
    e = math.floor(math.log2(float(a)))
    while Fraction(2) ** e > a:          # the exact binade: 2^e <= |q| < 2^(e+1)
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    step = Fraction(2) ** (max(e, -126) - 7)
    lo = (a / step).__floor__()
    d_lo, d_hi = a - lo * step, (lo + 1) * step - a
    c = lo if (d_lo < d_hi or (d_lo == d_hi and lo % 2 == 0)) else lo + 1
    return math.copysign(float(c * step), float(q))


def check_forward_16bit_against_exact_rationals(s_kind="none"):
    """forward_16bit by the definition written out: every dequantized weight
    and every scaled activation rounded once to bf16 from its exact value,
    the sum in exact rationals, the output rounded once."""
    W = _rand((2 * A.GROUP, 3), 21, 0.05)
    X = _rand((2, 2 * A.GROUP), 22, 1.0)
    b = _rand((3,), 23, 0.01)
    s = None if s_kind == "none" else np.exp(np.random.default_rng(24).uniform(-1, 1, 2 * A.GROUP)).astype(np.float32)
    aw = A.prepare(W, b, s=s)
    Y = A.forward_16bit(aw, X)["Y"]
    inv_s = [np.float32(1.0) / np.float32(v) for v in (s if s is not None else np.ones(2 * A.GROUP, np.float32))]
    for m in range(2):
        for n in range(3):
            acc = Fraction(float(b[n]))
            for k in range(2 * A.GROUP):
                g = k // A.GROUP
                w16 = _bf16_of_exact((int(aw.code[k, n]) - int(aw.zero[g, n])) * Fraction(float(aw.scale[g, n])))
                x16 = _bf16_of_exact(Fraction(float(np.float32(np.float32(X[m, k]) * inv_s[k]))))
                acc += Fraction(x16) * Fraction(w16)
            assert Y[m, n] == _bf16_of_exact(acc), (m, n)


def test_forward_16bit_against_exact_rationals():
    check_forward_16bit_against_exact_rationals("none")


def test_forward_16bit_with_awq_scale_against_exact_rationals():
    check_forward_16bit_against_exact_rationals("random")


def test_forward_16bit_is_forward_when_the_weights_fit_16_bits():
    """With scales that are powers of two, (code - zero) d has at most 4
    significant bits, and with s = 1 X' is X: the two forms then compute the
    same exact sum and give identical outputs."""
    d0 = 2.0 ** -7
    rng = np.random.default_rng(25)
    # every group spans exactly 15 steps (lo = -7 d0, hi = 8 d0), values on the grid
    W = (rng.integers(-7, 9, (3 * A.GROUP, 5)) * d0).astype(np.float32)
    W[0::A.GROUP] = -7 * d0
    W[1::A.GROUP] = 8 * d0
    X = _rand((6, 3 * A.GROUP), 26, 1.0)
    b = _rand((5,), 27, 0.01)
    aw = A.prepare(W, b)
    assert np.all(aw.scale == np.float32(d0))
    assert np.array_equal(A.dequantize_16bit(aw), A.dequantize(aw))
    assert np.array_equal(A.forward_16bit(aw, X)["Y"], A.forward(aw, X)["Y"])


def test_forward_16bit_stays_within_the_weight_rounding_of_forward():
    """|Y16 - Y| <= sum_k |x'_k| |w^16 - w^| + the activations' bf16 rounding
    + one bf16 ulp of each output: the 16-bit form only adds the roundings it
    names."""
    W = _rand((4 * A.GROUP, 40), 28)
    X = _rand((8, 4 * A.GROUP), 29, 1.0)
    aw = A.prepare(W, np.zeros(40))
    o, o16 = A.forward(aw, X), A.forward_16bit(aw, X)
    dw = np.abs(o16["W16"] - A.dequantize(aw))
    bound = np.abs(o["Xp"]) @ dw + np.abs(o16["Xp16"] - o["Xp"]) @ np.abs(o16["W16"])
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(o["Y"]), 1e-30))) - 7)
    assert np.all(np.abs(o16["Y"] - o["Y"]) <= bound + 2 * ulp + 1e-12)
    assert np.any(dw > 0)        # the case does exercise the rounding
