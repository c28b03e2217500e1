"""Pins for the oracle's 4-bit group quantizers: closed-form blocks, the
special cases of the scale rule, and the rounding-error bound that every
element must meet."""
import numpy as np

from oracle import formats as F
from oracle import svdquant as S


def _block(vals, n=16):
    v = np.zeros((1, n), np.float32)
    v[0, :len(vals)] = vals
    return v


# --------------------------------------------------------------------- NVFP4 closed forms
def test_nvfp4_closed_form_block():
    # s_t = 1, amax 12 -> block scale 12 / 6 = 2 (E4M3 0x40), d = 2, inv = 0.5
    q, s = S.quantize_nvfp4(_block([12, -12, 6, 3, 1, 0.5, -1, 0, 2.5, -5.5]), 1.0)
    assert s.tolist() == [[0x40]]
    # v * 0.5 = 6, -6, 3, 1.5, 0.5, 0.25(tie->0), -0.5, 0, 1.25(tie->1.0), -2.75(->-3)
    assert q[0, :10].tolist() == [0x7, 0xF, 0x5, 0x3, 0x1, 0x0, 0x9, 0x0, 0x2, 0xD]


def test_nvfp4_tensor_scale_enters_block_scale():
    s_t = np.float32(0.125)                 # power of two: every step exact
    q, s = S.quantize_nvfp4(_block([3.0, -1.5]), s_t)
    # a / (6 s_t) = 3 / 0.75 = 4 -> E4M3 0x48 ; d = 4 * 0.125 = 0.5 ; inv = 2
    assert s.tolist() == [[0x48]]
    assert q[0, :2].tolist() == [0x7, 0xD]  # 6, -3


def test_nvfp4_scale_saturates_at_448():
    q, s = S.quantize_nvfp4(_block([3000.0, -1.0]), 1.0)
    assert s.tolist() == [[0x7E]]            # 500 -> 448
    assert q[0, 0] == 0x7                    # 3000/448 = 6.7 -> saturates to 6


def test_nvfp4_zero_and_underflow_blocks_give_signed_zero_codes():
    q, s = S.quantize_nvfp4(np.zeros((1, 16), np.float32), 1.0)
    assert s.tolist() == [[0]] and np.all(q == 0)
    tiny = _block([1e-6, -1e-6, -0.0])       # a / 6 = 1.7e-7 < 2^-10: scale rounds to 0
    q, s = S.quantize_nvfp4(tiny, 1.0)
    assert s.tolist() == [[0]]
    assert q[0, :3].tolist() == [0x0, 0x8, 0x8]


def test_nvfp4_error_bound_every_element():
    """|dequant - v| <= half the E2M1 step at |v inv| (times d), unless the
    code saturated; and the block scale is the nearest E4M3 value."""
    rng = np.random.default_rng(5)
    V = (rng.standard_normal((64, 256)) * np.exp(rng.uniform(-3, 3, (64, 1)))).astype(np.float32)
    s_t = S.tensor_scale(V)
    q, s = S.quantize_nvfp4(V, s_t)
    sb = F.e4m3_decode(s).astype(np.float32)
    d = (sb * s_t).astype(np.float32)
    a = np.abs(V).reshape(64, 16, 16).max(axis=2)
    target = (a / np.float32(6.0 * s_t)).astype(np.float64)
    # scale: within half an E4M3 step of a / (6 s_t)
    e = np.maximum(np.floor(np.log2(np.maximum(target, 2.0 ** -6))), -6)
    assert np.all(np.abs(sb - target) <= 0.5 * 2.0 ** (e - 3) * (1 + 1e-9))
    deq = F.e2m1_decode(q).reshape(64, 16, 16) * d[:, :, None]
    x = (np.abs(V.reshape(64, 16, 16)) / d[:, :, None])
    step = np.where(x < 2, 0.5, np.where(x < 4, 1.0, 2.0))
    err = np.abs(deq - V.reshape(64, 16, 16))
    ok = (err <= 0.5 * step * d[:, :, None] * (1 + 1e-6)) | (x > 6)
    assert ok.all()


def test_nvfp4_groups_run_along_k_per_row():
    rng = np.random.default_rng(1)
    V = rng.standard_normal((4, 64)).astype(np.float32)
    _, s0 = S.quantize_nvfp4(V, 0.01)
    V2 = V.copy()
    V2[2, 37] = 50.0
    _, s1 = S.quantize_nvfp4(V2, 0.01)
    diff = np.argwhere(s0 != s1)
    assert diff.tolist() == [[2, 37 // 16]]


# --------------------------------------------------------------------- INT4
def test_int4_closed_form_block():
    v = np.zeros((1, 64), np.float32)
    v[0, :6] = [7, -7, 3.5, 2.5, -0.5, 0.4]
    q, s = S.quantize_int4(v)
    assert s.dtype == np.float16 and float(s[0, 0]) == 1.0
    assert q[0, :6].tolist() == [7, -7, 4, 2, 0, 0]


def test_int4_error_bound_every_element():
    rng = np.random.default_rng(9)
    V = (rng.standard_normal((32, 256)) * np.exp(rng.uniform(-4, 4, (32, 1)))).astype(np.float32)
    q, s = S.quantize_int4(V)
    d = s.astype(np.float64)
    deq = q.reshape(32, 4, 64) * d[:, :, None]
    err = np.abs(deq - V.reshape(32, 4, 64))
    # |v inv| can exceed 7 only by the fp16 rounding of a/7 (relative 2^-11)
    assert np.all(err <= d[:, :, None] * (0.5 + 7 * 2.0 ** -10))


def test_int4_zero_block():
    q, s = S.quantize_int4(np.zeros((2, 128), np.float32))
    assert np.all(q == 0) and np.all(s == 0)


def test_weight_tensor_scale_pairs_to_a_power_of_two():
    rng = np.random.default_rng(12)
    for trial in range(200):
        R = (rng.standard_normal((8, 64)) * np.exp(rng.uniform(-12, 6))).astype(np.float32)
        s_tX = np.float32(np.exp(rng.uniform(-12, 2)))
        s_tR, k = S.weight_tensor_scale(R, s_tX)
        amax = float(np.max(np.abs(R)))
        # 2^k is the smallest power of two >= s_tX amax / 2688
        assert 2.0 ** k >= s_tX * amax / 2688 and 2.0 ** (k - 1) < s_tX * amax / 2688
        # s_tX s_tR = 2^k within one float32 rounding
        assert abs(float(s_tX) * float(s_tR) / 2.0 ** k - 1) <= 2.0 ** -24
        # no block scale beyond E4M3's range is needed, and the largest is at least 224
        _, sc = S.quantize_nvfp4(R, s_tR)
        top = F.e4m3_decode(sc).max()
        assert 224 <= top <= 448


# ------------------------------------------------------------ per-call (dynamic) activation tensor scale
def _prepared_small():
    import workloads
    L = workloads.draw_layer("dyn", "nvfp4", 48, 128, 64, 8, seed=31, n_out=3)
    return L, S.calibrate_and_prepare("nvfp4", L.X, L.W, L.bias, L.rank)


def test_dynamic_scale_pairs_to_a_power_of_two_and_covers_the_batch():
    L, pw = _prepared_small()
    for f in (1.0, 3.0, 0.01, 250.0):
        X = (L.X * np.float32(f)).astype(np.float32)
        s, j = S.dynamic_act_scale(pw, X)
        a = float(np.max(np.abs(S.smooth_activation(X, pw.inv_lam))))
        # alpha = s s_tR is 2^j up to the one float32 rounding of s
        assert abs(float(s) * float(pw.s_tR) / 2.0 ** j - 1.0) < 2.0 ** -23
        # the scale covers the batch (no block scale above 448) and is within a factor 2 of the tight one
        assert float(s) * 2688.0 >= a * (1 - 2.0 ** -23)
        assert float(s) * 2688.0 < 2.0 * a * (1 + 2.0 ** -23)
        qX, sX = S.quantize_nvfp4(S.smooth_activation(X, pw.inv_lam), s)
        assert F.e4m3_decode(sX).max() <= 448.0


def test_dynamic_scale_is_tight_at_an_exact_power_of_two():
    # "smallest j with 2^j >= s_tR a / 2688": when that ratio is exactly 2^t,
    # j = t and the scale is tight (s 2688 = a), not one power above
    from dataclasses import replace
    L, pw = _prepared_small()
    for t_r, k in ((-10, 3), (-7, -2), (-12, 0)):
        pw2 = replace(pw, s_tR=np.float32(2.0 ** t_r), inv_lam=np.ones_like(pw.inv_lam))
        X = np.zeros((4, L.K), np.float32)
        X[1, 5] = np.float32(-2688.0 * 2.0 ** k)      # exact in bf16: 2688 = 21 * 2^7
        X[2, 7] = np.float32(1.5)
        s, j = S.dynamic_act_scale(pw2, X)
        assert j == k + t_r
        assert float(s) * 2688.0 == 2688.0 * 2.0 ** k


def test_dynamic_scale_is_equivariant_under_powers_of_two():
    # scaling X by 2^p scales the dynamic tensor scale by 2^p exactly and leaves every code and block scale
    L, pw = _prepared_small()
    s0, j0 = S.dynamic_act_scale(pw, L.X)
    q0, b0 = S.quantize_nvfp4(S.smooth_activation(L.X, pw.inv_lam), s0)
    for p in (-3, 2, 5):
        X = (L.X * np.float32(2.0 ** p)).astype(np.float32)
        s, j = S.dynamic_act_scale(pw, X)
        assert j == j0 + p and float(s) == float(s0) * 2.0 ** p
        q, b = S.quantize_nvfp4(S.smooth_activation(X, pw.inv_lam), s)
        assert np.array_equal(q, q0) and np.array_equal(b, b0)


def test_dynamic_forward_tracks_the_batch_where_the_static_scale_saturates():
    # a batch 1000x larger than the calibration one: the static scale clips every block above
    # 6 * 448 * s_tX, the dynamic one follows the batch and keeps the calibration-level error
    L, pw = _prepared_small()
    rel = lambda Y, X: float(np.sqrt(np.mean((Y - (X.astype(np.float64) @ L.W.astype(np.float64) + L.bias[None, :])) ** 2))
                             / np.sqrt(np.mean((X.astype(np.float64) @ L.W.astype(np.float64) + L.bias[None, :]) ** 2)))
    e_calib = rel(S.forward(pw, L.X)["Y"], L.X)
    X = (L.X * np.float32(1000.0)).astype(np.float32)
    e_static = rel(S.forward(pw, X)["Y"], X)
    e_dynamic = rel(S.forward(pw, X, dynamic=True)["Y"], X)
    assert e_dynamic < 1.05 * e_calib + 1e-4
    assert e_static > 3 * e_dynamic


# ------------------------------------------------------------ static NVFP4 activation tensor scale
def check_act_tensor_scale_definition():
    """act_tensor_scale = amax(|X^|) / 2688 (2688 = 6 x 448, the largest
    E2M1 magnitude times the largest E4M3 block scale), with X^ = X / lambda.
    Hand-built so that every step is exact: lambda is a power of two per
    channel, the largest |X^| is 336 = 2688 / 8 (so the scale is 0.125), it
    is a negative entry, and it sits in a channel whose raw |X| is NOT the
    largest (channel 3 holds |X| = 400, which lambda = 4 brings down to 100).
    Dividing by 448, taking the amax over X instead of X^, or dropping the
    absolute value all give another number."""
    lam = np.array([1.0, 2.0, 0.5, 4.0], np.float32)
    X = np.array([[10.0, -30.0, -168.0, 400.0],
                  [-50.0, 60.0, 20.0, -8.0]], np.float32)
    inv = S.inverse_lambda(lam)
    assert np.array_equal(inv, np.array([1.0, 0.5, 2.0, 0.25], np.float32))
    s = S.act_tensor_scale(X, inv)
    assert s.dtype == np.float32 and s == np.float32(0.125), s
    # a second exact point: amax(|X^|) = 2688 * 2^-10 -> 2^-10
    X2 = np.array([[2.625, -1.0, 0.5, 0.0]], np.float32)            # X^ = 2.625, -0.5, 1, 0
    assert S.act_tensor_scale(X2, inv) == np.float32(2.0 ** -10)
    # an all-zero calibration batch gives the reading's fallback of 1
    assert S.act_tensor_scale(np.zeros((3, 4), np.float32), inv) == np.float32(1.0)
    # with the calibrated scale, the block holding the batch's amax gets the
    # largest E4M3 block scale, 448, and its amax element code 6 (E2M1 0x7)
    codes, sc = S.quantize_nvfp4(np.pad(S.smooth_activation(X, inv), ((0, 0), (0, 12))), s)
    assert F.e4m3_decode(sc[0])[0] == 448.0 and codes[0, 2] == 0xF    # -6: sign bit + code 7


def test_act_tensor_scale_definition():
    check_act_tensor_scale_definition()
