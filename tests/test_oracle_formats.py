"""Pins for the oracle's number formats against the format definitions.

Each check is an independent restatement (a nearest-value search over the
format's grid, the golden tables from the OCP documents, torch's own
float32 -> bfloat16 conversion), not a re-run of the oracle's code."""
import numpy as np
import pytest
import torch

from conftest import read_golden
from oracle import formats as F


def _golden_table(name):
    out = {}
    for code, val in read_golden(name):
        out[int(code, 16)] = float(val)
    return out


# --------------------------------------------------------------------- E2M1
def check_e2m1_decode_table():
    for c, v in _golden_table("e2m1_ocp_mx_v1.txt").items():
        got = F.e2m1_decode(np.array([c]))[0]
        assert got == v and np.signbit(got) == np.signbit(v), (c, got, v)


def _e2m1_nearest(x):
    """Brute force: nearest E2M1 grid value by distance, ties to the even
    code, sign kept.  Grid values come from the golden OCP table."""
    tab = _golden_table("e2m1_ocp_mx_v1.txt")
    grid = [(tab[c], c) for c in range(8)]
    a = abs(float(x))
    best = min(abs(a - g) for g, _ in grid)
    cands = [c for g, c in grid if abs(a - g) == best]
    c = min(cands, key=lambda c: (c & 1, c))
    return c | (8 if np.signbit(x) else 0)


def _e2m1_sample():
    rng = np.random.default_rng(7)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0], np.float32)
    near = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(10))])
    pts = np.concatenate([
        near, -near,
        np.array([0.0, -0.0, 1e-30, -1e-30, 6.5, 7.0, 100.0, -1e9, 1.0, 0.5], np.float32),
        rng.uniform(-8, 8, 4000).astype(np.float32),
        (rng.standard_normal(2000) * 3).astype(np.float32),
    ]).astype(np.float32)
    return pts


def check_e2m1_encode_brute_force():
    x = _e2m1_sample()
    got = F.e2m1_encode(x)
    want = np.array([_e2m1_nearest(v) for v in x], np.uint8)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(float(x[i]), int(got[i]), int(want[i])) for i in bad[:5]]


def test_e2m1_decode_matches_ocp_table():
    check_e2m1_decode_table()


def test_e2m1_roundtrip_every_code():
    codes = np.arange(16)
    assert np.array_equal(F.e2m1_encode(F.e2m1_decode(codes).astype(np.float32)), codes)


def test_e2m1_encode_is_nearest_even_satfinite():
    check_e2m1_encode_brute_force()


# --------------------------------------------------------------------- E4M3
def test_e4m3_decode_matches_ocp_points():
    for c, v in _golden_table("e4m3_ocp_ofp8.txt").items():
        got = F.e4m3_decode(np.array([c]))[0]
        if np.isnan(v):
            assert np.isnan(got), c
        else:
            assert got == v and np.signbit(got) == np.signbit(v), (hex(c), got, v)


def test_e4m3_grid_structure():
    """Codes 0..126 are increasing; each binade above 2^-6 holds 8 equal steps
    of 2^(E-3); the subnormals are multiples of 2^-9."""
    v = F.e4m3_decode(np.arange(127))
    assert np.all(np.diff(v) > 0)
    assert np.allclose(v[:8], np.arange(8) * 2.0 ** -9, rtol=0, atol=0)
    for e in range(1, 16):
        blk = v[e * 8:(e + 1) * 8]
        if e == 15:
            blk = blk[:7]
        assert np.all(np.diff(blk) == 2.0 ** (e - 7 - 3))


def test_e4m3_roundtrip_every_finite_code():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F])
    assert np.array_equal(F.e4m3_encode_satfinite(F.e4m3_decode(codes).astype(np.float32)), codes)


def _e4m3_nearest(x):
    grid = F.e4m3_decode(np.arange(127))   # structure pinned above
    a = abs(float(x))
    d = np.abs(grid - a)
    best = d.min()
    cands = np.nonzero(d == best)[0]
    c = int(min(cands, key=lambda c: (c & 1, c)))
    return c | (0x80 if np.signbit(x) else 0)


def test_e4m3_encode_is_nearest_even_satfinite():
    rng = np.random.default_rng(3)
    grid = F.e4m3_decode(np.arange(127))
    mids = ((grid[1:] + grid[:-1]) / 2).astype(np.float32)
    x = np.concatenate([
        mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e4)),
        np.array([0.0, 1e-12, 2.0 ** -10, 2.0 ** -10 * 1.0001, 448.0, 449.0, 464.0, 480.0, 1e6], np.float32),
        np.exp(rng.uniform(np.log(1e-4), np.log(600), 5000)).astype(np.float32),
    ]).astype(np.float32)
    got = F.e4m3_encode_satfinite(x)
    want = np.array([_e4m3_nearest(v) for v in x], np.uint8)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(float(x[i]), int(got[i]), int(want[i])) for i in bad[:5]]


# --------------------------------------------------------------------- bf16 / fp16 / int4
def test_bf16_round_matches_torch_on_float32_inputs():
    rng = np.random.default_rng(11)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
                        np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 0.0, -0.0])]).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy().astype(np.float64)
    got = F.bf16_round(x.astype(np.float64))
    assert np.array_equal(got, want)


def test_bf16_round_float64_is_single_rounding():
    """A float64 value just above a bf16 tie must round up, although the same
    value rounded to float32 first would land on the tie and go to even."""
    x = 1.0 + 2.0 ** -8 + 2.0 ** -40           # float32(x) == 1 + 2^-8 (a tie)
    assert F.bf16_round(np.array([x]))[0] == 1.0 + 2.0 ** -7
    assert F.bf16_round(np.array([1.0 + 2.0 ** -8]))[0] == 1.0


def test_fp16_points():
    v = F.to_fp16(np.array([65504.0, 2.0 ** -24, 1 + 2 ** -11, 1 + 3 * 2 ** -11, 70000.0], np.float32))
    assert v[0] == 65504.0 and v[1] == 2.0 ** -24
    assert v[2] == 1.0 and v[3] == 1 + 2 ** -9      # ties to even
    assert np.isinf(v[4])


def test_int4_encode_half_even_and_clamp():
    x = np.array([0.5, 1.5, 2.5, -0.5, -1.5, 7.4, 7.6, -8.4, -9.0, 3.49], np.float32)
    assert F.int4_encode(x).tolist() == [0, 2, 2, 0, -2, 7, 7, -8, -8, 3]


def test_nibble_order_low_first():
    codes = np.array([[1, 2, 3, 4]], np.uint8)
    assert F.pack_nibbles(codes).tolist() == [[0x21, 0x43]]
    assert np.array_equal(F.unpack_nibbles(F.pack_nibbles(codes)), codes)
    assert F.int4_from_nibble(np.array([0x8, 0xF, 0x7])).tolist() == [-8, -1, 7]
