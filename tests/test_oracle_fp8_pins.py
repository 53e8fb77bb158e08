"""Pins for the oracle's FP8 (E4M3) variant, none comparing the oracle with
itself: the format's defining values, a brute-force nearest-value search
over every finite code, an exact library float64 product, and the
smoothing identity within the E4M3 quantization error bound."""
import numpy as np
import pytest

import oracle
from tests.golden.load import load

CODES = np.arange(256, dtype=np.uint8)


def _finite_table():
    vals = oracle.e4m3_decode(CODES)
    ok = ~np.isnan(vals)
    return CODES[ok], vals[ok].astype(np.float64)


def test_defining_values():
    g = load("p8_e4m3_values.txt")
    codes = np.array([int(c) for c in g["codes"]], np.uint8)
    vals = np.array([float(v) for v in g["values"]], np.float32)
    np.testing.assert_array_equal(oracle.e4m3_decode(codes), vals)
    assert np.signbit(oracle.e4m3_decode(np.array([0x80], np.uint8)))[0]
    assert np.isnan(oracle.e4m3_decode(np.array([int(c) for c in g["nan_codes"]], np.uint8))).all()
    # exactly two NaN codes; every other code is finite
    assert int(np.isnan(oracle.e4m3_decode(CODES)).sum()) == 2
    # and the encoder maps NaN onto the format's NaN pattern S.1111.111
    # (the quantizers never meet one: their inputs are finite)
    enc = oracle.e4m3_encode(np.array([np.nan, -np.nan], np.float32))
    assert all(int(c) & 0x7F == 0x7F for c in enc)


def test_hand_worked_rounding():
    g = load("p8_e4m3_values.txt")
    v = np.array([float(x) for x in g["ties_in"]], np.float32)
    np.testing.assert_array_equal(oracle.e4m3_encode(v), np.array([int(c) for c in g["ties_out"]], np.uint8))


def test_code_order_and_round_trip():
    vals = oracle.e4m3_decode(CODES)
    pos = vals[:0x7F].astype(np.float64)          # 0x00..0x7E
    assert np.all(np.diff(pos) > 0)
    np.testing.assert_array_equal(vals[0x80:0xFF], -vals[:0x7F])
    c, v = _finite_table()
    np.testing.assert_array_equal(oracle.e4m3_encode(v.astype(np.float32)), c)


def test_encoder_is_the_nearest_value_brute_force():
    c, v = _finite_table()
    rng = np.random.default_rng(31)
    x = np.concatenate([
        rng.uniform(-600, 600, 3000),
        np.sign(rng.standard_normal(3000)) * np.exp2(rng.uniform(-12, 9.5, 3000)),
        (v[1:] + v[:-1]) / 2,                                 # every midpoint (ties)
    ]).astype(np.float32)
    x = x[~np.isnan(x)]
    got = oracle.e4m3_encode(x)
    xd = x.astype(np.float64)
    for xi, gi in zip(xd, got):
        if abs(xi) >= 448:
            assert gi == (0xFE if xi < 0 else 0x7E)
            continue
        d = np.abs(v - xi)
        best = np.flatnonzero(d == d.min())
        cand = c[best]
        if len(cand) > 1:                                     # a tie: the even code (+-0 when at zero)
            cand = [k for k in cand if k % 2 == 0 and (np.signbit(xi) == bool(k & 0x80) or (k & 0x7F))]
        assert gi in cand, (xi, gi, cand)


def test_exact_product_against_library_float64():
    rng = np.random.default_rng(32)
    c, _ = _finite_table()
    xq = rng.choice(c, (5, 96)).astype(np.uint8)
    wq = rng.choice(c, (7, 96)).astype(np.uint8)
    acc = oracle.gemm_e4m3(xq, wq)
    ref = oracle.e4m3_decode(xq).astype(np.float64) @ oracle.e4m3_decode(wq).astype(np.float64).T
    np.testing.assert_array_equal(acc, ref)
    # the extreme: 448 * 448 * 32768 is exact
    big = np.full((1, 32768), 0x7E, np.uint8)
    assert oracle.gemm_e4m3(big, big)[0, 0] == 448.0 * 448.0 * 32768


@pytest.mark.parametrize("layout", [0, 1])
def test_row_maps_to_448_and_identity_within_bound(layout):
    rng = np.random.default_rng(33 + layout)
    M, K, N = 6, 64, 9
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[:, 5] *= 60
    w = (rng.standard_normal((K, N)) * 0.05).astype(np.float32)
    w_l = w if layout == 0 else np.ascontiguousarray(w.T)
    s, inv = oracle.smooth_factor(oracle.calib_absmax(x), oracle.weight_absmax(w_l, layout), 0.5)
    wq, dw = oracle.smooth_quant_weight_e4m3(w_l, layout, s)
    xq, dx = oracle.quant_act_e4m3(x, inv)
    # each token's and each output channel's largest magnitude maps to +-448
    assert np.all(np.abs(oracle.e4m3_decode(xq)).max(axis=1) == 448)
    assert np.all(np.abs(oracle.e4m3_decode(wq)).max(axis=1) == 448)
    xt = (x * inv).astype(np.float64)
    wt = (s[:, None] * w).astype(np.float64)                 # [K, N]
    # E4M3 keeps 3 mantissa bits: relative error <= 2^-4 for normals, and
    # an absolute 2^-10 code unit below 2^-6
    ex = np.abs(xt) * 2.0 ** -4 + 2.0 ** -10 * dx[:, None]
    ew = np.abs(wt) * 2.0 ** -4 + 2.0 ** -10 * dw[None, :]
    bound = np.abs(xt) @ ew + ex @ np.abs(wt) + ex @ ew
    y = oracle.dequant_f32acc(oracle.gemm_e4m3(xq, wq).astype(np.float32), dx, dw).astype(np.float64)
    exact = x.astype(np.float64) @ w.astype(np.float64)
    assert np.all(np.abs(y - exact) <= bound * 1.001 + 1e-6 * np.abs(exact))
