"""Pins for the CPU oracle: checks against what the SmoothQuant glossary page
(jisaku.com, "SmoothQuant (activation smoothing quantization)") and plain
mathematics fix, never against the oracle itself.

- worked examples built from the page's printed channel values ("Why
  activation quantization is hard"), worked by hand (tests/golden/);
- the smoothing identity Y = (X diag(s)^-1)(diag(s) W) ("The mathematics of
  the smoothing transformation") to fp32 rounding;
- closed-form invariants of s_j = max|X_j|^a / max|W_j|^(1-a) ("Hyper-
  parameter alpha") including the alpha = 0 and alpha = 1 limits;
- the defining property of round-to-nearest quantization on a uniform grid;
- brute-force integer matrix products and library reductions/conversions.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from tests.golden.load import load

KN, NK = oracle.LAYOUT_KN, oracle.LAYOUT_NK
F32_EPS = float(np.finfo(np.float32).eps)  # 2^-23


def _fl(rows):
    if rows and isinstance(rows[0], list):
        return np.array([[float(v) for v in r] for r in rows], np.float64)
    return np.array([float(v) for v in rows], np.float64)


def _int(rows):
    if rows and isinstance(rows[0], list):
        return np.array([[int(v) for v in r] for r in rows], np.int64)
    return np.array([int(v) for v in rows], np.int64)


def _ulps(got, exact):
    """Distance of fp32 'got' from the exact value, in fp32 ulps of exact."""
    got = np.asarray(got, np.float64)
    exact = np.asarray(exact, np.float64)
    ulp = np.spacing(np.abs(exact).astype(np.float32)).astype(np.float64)
    return np.abs(got - exact) / ulp


# ---------------------------------------------------------------------------
# worked examples (tests/golden)
# ---------------------------------------------------------------------------

def test_p5_page_channels_worked_example():
    g = load("p5_outlier_channel_example.txt")
    x = _fl(g["x"]).astype(np.float32)
    w = _fl(g["w_kn"]).astype(np.float32)
    alpha = float(g["alpha"][0])
    r = oracle.pipeline([x], w, KN, alpha, x, "f32")

    # channel maxima are exact selections of input values
    np.testing.assert_array_equal(r["amax"], _fl(g["a"]).astype(np.float32))
    np.testing.assert_array_equal(r["wmax"], _fl(g["wmax"]).astype(np.float32))
    # s from three IEEE-rounded operations on rounded inputs: a few ulps
    assert _ulps(r["s"], _fl(g["s"])).max() <= 4
    smoothed_x_max = r["amax"].astype(np.float64) * r["inv_s"]
    assert _ulps(smoothed_x_max, _fl(g["smoothed_channel_max"])).max() <= 8
    assert _ulps(r["dw"], _fl(g["dw"])).max() <= 8
    assert _ulps(r["dx"], _fl(g["dx"])).max() <= 8
    # integer codes and accumulators: exact
    np.testing.assert_array_equal(r["wq"], _int(g["wq_nk"]))
    np.testing.assert_array_equal(r["xq"], _int(g["xq"]))
    np.testing.assert_array_equal(r["acc"], _int(g["acc"]))
    # without smoothing (s = 1) the normal channel collapses as the page says
    xq0, _ = oracle.quant_act(x, np.ones(2, np.float32))
    np.testing.assert_array_equal(xq0, _int(g["xq_unsmoothed"]))

    # Y against the exact product, within the rounding-error bound of
    # quantizing both smoothed operands to their grids
    y_exact = _fl(g["y_exact"])
    xt = x.astype(np.float64) / _fl(g["s"])[None, :]
    wt = _fl(g["s"])[:, None] * w.astype(np.float64)
    dx = _fl(g["dx"])
    dw = _fl(g["dw"])
    bound = (np.abs(xt) @ np.ones_like(wt)) * dw[None, :] / 2 \
        + dx[:, None] * (np.ones_like(xt) @ np.abs(wt)) / 2 \
        + dx[:, None] * dw[None, :] * x.shape[1] / 4
    assert np.all(np.abs(r["y"] - y_exact) <= bound * 1.001 + 1e-6)


def test_p4_round_half_to_even_ties():
    g = load("p4_rne_ties.txt")
    x = _fl(g["x"]).astype(np.float32)[None, :]
    xq, dx = oracle.quant_act(x, np.ones(x.shape[1], np.float32))
    np.testing.assert_array_equal(xq[0], _int(g["xq"]))
    assert dx[0] == np.float32(float(g["dx"][0]))


def test_p6_outlier_x100_spread_and_codes():
    g = load("p6_outlier_x100.txt")
    x = _fl(g["x"]).astype(np.float32)
    w = _fl(g["w_kn"]).astype(np.float32)
    r = oracle.pipeline([x], w, KN, float(g["alpha"][0]), x, "f32")
    np.testing.assert_array_equal(r["amax"], _fl(g["a"]).astype(np.float32))
    np.testing.assert_array_equal(r["wmax"], _fl(g["wmax"]).astype(np.float32))
    smoothed = r["amax"].astype(np.float64) * r["inv_s"]
    assert _ulps(smoothed, _fl(g["smoothed_channel_max"])).max() <= 8
    # the outlier channel's spread drops from 100x to 10x
    assert abs(smoothed[3] / smoothed[0] - 10.0) < 1e-5
    np.testing.assert_array_equal(r["xq"][0], _int(g["xq_token0"]))
    xq0, _ = oracle.quant_act(x, np.ones(4, np.float32))
    np.testing.assert_array_equal(xq0[0], _int(g["xq_token0_unsmoothed"]))
    # every non-outlier code of an outlier token collapses to |q| <= 1
    assert np.abs(xq0[0, :3]).max() <= 1


# ---------------------------------------------------------------------------
# smoothing identity and alpha invariants
# ---------------------------------------------------------------------------

ALPHAS = [0.0, 0.25, 0.5, 0.75, 1.0, 0.3, 0.85]


@pytest.mark.parametrize("alpha", ALPHAS)
@pytest.mark.parametrize("layout", [KN, NK])
def test_p1_smoothing_identity(alpha, layout):
    rng = np.random.default_rng(11)
    x = rng.standard_normal((4, 8)).astype(np.float32)
    x[:, 3] *= 100.0
    w_kn = (rng.standard_normal((8, 3)) * 0.02).astype(np.float32)
    w = w_kn if layout == KN else np.ascontiguousarray(w_kn.T)
    amax = oracle.calib_absmax(x)
    wmax = oracle.weight_absmax(w, layout)
    s, inv_s = oracle.smooth_factor(amax, wmax, alpha)
    xt = oracle.smooth_act(x, inv_s).astype(np.float64)
    wt = oracle.smooth_weight(w, layout, s).astype(np.float64)
    wt_kn = wt if layout == KN else wt.T
    y = x.astype(np.float64) @ w_kn.astype(np.float64)
    yt = xt @ wt_kn
    # three fp32 roundings per term (1/s, x*inv_s, s*w) -> <= ~4 ulp per term
    bound = 4 * F32_EPS * (np.abs(x).astype(np.float64) @ np.abs(w_kn).astype(np.float64))
    assert np.all(np.abs(y - yt) <= bound + 1e-30)
    # and a mistaken axis would break it by O(1): guard the bound is tight
    assert bound.max() < 1e-4 * np.abs(y).max() + 1e-30


@pytest.mark.parametrize("alpha", ALPHAS)
def test_p2_alpha_invariants(alpha):
    rng = np.random.default_rng(5)
    K = 257
    a = np.exp(rng.uniform(-3, 5, K)).astype(np.float32)
    w = np.exp(rng.uniform(-6, 0, K)).astype(np.float32)
    s, inv_s = oracle.smooth_factor(a, w, alpha)
    a64, w64 = a.astype(np.float64), w.astype(np.float64)
    xmax = a64 * inv_s.astype(np.float64)  # max|X~_j|
    wmax_t = s.astype(np.float64) * w64     # max|W~_j|
    # product of the two smoothed maxima is invariant for every alpha
    np.testing.assert_allclose(xmax * wmax_t, a64 * w64, rtol=8 * F32_EPS)
    # s against the formula evaluated in fp64 at the fp32 value of alpha
    a32 = float(np.float32(alpha))
    s_exact = a64 ** a32 / w64 ** (1 - a32)
    assert _ulps(s, s_exact).max() <= (1 if alpha not in (0.25, 0.5, 0.75) else 4)
    if alpha == 1.0:    # all difficulty moved to W: activations max to 1
        np.testing.assert_allclose(xmax, 1.0, rtol=2 * F32_EPS)
    if alpha == 0.0:    # all difficulty kept on X: weights max to 1
        np.testing.assert_allclose(wmax_t, 1.0, rtol=2 * F32_EPS)
    if alpha == 0.5:    # even split: both equal sqrt(a w)
        np.testing.assert_allclose(xmax, np.sqrt(a64 * w64), rtol=6 * F32_EPS)
        np.testing.assert_allclose(wmax_t, np.sqrt(a64 * w64), rtol=6 * F32_EPS)
    np.testing.assert_array_equal(inv_s, (np.float32(1) / s).astype(np.float32))


def test_smooth_factor_floor_on_empty_channels():
    a = np.array([0.0, 3.0, 0.0], np.float32)
    w = np.array([0.2, 0.0, 0.0], np.float32)
    s, inv_s = oracle.smooth_factor(a, w, 0.5)
    assert np.all(np.isfinite(s)) and np.all(np.isfinite(inv_s)) and np.all(s > 0)
    np.testing.assert_allclose(s, np.sqrt([1e-5 / 0.2, 3.0 / 1e-5, 1.0]), rtol=1e-6)


def _alternative_sequences(alpha, a, w):
    """Other plausible fp32 evaluations of a^alpha / w^(1-alpha) (numpy fp32:
    IEEE-correct sqrt, product and division)."""
    f = np.float32
    sq = lambda v: f(np.sqrt(f(v)))  # noqa: E731
    once = f(np.float64(a) ** alpha / np.float64(w) ** (1.0 - alpha))
    if alpha == 0.5:
        return [sq(f(a / w)), f(sq(a) * f(f(1) / sq(w))), once]
    if alpha == 0.25:
        w3 = f(f(w * w) * w)
        return [sq(sq(f(a / w3))), f(sq(sq(a)) / sq(sq(w3))), f(sq(sq(a)) / sq(f(w * sq(w)))), once]
    a3 = f(f(a * a) * a)
    return [sq(sq(f(a3 / w))), f(sq(sq(a3)) / sq(sq(w))), once]


def _reciprocal_formula(alpha, a, w):
    """inv_s as w^(1-alpha) / a^alpha by the mirrored sqrt sequence, in place of 1/s."""
    f = np.float32
    sq = lambda v: f(np.sqrt(f(v)))  # noqa: E731
    if alpha == 0.5:
        return f(sq(w) / sq(a))
    if alpha == 0.25:
        return f(f(sq(w) * sq(sq(w))) / sq(sq(a)))
    return f(sq(sq(w)) / f(sq(a) * sq(sq(a))))


def test_p12_smooth_factor_fp32_sequence():
    """s and 1/s bit for bit against the hand-derived table
    (tests/golden/p12_smooth_factor_sequences.txt: the reading's sequence of
    square roots, one product and one division, worked in exact rationals).
    Each case also shows that the alternative sequences give a different
    float, so an oracle that evaluated the power another way fails here.
    (inv_s computed in double and rounded to fp32 is not a distinct
    alternative: double rounding of a quotient of fp32 values is innocuous,
    53 >= 2*24 + 2, so it equals the fp32 division on every input.)"""
    g = load("p12_smooth_factor_sequences.txt")
    assert len(g) == 11
    for key in sorted(g):
        alpha, ah, wh, sh, ih = g[key]
        alpha = float(alpha)
        a, w = np.float32(float.fromhex(ah)), np.float32(float.fromhex(wh))
        s, inv = oracle.smooth_factor(np.array([a]), np.array([w]), alpha)
        assert s[0] == np.float32(float.fromhex(sh)), key
        assert inv[0] == np.float32(float.fromhex(ih)), key
        if alpha in (0.25, 0.5, 0.75):
            for alt in _alternative_sequences(alpha, a, w):
                assert alt != s[0], key
            assert _reciprocal_formula(alpha, a, w) != inv[0], key


# ---------------------------------------------------------------------------
# reductions against library routines
# ---------------------------------------------------------------------------

def test_calib_absmax_matches_library_and_is_running():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((300, 96)).astype(np.float32)
    x[:, 7] *= -100
    full = oracle.calib_absmax(x)
    np.testing.assert_array_equal(full, np.abs(x).max(axis=0))
    run = oracle.calib_absmax(x[:100])
    run = oracle.calib_absmax(x[100:250], run)
    run = oracle.calib_absmax(x[250:], run)
    np.testing.assert_array_equal(run, full)


def test_weight_absmax_both_layouts():
    rng = np.random.default_rng(2)
    w_kn = rng.standard_normal((40, 24)).astype(np.float32)
    np.testing.assert_array_equal(oracle.weight_absmax(w_kn, KN), np.abs(w_kn).max(axis=1))
    np.testing.assert_array_equal(oracle.weight_absmax(np.ascontiguousarray(w_kn.T), NK),
                                  np.abs(w_kn).max(axis=1))


# ---------------------------------------------------------------------------
# quantizers: defining property of rounding to a uniform symmetric grid
# ---------------------------------------------------------------------------

def _fp32_round(q):
    """A rational rounded to the nearest fp32 value (ties to even)."""
    from fractions import Fraction
    if q == 0:
        return Fraction(0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    ulp = Fraction(2) ** (e - 23)
    n, r = divmod(a, ulp)
    if r > ulp / 2 or (r == ulp / 2 and n % 2 == 1):
        n += 1
    return sign * n * ulp


def _rne_int(q):
    from fractions import Fraction
    n = q.numerator // q.denominator
    r = q - n
    if r > Fraction(1, 2) or (r == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return n


@pytest.mark.parametrize("v,delta", [(-22.80670928955078, 0.5366284251213074), (-8.67187786102295, 0.4955359101295471),
                                     (-31.285537719726562, 0.3935287892818451),
                                     (-50.01250457763672, 0.5989521741867065)])
def test_quantizer_divides_by_the_scale(v, delta):
    # The reading: q = rne(fl(v / delta)) with an IEEE division.  These
    # inputs put v / delta within an ulp of a half-integer, where a multiply
    # by the rounded reciprocal 1/delta lands on the other side; the expected
    # code is worked in exact rational arithmetic.
    from fractions import Fraction
    v32, d32 = np.float32(v), np.float32(delta)
    expected = _rne_int(_fp32_round(Fraction(float(v32)) / Fraction(float(d32))))
    assert oracle.quantize_value(float(v32), float(d32)) == expected
    via_reciprocal = int(np.rint(np.float32(v32 * np.float32(np.float32(1.0) / d32))))
    assert via_reciprocal != expected


def test_quantize_value_saturation_and_ties():
    assert oracle.quantize_value(200.0, 1.0) == 127
    assert oracle.quantize_value(-200.0, 1.0) == -127
    assert oracle.quantize_value(-128.0, 1.0) == -127
    assert oracle.quantize_value(126.5, 1.0) == 126
    assert oracle.quantize_value(-125.5, 1.0) == -126
    assert oracle.quantize_value(0.49999997, 1.0) == 0


def test_quant_act_grid_property_and_zero_rows():
    rng = np.random.default_rng(3)
    M, K = 37, 160
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[:, [3, 77]] *= 100
    x[5] = 0.0
    inv_s = np.exp(rng.uniform(-2, 2, K)).astype(np.float32)
    xq, dx = oracle.quant_act(x, inv_s)
    xt = x.astype(np.float64) * inv_s.astype(np.float64)
    for t in range(M):
        if t == 5:
            assert dx[t] == 0 and not xq[t].any()
            continue
        assert np.abs(xq[t]).max() == 127       # per-token: each row reaches 127
        err = np.abs(xt[t] - xq[t].astype(np.float64) * dx[t])
        assert err.max() <= dx[t] * 0.5 * (1 + 1e-5) + 1e-12
        np.testing.assert_allclose(dx[t], np.abs(xt[t]).max() / 127, rtol=4 * F32_EPS)


@pytest.mark.parametrize("layout", [KN, NK])
def test_weight_quant_grid_property_per_output_channel(layout):
    rng = np.random.default_rng(4)
    K, N = 96, 48
    w_kn = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
    w_kn[:, 9] = 0.0
    w = w_kn if layout == KN else np.ascontiguousarray(w_kn.T)
    s = np.exp(rng.uniform(-2, 2, K)).astype(np.float32)
    wq, dw = oracle.smooth_quant_weight(w, layout, s)
    assert wq.shape == (N, K)
    wt = s.astype(np.float64)[:, None] * w_kn.astype(np.float64)  # [K, N]
    for n in range(N):
        if n == 9:
            assert dw[n] == 0 and not wq[n].any()
            continue
        assert np.abs(wq[n]).max() == 127
        err = np.abs(wt[:, n] - wq[n].astype(np.float64) * dw[n])
        assert err.max() <= dw[n] * 0.5 * (1 + 1e-5) + 1e-12
    # both layouts give the same codes
    other = np.ascontiguousarray(w.T)
    wq2, dw2 = oracle.smooth_quant_weight(other, NK if layout == KN else KN, s)
    np.testing.assert_array_equal(wq, wq2)
    np.testing.assert_array_equal(dw, dw2)


# ---------------------------------------------------------------------------
# integer product and epilogue
# ---------------------------------------------------------------------------

def test_p3_gemm_brute_force_small():
    rng = np.random.default_rng(6)
    M, N, K = 3, 4, 5
    xq = rng.integers(-127, 128, (M, K), dtype=np.int8)
    wq = rng.integers(-127, 128, (N, K), dtype=np.int8)
    acc = oracle.gemm_i8(xq, wq)
    for t in range(M):
        for n in range(N):
            assert acc[t, n] == sum(int(xq[t, j]) * int(wq[n, j]) for j in range(K))


def test_p3_gemm_against_int64_matmul_and_extremes():
    rng = np.random.default_rng(7)
    M, N, K = 33, 40, 272
    xq = rng.integers(-127, 128, (M, K), dtype=np.int8)
    wq = rng.integers(-127, 128, (N, K), dtype=np.int8)
    np.testing.assert_array_equal(oracle.gemm_i8(xq, wq), xq.astype(np.int64) @ wq.astype(np.int64).T)
    K = 28672  # largest K in the workloads: 127*127*K still fits in int32
    xe = np.full((2, K), 127, np.int8)
    xe[1] = -127
    we = np.full((1, K), 127, np.int8)
    np.testing.assert_array_equal(oracle.gemm_i8(xe, we)[:, 0], [127 * 127 * K, -127 * 127 * K])


def test_dequant_exact_on_power_of_two_scales():
    acc = np.array([[1, -2, 3], [40000, -7, 0]], np.int32)
    dx = np.array([0.5, 2.0 ** -10], np.float32)
    dw = np.array([4.0, 2.0 ** -3, 1.0], np.float32)
    y = oracle.dequant(acc, dx, dw)
    np.testing.assert_array_equal(y, acc.astype(np.float64) * dx[:, None] * dw[None, :])


# (acc, dx, dw) triples where the three ways of forming acc * dx * dw in fp32
# give three different floats: ((float)acc * dx) * dw (the reading),
# (float)acc * (dx * dw), and the exact product rounded once (an fma or a
# double-precision product).  Found by a random search over the configs'
# scale ranges; the expected values are worked below in exact rationals.
DEQUANT_ORDER_CASES = [
    (205907, 0.0008812682353891432, 0.019935712218284607),
    (58144, 0.004028223920613527, 0.015843471512198448),
    (-219780, 0.004683542996644974, 0.000896687270142138),
    (-46418, 0.0029101360123604536, 0.013552580028772354),
]


def test_dequant_order_of_rounding():
    """y = ((float)acc * dx) * dw: each product rounded to fp32 in that order
    (the reading of the epilogue; the page states only Y = X~ W~).  The
    expected values are worked in exact rational arithmetic with explicit
    round-to-nearest-even, and the test checks that the other groupings give
    a different float on every case, so a re-grouped oracle fails here."""
    # (float)acc rounds to nearest even beyond 2^24
    for acc, want in ((16777217, 16777216.0), (16777219, 16777220.0), (-16777221, -16777220.0)):
        y = oracle.dequant(np.array([[acc]], np.int32), np.ones(1, np.float32), np.ones(1, np.float32))
        assert y[0, 0] == np.float32(want)
    for acc, dx, dw in DEQUANT_ORDER_CASES:
        dx32, dw32 = np.float32(dx), np.float32(dw)
        A, DX, DW = _fp32_round(Fraction(acc)), Fraction(float(dx32)), Fraction(float(dw32))
        reading = _fp32_round(_fp32_round(A * DX) * DW)
        regrouped = _fp32_round(A * _fp32_round(DX * DW))
        once = _fp32_round(Fraction(acc) * DX * DW)
        assert len({reading, regrouped, once}) == 3
        y = oracle.dequant(np.array([[acc]], np.int32), np.array([dx32]), np.array([dw32]))
        assert Fraction(float(y[0, 0])) == reading
    # the same cases as one [M, N] call: row t takes dx[t], column n takes dw[n]
    accs = np.array([[c[0] for c in DEQUANT_ORDER_CASES]], np.int32).repeat(2, 0)
    dxs = np.array([DEQUANT_ORDER_CASES[0][1], 1.0], np.float32)
    dws = np.array([c[2] for c in DEQUANT_ORDER_CASES], np.float32)
    y = oracle.dequant(accs, dxs, dws)
    for t in range(2):
        for n in range(len(DEQUANT_ORDER_CASES)):
            want = _fp32_round(_fp32_round(_fp32_round(Fraction(int(accs[t, n]))) * Fraction(float(dxs[t])))
                               * Fraction(float(dws[n])))
            assert Fraction(float(y[t, n])) == want


def test_output_rounding_matches_library_conversions():
    rng = np.random.default_rng(8)
    y = (rng.standard_normal(4000) * np.exp(rng.uniform(-20, 20, 4000))).astype(np.float32)
    # exact ties for bf16 (low 16 bits = 0x8000) and for f16
    ties = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8),
                     1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, 65504.0, 1e-8], np.float32)
    y = np.concatenate([y, ties])
    bf = oracle.round_to(y, "bf16")
    ref_bf = torch.from_numpy(y).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(bf, ref_bf)
    h = oracle.round_to(y, "f16")
    with np.errstate(over="ignore"):  # values beyond the f16 range round to infinity on both sides
        h_ref = y.astype(np.float16).view(np.uint16)
    np.testing.assert_array_equal(h, h_ref)


# ---------------------------------------------------------------------------
# upstream producer: RMSNorm folded with X diag(s)^-1, and the static scale
# ---------------------------------------------------------------------------

def test_p11_rmsnorm_worked_example():
    g = load("p11_rmsnorm.txt")
    x = _fl(g["x"]).astype(np.float32)[None, :]
    eps = float(g["eps"][0])
    r = oracle.rmsnorm_factor(x, eps)
    assert r[0] == np.float32(1.0 / float(g["r_inv"][0]))
    for case in ("a", "b"):
        gs = _fl(g["gs_" + case]).astype(np.float32)
        xq, dx = oracle.rmsnorm_quant_act(x, gs, eps)
        np.testing.assert_array_equal(xq[0], _int(g["xq_" + case]))
        v = ((x[0] * r[0]).astype(np.float32) * gs).astype(np.float32)
        assert dx[0] == np.float32(np.abs(v).max() / np.float32(127))


def test_rmsnorm_factor_matches_library_rms_norm():
    rng = np.random.default_rng(21)
    x = rng.standard_normal((9, 320)).astype(np.float32)
    x[:, 5] *= 80
    eps = 1e-5
    r = oracle.rmsnorm_factor(x, eps)
    xt = torch.from_numpy(x.astype(np.float64))
    normed = torch.nn.functional.rms_norm(xt, (320,), eps=eps)  # x / sqrt(mean(x^2) + eps)
    r_lib = (normed / xt)[:, 0].numpy()
    assert _ulps(r, r_lib).max() <= 1


@pytest.mark.parametrize("dt", [np.float32, np.float16])
def test_rmsnorm_quant_power_of_two_identity(dt):
    # rows with mean(x^2) = 4 exactly (and eps = 0) have r = 1/2 exactly, so
    # (x r) gs = (x gs) / 2 with no extra rounding: the codes equal plain
    # per-token quantization of x with column scales gs, and the scale
    # halves.  This fixes that gs acts per column and r per row.
    rng = np.random.default_rng(22)
    base = np.array([7, 3, 1, 1, 1, 1, 1, 1] + [0] * 8, np.float32)  # sum of squares 64, K = 16
    rows = []
    for _ in range(6):
        rows.append(base[rng.permutation(16)] * rng.choice([-1.0, 1.0], 16).astype(np.float32))
    x = np.stack(rows).astype(dt).astype(np.float32)
    gamma = np.exp(rng.uniform(-1, 1, 16)).astype(np.float32)
    inv_s = np.exp(rng.uniform(-2, 2, 16)).astype(np.float32)
    gs = oracle.fold_norm_weight(gamma, inv_s)
    np.testing.assert_array_equal(oracle.rmsnorm_factor(x, 0.0), 0.5)
    xq, dx = oracle.rmsnorm_quant_act(x, gs, 0.0)
    xq_plain, dx_plain = oracle.quant_act(x, gs)
    np.testing.assert_array_equal(xq, xq_plain)
    np.testing.assert_array_equal(dx, dx_plain * np.float32(0.5))


def test_folded_norm_equals_norm_then_smoothing():
    # with inv_s a power of two per channel, folding it into the norm weight
    # changes no rounding: ((x r) gamma) inv_s == (x r)(gamma inv_s) exactly.
    # So the folded producer must equal the unfolded sequence -- normalise,
    # apply gamma, then X diag(s)^-1 and per-token quantization.  A fold that
    # used s instead of 1/s, or dropped gamma, fails here.
    rng = np.random.default_rng(24)
    K = 64
    x = rng.standard_normal((7, K)).astype(np.float32)
    x[:, 3] *= 40
    gamma = rng.uniform(0.2, 3.0, K).astype(np.float32)
    inv_s = np.float32(2.0) ** rng.integers(-6, 7, K).astype(np.float32)
    eps = 1e-5
    gs = oracle.fold_norm_weight(gamma, inv_s)
    xq, dx = oracle.rmsnorm_quant_act(x, gs, eps)
    r = oracle.rmsnorm_factor(x, eps)
    normed = ((x * r[:, None]).astype(np.float32) * gamma).astype(np.float32)
    xq_u, dx_u = oracle.quant_act(normed, inv_s)
    np.testing.assert_array_equal(xq, xq_u)
    np.testing.assert_array_equal(dx, dx_u)
    assert not np.array_equal(xq, oracle.rmsnorm_quant_act(x, oracle.fold_norm_weight(gamma, 1 / inv_s), eps)[0])


def test_fold_is_one_fp32_product():
    """gs_j = fl(gamma_j * inv_s_j): the fold multiplies the stored
    reciprocal, as diag(s)^-1 is applied to X (a single fp32 product, worked
    here in exact rationals).  On these inputs dividing by s, or by the
    re-inverted 1/inv_s, gives a different float for some channel."""
    rng = np.random.default_rng(31)
    gamma = rng.uniform(0.2, 3.0, 256).astype(np.float32)
    inv_s = np.exp(rng.uniform(-4, 4, 256)).astype(np.float32)
    s = (np.float32(1) / inv_s).astype(np.float32)
    gs = oracle.fold_norm_weight(gamma, inv_s)
    for j in range(256):
        assert Fraction(float(gs[j])) == _fp32_round(Fraction(float(gamma[j])) * Fraction(float(inv_s[j])))
    assert np.any((gamma / s).astype(np.float32) != gs)
    assert np.any((gamma / (np.float32(1) / inv_s)).astype(np.float32) != gs)


def test_rmsnorm_quant_scale_invariance():
    # per-token quantization after RMSNorm ignores a power-of-two rescaling
    # of the token (eps = 0): r absorbs it exactly
    rng = np.random.default_rng(23)
    x = rng.standard_normal((5, 96)).astype(np.float32)
    gs = oracle.fold_norm_weight(rng.uniform(0.5, 2, 96), rng.uniform(0.1, 3, 96))
    a = oracle.rmsnorm_quant_act(x, gs, 0.0)
    b = oracle.rmsnorm_quant_act(x * np.float32(8.0), gs, 0.0)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_p7_static_scale_and_saturation():
    g = load("p7_static_scale.txt")
    delta = oracle.static_act_scale(_fl(g["amax"]), _fl(g["inv_s_scale"]))
    assert delta == np.float32(np.float32(float(g["delta_num"][0])) / np.float32(127))
    x = _fl(g["x"]).astype(np.float32)[None, :]
    xq, dx = oracle.quant_act_static(x, np.ones(x.shape[1], np.float32), float(g["delta"][0]))
    np.testing.assert_array_equal(xq[0], _int(g["xq"]))
    assert dx[0] == np.float32(float(g["delta"][0]))


# ---------------------------------------------------------------------------
# upstream producer: LayerNorm (weight and bias) folded with X diag(s)^-1
# ---------------------------------------------------------------------------

def test_p10_layernorm_worked_example():
    g = load("p10_layernorm.txt")
    x = _fl(g["x"]).astype(np.float32)[None, :]
    eps = float(g["eps"][0])
    mu, r = oracle.layernorm_stats(x, eps)
    assert mu[0] == float(g["mu"][0]) and r[0] == float(g["r"][0])
    ones = np.ones(4, np.float32)
    for case, gs, bs in (("a", _fl(g["gs_a"]), None), ("b", _fl(g["gs_b"]), None),
                         ("c", ones, _fl(g["bs_c"]))):
        xq, dx = oracle.layernorm_quant_act(x, gs, bs, eps)
        np.testing.assert_array_equal(xq[0], _int(g["xq_" + case]))
        assert dx[0] == np.float32(np.float32(float(g["dx_%s_num" % case][0])) / np.float32(127))


def test_layernorm_stats_match_library_layer_norm():
    rng = np.random.default_rng(31)
    x = (rng.standard_normal((9, 320)) + rng.uniform(-3, 3, (9, 1))).astype(np.float32)
    x[:, 5] *= 80
    eps = 1e-5
    mu, r = oracle.layernorm_stats(x, eps)
    xt = torch.from_numpy(x.astype(np.float64))
    normed = torch.nn.functional.layer_norm(xt, (320,), eps=eps).numpy()  # (x - mean) / sqrt(var + eps)
    mean = xt.mean(dim=1).numpy()
    assert _ulps(mu, mean).max() <= 0.5
    j = np.argmax(np.abs(x - mean[:, None]), axis=1)  # the largest deviation in each row
    rows = np.arange(9)
    r_lib = normed[rows, j] / (x[rows, j].astype(np.float64) - mean)
    assert _ulps(r, r_lib).max() <= 1


def test_layernorm_on_zero_mean_rows_equals_rmsnorm():
    # rows made of +-pairs have mean exactly 0, so the variance is the mean
    # square: LayerNorm without bias must give the RMSNorm producer's codes
    # and scales bit for bit.  A 1/(K-1) variance or a mean taken of |x|
    # fails here.
    rng = np.random.default_rng(32)
    half = (rng.standard_normal((6, 48)) * 3).astype(np.float32)
    x = np.concatenate([half, -half], axis=1)[:, rng.permutation(96)]
    gs = oracle.fold_norm_weight(rng.uniform(0.3, 2, 96), rng.uniform(0.1, 3, 96))
    eps = 1e-5
    mu, _ = oracle.layernorm_stats(x, eps)
    np.testing.assert_array_equal(mu, 0.0)
    a = oracle.layernorm_quant_act(x, gs, None, eps)
    b = oracle.rmsnorm_quant_act(x, gs, eps)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_layernorm_shift_and_scale_invariance():
    # values on a 1/8 grid, K = 16: the mean is exact, and so is every
    # deviation, with or without a shift of the whole token by a constant,
    # so the codes cannot change.  A power-of-two rescale with negligible
    # eps is absorbed exactly by r.  A producer that skips the mean (RMS of
    # the raw values) fails the shift.
    rng = np.random.default_rng(33)
    x = (rng.integers(-40, 41, (7, 16)) / 8.0).astype(np.float32)
    gs = oracle.fold_norm_weight(rng.uniform(0.5, 2, 16), rng.uniform(0.2, 3, 16))
    bs = rng.uniform(-0.5, 0.5, 16).astype(np.float32)
    eps = 1e-30
    base = oracle.layernorm_quant_act(x, gs, bs, eps)
    shifted = oracle.layernorm_quant_act(x + np.float32(37.0), gs, bs, eps)
    scaled = oracle.layernorm_quant_act(x * np.float32(16.0), gs, bs, eps)
    for other in (shifted, scaled):
        np.testing.assert_array_equal(base[0], other[0])
        np.testing.assert_array_equal(base[1], other[1])
    assert not np.array_equal(base[0], oracle.rmsnorm_quant_act(x + np.float32(37.0), gs, eps)[0])


def test_layernorm_values_are_what_is_quantized():
    # the exposed values v (used by the GPU tests to find rounding
    # boundaries) quantize per token to the producer's own codes and scales
    rng = np.random.default_rng(35)
    x = (rng.standard_normal((6, 48)) + 0.5).astype(np.float32)
    gs = rng.uniform(0.2, 3.0, 48).astype(np.float32)
    bs = rng.uniform(-1, 1, 48).astype(np.float32)
    for b in (bs, None):
        v = oracle.layernorm_values(x, gs, b, 1e-5)
        xq, dx = oracle.layernorm_quant_act(x, gs, b, 1e-5)
        vq, vd = oracle.quant_act(v, np.ones(48, np.float32))
        np.testing.assert_array_equal(xq, vq)
        np.testing.assert_array_equal(dx, vd)


def test_layernorm_bias_alone():
    # with gs = 0 every token normalises to v = bs, whatever x is: the codes
    # are plain quantization of the bias row (its sign and per-column place
    # fixed by quant_act's own pins)
    rng = np.random.default_rng(34)
    x = rng.standard_normal((4, 32)).astype(np.float32)
    bs = rng.uniform(-2, 2, 32).astype(np.float32)
    xq, dx = oracle.layernorm_quant_act(x, np.zeros(32, np.float32), bs, 1e-5)
    bq, bd = oracle.quant_act(bs[None, :], np.ones(32, np.float32))
    np.testing.assert_array_equal(xq, np.repeat(bq, 4, axis=0))
    np.testing.assert_array_equal(dx, np.repeat(bd, 4))


def test_folded_layernorm_equals_norm_then_smoothing():
    # with inv_s a power of two per channel, folding it into the weight and
    # the bias changes no rounding: (n gamma + beta) inv_s == n (gamma inv_s)
    # + beta inv_s exactly.  So the folded producer must equal the unfolded
    # sequence: normalise, apply gamma and beta, then X diag(s)^-1 and
    # per-token quantization.
    rng = np.random.default_rng(35)
    K = 64
    x = (rng.standard_normal((7, K)) + 2.0).astype(np.float32)
    x[:, 3] *= 40
    gamma = rng.uniform(0.2, 3.0, K).astype(np.float32)
    beta = rng.uniform(-1.0, 1.0, K).astype(np.float32)
    inv_s = np.float32(2.0) ** rng.integers(-6, 7, K).astype(np.float32)
    eps = 1e-5
    xq, dx = oracle.layernorm_quant_act(x, oracle.fold_norm_weight(gamma, inv_s),
                                        oracle.fold_norm_weight(beta, inv_s), eps)
    mu, r = oracle.layernorm_stats(x, eps)
    n = ((x - mu[:, None]).astype(np.float32) * r[:, None]).astype(np.float32)
    # the affine step n * gamma + beta, taken exactly in rationals and
    # rounded once to fp32
    normed = np.array([[float(_fp32_round(Fraction(float(n[t, j])) * Fraction(float(gamma[j]))
                                          + Fraction(float(beta[j])))) for j in range(K)]
                       for t in range(n.shape[0])], np.float32)
    xq_u, dx_u = oracle.quant_act(normed, inv_s)
    np.testing.assert_array_equal(xq, xq_u)
    np.testing.assert_array_equal(dx, dx_u)
