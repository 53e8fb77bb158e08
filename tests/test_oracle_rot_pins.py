"""Pins for the oracle's butterfly rotation (NEXT-4), none comparing the
oracle with itself: hand-worked rotations, the Hadamard special case against
a library Walsh-Hadamard matrix, the identity at zero angles, orthogonality,
block independence, and the rotated W8A8 product within the quantization
error bound of the exact X W."""
import numpy as np
import pytest
import scipy.linalg

import oracle
from tests.golden.load import load


def _tables(n, theta):
    return np.cos(theta).astype(np.float32), np.sin(theta).astype(np.float32)


def _random_angles(n, seed):
    L = n.bit_length() - 1
    return np.random.default_rng(seed).uniform(-np.pi, np.pi, (L, n // 2))


@pytest.mark.parametrize("k", ["1", "2"])
def test_hand_worked_rotations(k):
    g = load("p9_butterfly.txt")
    x = np.array([[float(v) for v in g["x" + k]]], np.float32)
    c = np.array([[float(v) for v in r] for r in g["c" + k]], np.float32)
    s = np.array([[float(v) for v in r] for r in g["s" + k]], np.float32)
    y = np.array([float(v) for v in g["y" + k]], np.float32)
    np.testing.assert_array_equal(oracle.butterfly_rotate(x, x.shape[1], c, s)[0], y)


@pytest.mark.parametrize("n", [2, 4, 8, 32, 256])
def test_all_angles_pi_over_4_give_a_walsh_hadamard_matrix(n):
    # the section's special case: every Givens rotation at pi/4 turns the
    # butterfly into the normalised Walsh-Hadamard transform, up to the order
    # and signs of its rows.  Pairing neighbours at every stage (as the
    # page's listing does) would leave zeros in the matrix and fail here.
    L = n.bit_length() - 1
    c = np.full((L, n // 2), np.sqrt(0.5), np.float32)
    R = oracle.butterfly_rotate(np.eye(n, dtype=np.float32), n, c, c).T.astype(np.float64)  # columns: R e_k
    H = scipy.linalg.hadamard(n).astype(np.float64)
    Rs = R * np.sqrt(n)
    assert np.allclose(np.abs(Rs), 1.0, atol=4e-6 * L)
    signs = np.sign(Rs)
    rows = {tuple(h) for h in H} | {tuple(-h) for h in H}
    assert all(tuple(r) in rows for r in signs)
    assert len({int(np.abs(r @ H.T).argmax()) for r in signs}) == n  # a permutation of H's rows


def test_zero_angles_are_the_identity():
    rng = np.random.default_rng(51)
    M, K, N, n = 6, 64, 8, 16
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[:, 3] *= 50
    inv = rng.uniform(0.2, 3, K).astype(np.float32)
    L = n.bit_length() - 1
    c, s = np.ones((L, n // 2), np.float32), np.zeros((L, n // 2), np.float32)
    np.testing.assert_array_equal(oracle.butterfly_rotate(x, n, c, s), x)
    a = oracle.quant_act_rotated(x, inv, n, c, s)
    b = oracle.quant_act(x, inv)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])
    w = (rng.standard_normal((N, K)) * 0.05).astype(np.float32)
    sm = rng.uniform(0.5, 2, K).astype(np.float32)
    a = oracle.smooth_quant_weight_rotated(w, oracle.LAYOUT_NK, sm, n, c, s)
    b = oracle.smooth_quant_weight(w, oracle.LAYOUT_NK, sm)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


@pytest.mark.parametrize("n", [8, 64, 512])
def test_rotation_is_orthogonal(n):
    rng = np.random.default_rng(n)
    c, s = _tables(n, _random_angles(n, n))
    x = rng.standard_normal((5, n)).astype(np.float32)
    w = rng.standard_normal((3, n)).astype(np.float32)
    rx = oracle.butterfly_rotate(x, n, c, s).astype(np.float64)
    rw = oracle.butterfly_rotate(w, n, c, s).astype(np.float64)
    L = n.bit_length() - 1
    tol = 4 * L * 2.0 ** -24
    nx = np.linalg.norm(x.astype(np.float64), axis=1)
    assert np.all(np.abs(np.linalg.norm(rx, axis=1) - nx) <= tol * nx)
    dots = x.astype(np.float64) @ w.astype(np.float64).T
    bound = tol * 2 * np.outer(nx, np.linalg.norm(w.astype(np.float64), axis=1))
    assert np.all(np.abs(rx @ rw.T - dots) <= bound)


def test_blocks_rotate_independently():
    rng = np.random.default_rng(52)
    n, K = 16, 48
    c, s = _tables(n, _random_angles(n, 3))
    x = rng.standard_normal((2, K)).astype(np.float32)
    whole = oracle.butterfly_rotate(x, n, c, s)
    for b in range(K // n):
        np.testing.assert_array_equal(whole[:, b * n:(b + 1) * n],
                                      oracle.butterfly_rotate(x[:, b * n:(b + 1) * n], n, c, s))


@pytest.mark.parametrize("layout", [0, 1])
def test_rotated_w8a8_product_within_bound(layout):
    # (R x~) . (R w~_n) = x~ . w~_n, so the dequantized INT8 product of the
    # rotated operands approximates X W within the quantization error
    rng = np.random.default_rng(53 + layout)
    M, K, N, n = 8, 128, 12, 64
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[:, 7] *= 80
    w = (rng.standard_normal((K, N)) * 0.05).astype(np.float32)
    w_l = w if layout == 0 else np.ascontiguousarray(w.T)
    sm, inv = oracle.smooth_factor(oracle.calib_absmax(x), oracle.weight_absmax(w_l, layout), 0.5)
    c, s = _tables(n, _random_angles(n, 9))
    xq, dx = oracle.quant_act_rotated(x, inv, n, c, s)
    wq, dw = oracle.smooth_quant_weight_rotated(w_l, layout, sm, n, c, s)
    y = oracle.dequant(oracle.gemm_i8(xq, wq), dx, dw).astype(np.float64)
    xr = oracle.butterfly_rotate((x * inv).astype(np.float32), n, c, s).astype(np.float64)
    wr = oracle.butterfly_rotate((w.T * sm).astype(np.float32), n, c, s).astype(np.float64)  # [N, K]
    # per element the codes are within half a step of the rotated values
    assert np.all(np.abs(xr - xq * dx[:, None].astype(np.float64)) <= dx[:, None] * (0.5 + 1e-5))
    assert np.all(np.abs(wr - wq * dw[:, None].astype(np.float64)) <= dw[:, None] * (0.5 + 1e-5))
    bound = (np.abs(xr) @ (0.5 * dw[:, None] * np.ones((1, K))).T + (0.5 * dx[:, None]) @ np.abs(wr).sum(
        axis=1)[None, :] + 0.25 * K * np.outer(dx, dw))
    exact = x.astype(np.float64) @ w.astype(np.float64)
    assert np.all(np.abs(y - exact) <= bound * 1.01 + 1e-4 * np.abs(exact) + 1e-4)
