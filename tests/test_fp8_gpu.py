"""Parity of the FP8 (E4M3) variant against the oracle.

Codes and scales are bit-exact (the quantizers take the same fp32 decisions
as the oracle and round with the hardware E4M3 conversion, nearest-even and
saturating).  The product's fp32 accumulator is compared with the exact
double-precision sum: every product of two E4M3 values is exact, so the only
error is the fp32 addition inside the tensor cores.  Modelled as recursive
summation with one rounding of at most 2^-23 (one fp32 ulp, so truncation
is covered too) per accumulator update -- K/32 MMA instructions, up to 16
split-K partials and one more for the instruction's own sum -- the error is
below acc_bound(K) * sum_j |x_j w_j|.  Given the accumulator, the dequant
epilogue is exact: y == ((acc * dx) * dw) rounded to the output type.
"""
import numpy as np
import pytest
import torch

import oracle
import w8a8_post_quantization_channel_b200 as sq
from w8a8_post_quantization_channel_b200 import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"
TORCH_DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
LAYOUT = {"kn": sq.SQ_W_KN, "nk": sq.SQ_W_NK}
def acc_bound(K):
    """Bound on |acc - exact| / sum_j |x_j w_j| for an fp32 accumulator."""
    return (K / 32 + 17) * 2.0 ** -23


def f32(t):
    return t.detach().to("cpu", torch.float32).numpy()


def _finite_values():
    c = np.arange(256, dtype=np.uint8)
    v = oracle.e4m3_decode(c).astype(np.float64)
    return np.sort(v[~np.isnan(v)])


def test_conversion_matches_the_format_everywhere():
    # rows whose absmax is 448 quantize with multiplier fl(448/448) = 1, so
    # the codes are e4m3(x) itself: every finite value, every midpoint
    # between neighbours (ties), values beyond the subnormal range, random
    vals = _finite_values()
    mids = (vals[1:] + vals[:-1]) / 2
    rng = np.random.default_rng(41)
    pool = np.concatenate([vals, mids, rng.uniform(-448, 448, 4000),
                           np.sign(rng.standard_normal(4000)) * np.exp2(rng.uniform(-14, 8.8, 4000)),
                           [2.0 ** -12, -(2.0 ** -12), 0.0, -0.0, 447.99, -447.99]]).astype(np.float32)
    K = 256
    per = K - 1
    n_rows = (len(pool) + per - 1) // per
    x = np.zeros((n_rows, K), np.float32)
    x[:, 0] = 448.0
    flat = np.zeros(n_rows * per, np.float32)
    flat[:len(pool)] = pool
    x[:, 1:] = flat.reshape(n_rows, per)
    ones = torch.ones(K, device=DEV)
    xq, xs = sq.sq_quant_act_e4m3(torch.from_numpy(x).to(DEV), ones)
    np.testing.assert_array_equal(xs.cpu().numpy(), np.float32(448.0) / np.float32(448.0))
    np.testing.assert_array_equal(xq.cpu().numpy(), oracle.e4m3_encode(x))


def test_codes_next_to_e4m3_midpoints():
    # rows with absmax m (first value) and values within a few ulps of
    # (E4M3 midpoint) * delta, delta = fl(m / 448): v / delta lands next to a
    # rounding boundary of the format, where fl(v * fl(1/delta)) alone could
    # round to the neighbouring code
    vals = _finite_values()
    mids = ((vals[1:] + vals[:-1]) / 2)
    mids = mids[np.abs(mids) < 448]
    rng = np.random.default_rng(43)
    K, n_rows = 512, 32
    x = np.zeros((n_rows, K), np.float32)
    for t in range(n_rows):
        m = np.float32(rng.uniform(0.01, 100.0))
        d = np.float32(m / np.float32(448.0))
        x[t, 0] = m
        base = (rng.choice(mids, K - 1) * np.float64(d)).astype(np.float32)
        steps = rng.integers(-2, 3, K - 1)
        for i in range(K - 1):
            for _ in range(abs(int(steps[i]))):
                base[i] = np.nextafter(base[i], np.float32(np.inf) if steps[i] > 0 else np.float32(-np.inf))
        x[t, 1:] = np.clip(base, -m, m)
    ones = np.ones(K, np.float32)
    xq, xs = sq.sq_quant_act_e4m3(torch.from_numpy(x).to(DEV), torch.from_numpy(ones).to(DEV))
    xq_ref, xs_ref = oracle.quant_act_e4m3(x, ones)
    np.testing.assert_array_equal(xs.cpu().numpy(), xs_ref)
    np.testing.assert_array_equal(xq.cpu().numpy(), xq_ref)


@pytest.mark.parametrize("dt,K", [("bf16", 16), ("f32", 256), ("bf16", 1040), ("f16", 4096), ("bf16", 16384),
                                  ("f16", 28672), ("bf16", 40960)])
@pytest.mark.parametrize("M", [1, 37])
def test_quant_act_e4m3(dt, K, M):
    o = synth.outliers(K, frac=0.01, mult=80.0, seed=K)
    x = synth.activations(M, K, o, seed=K + M, dtype=TORCH_DT[dt])
    if M > 5:
        x[5] = 0  # all-zero token: scale 0, codes +0
        x[6, ::3] = -0.0
    inv = torch.exp(torch.randn(K, generator=synth.gen(K + 3)))
    xq, xs = sq.sq_quant_act_e4m3(x.to(DEV), inv.to(DEV))
    xq_ref, xs_ref = oracle.quant_act_e4m3(f32(x), inv.numpy())
    np.testing.assert_array_equal(xs.cpu().numpy(), xs_ref)
    np.testing.assert_array_equal(xq.cpu().numpy(), xq_ref)
    assert sq.sq_check_device_error() == sq.SQ_OK


# Long batches (8192 tokens or more) run on the staged row kernel (four
# vectors per thread for E4M3 codes).
@pytest.mark.parametrize("dt,K", [("bf16", 4096), ("f16", 7168), ("bf16", 16384)])
def test_quant_act_e4m3_long_batches(dt, K):
    M = 8200
    o = synth.outliers(K, frac=0.01, mult=80.0, seed=K + 11)
    x = synth.activations(M, K, o, seed=K + M, dtype=TORCH_DT[dt], kind="student_t3")
    x[9] = 0  # all-zero token
    inv = torch.exp(torch.randn(K, generator=synth.gen(K + 13)))
    xq, xs = sq.sq_quant_act_e4m3(x.to(DEV), inv.to(DEV))
    xq_ref, xs_ref = oracle.quant_act_e4m3(f32(x), inv.numpy())
    np.testing.assert_array_equal(xs.cpu().numpy(), xs_ref)
    np.testing.assert_array_equal(xq.cpu().numpy(), xq_ref)
    assert sq.sq_check_device_error() == sq.SQ_OK


@pytest.mark.parametrize("layout", ["kn", "nk"])
@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("K,N", [(48, 80), (1040, 528)])
def test_smooth_quant_weight_e4m3(layout, dt, K, N):
    seed = K * 5 + N
    w = synth.weights(K, N, seed, TORCH_DT[dt], layout)
    if layout == "kn":
        w[:, N // 2] = 0
    else:
        w[N // 2, :] = 0
    o = synth.outliers(K, count=max(1, K // 50), seed=seed + 1)
    amax = torch.from_numpy(oracle.calib_absmax(f32(synth.activations(64, K, o, seed + 2))))
    wq, ws, s, inv = sq.sq_smooth_quant_weight_e4m3(w.to(DEV), LAYOUT[layout], amax.to(DEV), 0.5)
    wmax = oracle.weight_absmax(f32(w), LAYOUT[layout])
    s_ref, inv_ref = oracle.smooth_factor(amax.numpy(), wmax, 0.5)
    wq_ref, ws_ref = oracle.smooth_quant_weight_e4m3(f32(w), LAYOUT[layout], s_ref)
    np.testing.assert_array_equal(s.cpu().numpy(), s_ref)
    np.testing.assert_array_equal(inv.cpu().numpy(), inv_ref)
    np.testing.assert_array_equal(ws.cpu().numpy(), ws_ref)
    np.testing.assert_array_equal(wq.cpu().numpy(), wq_ref)


def _codes(M, N, K, seed):
    """E4M3 operands as the quantizers produce them from outlier activations
    and Gaussian weights (every row reaches +-448)."""
    o = synth.outliers(K, frac=0.01, mult=60.0, seed=seed)
    x = synth.activations(M, K, o, seed=seed + 1, dtype=torch.float32)
    w = synth.weights(K, N, seed + 2, torch.float32, "nk")
    xq, dx = oracle.quant_act_e4m3(f32(x), np.ones(K, np.float32))
    wq, dw = oracle.smooth_quant_weight_e4m3(f32(w), oracle.LAYOUT_NK, np.ones(K, np.float32))
    return xq, dx, wq, dw


def _check_acc(acc_gpu, xq, wq):
    exact = oracle.gemm_e4m3(xq, wq)
    absum = np.abs(oracle.e4m3_decode(xq)).astype(np.float64) @ np.abs(oracle.e4m3_decode(wq)).astype(np.float64).T
    err = np.abs(acc_gpu.astype(np.float64) - exact)
    ratio = float((err / np.maximum(absum, 1e-300)).max())
    K = xq.shape[1]
    assert np.all(err <= acc_bound(K) * absum), f"max error / sum|xw| = {ratio:.3e} > {acc_bound(K):.3e}"
    return ratio


SHAPES = [(1, 256, 4096), (16, 4096, 4096), (33, 1024, 11008), (64, 28672, 1024), (8, 19968, 256),
          (200, 512, 4096), (300, 2048, 272), (1024, 4096, 2048), (300, 10000, 1040)]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_accumulate_e4m3_within_bound_and_deterministic(M, N, K):
    xq, dx, wq, dw = _codes(M, N, K, seed=M + N + K)
    xq_d, wq_d = torch.from_numpy(xq).to(DEV), torch.from_numpy(wq).to(DEV)
    acc = sq.sq_w8a8_accumulate_e4m3(xq_d, wq_d)
    acc2 = sq.sq_w8a8_accumulate_e4m3(xq_d, wq_d)
    assert torch.equal(acc, acc2)
    ratio = _check_acc(acc.cpu().numpy(), xq, wq)
    print(f"M={M} N={N} K={K}: max |acc - exact| / sum|xw| = {ratio:.3e}")
    assert sq.sq_check_device_error() == sq.SQ_OK


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_linear_e4m3_epilogue_exact(M, N, K, out):
    xq, dx, wq, dw = _codes(M, N, K, seed=3 * M + N + K)
    args = [torch.from_numpy(a).to(DEV) for a in (xq, dx, wq, dw)]
    acc = sq.sq_w8a8_accumulate_e4m3(args[0], args[2]).cpu().numpy()
    y = sq.sq_w8a8_linear_e4m3(*args, out_dtype=TORCH_DT[out])
    y_ref = oracle.dequant_f32acc(acc, dx, dw)
    if out == "f32":
        np.testing.assert_array_equal(y.cpu().numpy(), y_ref)
    else:
        np.testing.assert_array_equal(y.view(torch.int16).cpu().numpy().view(np.uint16), oracle.round_to(y_ref, "bf16"))


def test_pipeline_e4m3_approximates_the_product():
    # calibration -> smoothing -> E4M3 weights and activations -> linear:
    # within the E4M3 quantization error bound of the exact X W
    M, K, N = 64, 1024, 768
    o = synth.outliers(K, frac=0.01, mult=100.0, seed=5)
    x = synth.activations(M, K, o, seed=6, dtype=torch.float32)
    w = synth.weights(K, N, 7, torch.float32, "nk")
    amax = torch.zeros(K, device=DEV)
    sq.sq_calib_absmax(x.to(DEV), amax)
    wq, dw, s, inv = sq.sq_smooth_quant_weight_e4m3(w.to(DEV), sq.SQ_W_NK, amax, 0.5)
    xq, dx = sq.sq_quant_act_e4m3(x.to(DEV), inv)
    y = sq.sq_w8a8_linear_e4m3(xq, dx, wq, dw, out_dtype=torch.float32).cpu().numpy().astype(np.float64)
    xt = (f32(x) * inv.cpu().numpy()).astype(np.float64)
    wt = (f32(w) * s.cpu().numpy()[None, :]).astype(np.float64)   # [N, K]
    dxn, dwn = dx.cpu().numpy()[:, None], dw.cpu().numpy()[None, :]
    ex = np.abs(xt) * 2.0 ** -4 + 2.0 ** -10 * dxn
    ew = np.abs(wt) * 2.0 ** -4 + 2.0 ** -10 * dw.cpu().numpy()[:, None]
    bound = np.abs(xt) @ ew.T + ex @ np.abs(wt).T + ex @ ew.T
    exact = f32(x).astype(np.float64) @ f32(w).astype(np.float64).T
    assert np.all(np.abs(y - exact) <= bound * 1.01 + 1e-5 * np.abs(exact))
