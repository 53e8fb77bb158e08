"""Parity of the upstream-producer calls against the oracle.

sq_fold_smooth_into_norm: gs = gamma * inv_s, bit-exact.
sq_rmsnorm_quant_act: RMS normalisation with the folded weight gs +
per-token INT8.
The sum of squares is accumulated in double precision in an order neither
side fixes, so r_t may differ by one fp32 ulp; codes must then agree
everywhere except where the oracle's own pre-rounding value lies within
1e-4 of a rounding boundary, and there by at most one.  Scales agree within
two fp32 ulps.

sq_layernorm_quant_act: LayerNorm with the folded weight gs and bias bs +
per-token INT8; the mean and the variance are double-precision sums in an
order neither side fixes, with the same tolerance as above.

sq_static_act_scale / sq_quant_act_static: bit-exact, including values
beyond the calibrated range, which saturate at +-127.
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


def f32(t):
    return t.detach().to("cpu", torch.float32).numpy()


def _boundary_mask(x, gs, eps):
    """Elements whose oracle value v / (max|v| / 127) sits within 1e-4 of a
    half-integer, recomputed in fp32 with the oracle's own r."""
    r = oracle.rmsnorm_factor(x, eps)
    v = (x * r[:, None]).astype(np.float32)
    v = (v * gs).astype(np.float32)
    m = np.abs(v).max(axis=1)
    delta = (m / np.float32(127.0)).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        u = np.abs(np.where(delta[:, None] > 0, v / delta[:, None], 0).astype(np.float32)).astype(np.float64)
    return np.abs(u - np.floor(u) - 0.5) < 1e-4


@pytest.mark.parametrize("K", [16, 4096, 5000])
def test_fold_smooth_into_norm(K):
    g = synth.gen(K)
    gamma = torch.rand(K, generator=g) * 2.0 + 0.05
    inv_s = torch.exp(torch.randn(K, generator=g))
    gs = sq.sq_fold_smooth_into_norm(gamma.to(DEV), inv_s.to(DEV))
    np.testing.assert_array_equal(gs.cpu().numpy(), oracle.fold_norm_weight(gamma.numpy(), inv_s.numpy()))
    # in place over gamma
    gd = gamma.to(DEV)
    sq.sq_fold_smooth_into_norm(gd, inv_s.to(DEV), gs=gd)
    np.testing.assert_array_equal(gd.cpu().numpy(), gs.cpu().numpy())


@pytest.mark.parametrize("dt,K", [("bf16", 16), ("bf16", 256), ("f16", 1040), ("bf16", 4096), ("f32", 4096),
                                  ("f16", 11008), ("bf16", 16384), ("f32", 8192)])
@pytest.mark.parametrize("M", [1, 7, 300])
def test_rmsnorm_quant_act(dt, K, M):
    o = synth.outliers(K, frac=0.01, mult=50.0, seed=K)
    x = synth.activations(M, K, o, seed=K + M, dtype=TORCH_DT[dt])
    if M > 3:
        x[3] = 0  # an all-zero token: scale 0, codes 0
    g = synth.gen(K + 7)
    gamma = torch.rand(K, generator=g) * 2.0 + 0.05
    inv_s = torch.exp(torch.randn(K, generator=g))
    gs = oracle.fold_norm_weight(gamma.numpy(), inv_s.numpy())
    eps = 1e-5
    xq, xs = sq.sq_rmsnorm_quant_act(x.to(DEV), torch.from_numpy(gs).to(DEV), eps)
    xf = f32(x)
    xq_ref, xs_ref = oracle.rmsnorm_quant_act(xf, gs, eps)
    xs_g = xs.cpu().numpy()
    ulp = np.spacing(np.abs(xs_ref).astype(np.float32)).astype(np.float64)
    assert np.all(np.abs(xs_g.astype(np.float64) - xs_ref) <= 2 * ulp)
    diff = xq.cpu().numpy().astype(np.int32) - xq_ref.astype(np.int32)
    near = _boundary_mask(xf, gs, eps)
    assert np.abs(diff).max() <= 1
    assert np.all(diff[~near] == 0), f"{int((diff[~near] != 0).sum())} codes differ away from rounding boundaries"
    assert sq.sq_check_device_error() == sq.SQ_OK


def test_rmsnorm_quant_feeds_the_linear():
    M, K, N = 64, 4096, 512
    o = synth.outliers(K, frac=0.005, mult=100.0, seed=3)
    x = synth.activations(M, K, o, seed=4, dtype=torch.bfloat16)
    gamma = torch.rand(K, generator=synth.gen(5)) + 0.5
    w = synth.weights(K, N, 6, torch.bfloat16, "nk")
    amax = oracle.calib_absmax(f32(x))
    s, inv = oracle.smooth_factor(amax, oracle.weight_absmax(f32(w), oracle.LAYOUT_NK), 0.5)
    wq, dw = oracle.smooth_quant_weight(f32(w), oracle.LAYOUT_NK, s)
    gs = sq.sq_fold_smooth_into_norm(gamma.to(DEV), torch.from_numpy(inv).to(DEV))
    xq, xs = sq.sq_rmsnorm_quant_act(x.to(DEV), gs, 1e-6)
    y = sq.sq_w8a8_linear(xq, xs, torch.from_numpy(wq).to(DEV), torch.from_numpy(dw).to(DEV), torch.float32)
    # the linear is exact given the GPU's own codes and scales
    y_ref = oracle.dequant(oracle.gemm_i8(xq.cpu().numpy(), wq), xs.cpu().numpy(), dw)
    np.testing.assert_array_equal(y.cpu().numpy(), y_ref)


def _ln_boundary_mask(x, gs, bs, eps):
    """As _boundary_mask, for the oracle's LayerNorm value fma((x - mu) r, gs, bs)."""
    v = oracle.layernorm_values(x, gs, bs, eps)
    m = np.abs(v).max(axis=1)
    delta = (m / np.float32(127.0)).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        u = np.abs(np.where(delta[:, None] > 0, v / delta[:, None], 0).astype(np.float32)).astype(np.float64)
    return np.abs(u - np.floor(u) - 0.5) < 1e-4


@pytest.mark.parametrize("dt,K", [("bf16", 16), ("bf16", 256), ("f16", 1040), ("bf16", 4096), ("f32", 4096),
                                  ("f16", 11008), ("bf16", 16384), ("f32", 8192)])
@pytest.mark.parametrize("M", [1, 7, 300])
@pytest.mark.parametrize("bias", [True, False])
def test_layernorm_quant_act(dt, K, M, bias):
    o = synth.outliers(K, frac=0.01, mult=50.0, seed=K)
    x = synth.activations(M, K, o, seed=K + M + 11, dtype=TORCH_DT[dt])
    x += 0.75  # a nonzero mean for the normalisation to remove
    if M > 3:
        x[3] = 2.5  # a constant token: variance 0, every value -> the bias
    if M > 6:
        # a token with a large mean and a small spread (mean^2 / var ~ 1e5),
        # and one whose first value is an outlier
        x[5] = 1000.0 + 4.0 * torch.randint(-1, 2, (K,), generator=synth.gen(K + 10)).to(x.dtype)
        x[6, 0] = 3000.0
    g = synth.gen(K + 9)
    gamma = torch.rand(K, generator=g) * 2.0 + 0.05
    beta = torch.rand(K, generator=g) - 0.5
    inv_s = torch.exp(torch.randn(K, generator=g))
    gs = oracle.fold_norm_weight(gamma.numpy(), inv_s.numpy())
    bs = oracle.fold_norm_weight(beta.numpy(), inv_s.numpy()) if bias else None
    eps = 1e-5
    xq, xs = sq.sq_layernorm_quant_act(x.to(DEV), torch.from_numpy(gs).to(DEV),
                                       None if bs is None else torch.from_numpy(bs).to(DEV), eps)
    xf = f32(x)
    xq_ref, xs_ref = oracle.layernorm_quant_act(xf, gs, bs, eps)
    xs_g = xs.cpu().numpy()
    ulp = np.spacing(np.abs(xs_ref).astype(np.float32)).astype(np.float64)
    assert np.all(np.abs(xs_g.astype(np.float64) - xs_ref) <= 2 * ulp)
    diff = xq.cpu().numpy().astype(np.int32) - xq_ref.astype(np.int32)
    near = _ln_boundary_mask(xf, gs, bs, eps)
    assert np.abs(diff).max() <= 1
    assert np.all(diff[~near] == 0), f"{int((diff[~near] != 0).sum())} codes differ away from rounding boundaries"
    if M > 3 and not bias:
        assert xs_g[3] == 0 and not xq.cpu().numpy()[3].any()
    assert sq.sq_check_device_error() == sq.SQ_OK


def test_layernorm_quant_feeds_the_linear():
    # OPT-style block: LayerNorm with bias folded with 1/s, then the INT8
    # linear; the linear is exact given the GPU's own codes and scales
    M, K, N = 64, 4096, 512
    o = synth.outliers(K, frac=0.01, mult=60.0, seed=13)
    x = synth.activations(M, K, o, seed=14, dtype=torch.float16)
    g = synth.gen(15)
    gamma = torch.rand(K, generator=g) + 0.5
    beta = torch.rand(K, generator=g) - 0.5
    w = synth.weights(K, N, 16, torch.float16, "nk")
    amax = oracle.calib_absmax(f32(x))
    s, inv = oracle.smooth_factor(amax, oracle.weight_absmax(f32(w), oracle.LAYOUT_NK), 0.5)
    wq, dw = oracle.smooth_quant_weight(f32(w), oracle.LAYOUT_NK, s)
    inv_d = torch.from_numpy(inv).to(DEV)
    gs = sq.sq_fold_smooth_into_norm(gamma.to(DEV), inv_d)
    bs = sq.sq_fold_smooth_into_norm(beta.to(DEV), inv_d)
    xq, xs = sq.sq_layernorm_quant_act(x.to(DEV), gs, bs, 1e-5)
    y = sq.sq_w8a8_linear(xq, xs, torch.from_numpy(wq).to(DEV), torch.from_numpy(dw).to(DEV), torch.float32)
    y_ref = oracle.dequant(oracle.gemm_i8(xq.cpu().numpy(), wq), xs.cpu().numpy(), dw)
    np.testing.assert_array_equal(y.cpu().numpy(), y_ref)
    # and the codes are the oracle's (up to the boundary tolerance)
    xq_ref, _ = oracle.layernorm_quant_act(f32(x), gs.cpu().numpy(), bs.cpu().numpy(), 1e-5)
    assert np.abs(xq.cpu().numpy().astype(np.int32) - xq_ref).max() <= 1


@pytest.mark.parametrize("dt,K", [("bf16", 4096), ("f16", 1040), ("f32", 272)])
def test_static_scale_and_quantization(dt, K):
    o = synth.outliers(K, frac=0.01, mult=100.0, seed=K)
    calib = synth.activations(256, K, o, seed=K + 1, dtype=TORCH_DT[dt])
    x = synth.activations(50, K, o, seed=K + 2, dtype=TORCH_DT[dt])
    x[7] *= 4  # a token beyond the calibrated range: its codes saturate
    amax = oracle.calib_absmax(f32(calib))
    inv_s = np.exp(np.random.default_rng(K).uniform(-1.5, 1.5, K)).astype(np.float32)
    delta = sq.sq_static_act_scale(torch.from_numpy(amax).to(DEV), torch.from_numpy(inv_s).to(DEV))
    delta_ref = oracle.static_act_scale(amax, inv_s)
    assert delta.item() == np.float32(delta_ref)
    xq, xs = sq.sq_quant_act_static(x.to(DEV), torch.from_numpy(inv_s).to(DEV), delta)
    xq_ref, xs_ref = oracle.quant_act_static(f32(x), inv_s, delta_ref)
    np.testing.assert_array_equal(xq.cpu().numpy(), xq_ref)
    np.testing.assert_array_equal(xs.cpu().numpy(), xs_ref)
    assert (np.abs(xq_ref[7]) == 127).sum() > 0
    assert sq.sq_check_device_error() == sq.SQ_OK


@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_producers_on_strided_rows(dt):
    # rows K = 1024 wide inside a buffer with leading dimension K + 64: every
    # producer reads only its row's K values
    M, K = 19, 1024
    base = synth.activations(M, K + 64, synth.outliers(K + 64, frac=0.01, mult=40.0, seed=5), seed=6,
                             dtype=TORCH_DT[dt])
    base[:, K:] = 1.0e4  # beyond the row: would dominate every maximum if read
    x = base.to(DEV)[:, :K]
    xf = f32(base[:, :K])
    g = synth.gen(7)
    gamma = torch.rand(K, generator=g) + 0.5
    beta = torch.rand(K, generator=g) - 0.5
    inv_s = torch.exp(torch.randn(K, generator=g) * 0.5)
    gs = oracle.fold_norm_weight(gamma.numpy(), inv_s.numpy())
    bs = oracle.fold_norm_weight(beta.numpy(), inv_s.numpy())
    eps = 1e-5
    xq, xs = sq.sq_rmsnorm_quant_act(x, torch.from_numpy(gs).to(DEV), eps)
    xq_ref, xs_ref = oracle.rmsnorm_quant_act(xf, gs, eps)
    diff = xq.cpu().numpy().astype(np.int32) - xq_ref
    assert np.abs(diff).max() <= 1 and np.all(diff[~_boundary_mask(xf, gs, eps)] == 0)
    assert np.all(np.abs(xs.cpu().numpy().astype(np.float64) - xs_ref) <= 2 * np.spacing(xs_ref))
    xq, xs = sq.sq_layernorm_quant_act(x, torch.from_numpy(gs).to(DEV), torch.from_numpy(bs).to(DEV), eps)
    xq_ref, xs_ref = oracle.layernorm_quant_act(xf, gs, bs, eps)
    diff = xq.cpu().numpy().astype(np.int32) - xq_ref
    assert np.abs(diff).max() <= 1 and np.all(diff[~_ln_boundary_mask(xf, gs, bs, eps)] == 0)
    assert np.all(np.abs(xs.cpu().numpy().astype(np.float64) - xs_ref) <= 2 * np.spacing(xs_ref))
    amax = oracle.calib_absmax(xf)
    delta = sq.sq_static_act_scale(torch.from_numpy(amax).to(DEV), inv_s.to(DEV))
    xq, xs = sq.sq_quant_act_static(x, inv_s.to(DEV), delta)
    xq_ref, xs_ref = oracle.quant_act_static(xf, inv_s.numpy(), oracle.static_act_scale(amax, inv_s.numpy()))
    np.testing.assert_array_equal(xq.cpu().numpy(), xq_ref)
    np.testing.assert_array_equal(xs.cpu().numpy(), xs_ref)
    assert sq.sq_check_device_error() == sq.SQ_OK
