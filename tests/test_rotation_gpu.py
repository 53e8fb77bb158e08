"""Parity of the butterfly-rotated quantizers against the oracle: the
rotation's products and sums are the definition's own fp32 operations, so
codes and scales are bit-exact."""
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


def _table(n, seed, kind="random"):
    L = n.bit_length() - 1
    if kind == "hadamard":
        theta = np.full((L, n // 2), np.pi / 4)
    elif kind == "zero":
        theta = np.zeros((L, n // 2))
    else:
        theta = np.random.default_rng(seed).uniform(-np.pi, np.pi, (L, n // 2))
    c, s = np.cos(theta).astype(np.float32), np.sin(theta).astype(np.float32)
    cs = np.stack([c, s], axis=-1)  # [L, n/2, 2]
    return c, s, torch.from_numpy(np.ascontiguousarray(cs)).to(DEV)


@pytest.mark.parametrize("dt,K,n", [("bf16", 16, 2), ("bf16", 256, 4), ("bf16", 4096, 256), ("f16", 1040, 16),
                                    ("bf16", 11008, 128), ("f32", 4096, 128), ("f32", 272, 8),
                                    ("bf16", 16384, 64), ("f16", 2048, 32),
                                    # blocks wider than a warp: the shared-memory kernel
                                    ("bf16", 4096, 4096), ("bf16", 12288, 1024), ("f16", 16384, 16384),
                                    ("f32", 8192, 8192), ("f32", 768, 256), ("bf16", 1536, 512)])
@pytest.mark.parametrize("M", [1, 37])
def test_quant_act_rotated(dt, K, n, M):
    o = synth.outliers(K, frac=0.01, mult=80.0, seed=K)
    x = synth.activations(M, K, o, seed=K + M + n, dtype=TORCH_DT[dt])
    if M > 3:
        x[3] = 0
    inv = torch.exp(torch.randn(K, generator=synth.gen(K + 1)) * 0.5)
    c, s, cs = _table(n, n + K)
    xq, xs = sq.sq_quant_act_rotated(x.to(DEV), inv.to(DEV), n, cs)
    xq_ref, xs_ref = oracle.quant_act_rotated(f32(x), inv.numpy(), n, c, s)
    np.testing.assert_array_equal(xs.cpu().numpy(), xs_ref)
    np.testing.assert_array_equal(xq.cpu().numpy(), xq_ref)
    assert sq.sq_check_device_error() == sq.SQ_OK


@pytest.mark.parametrize("kind", ["hadamard", "zero"])
def test_special_angles(kind):
    M, K, n = 33, 4096, 256
    o = synth.outliers(K, frac=0.01, mult=100.0, seed=2)
    x = synth.activations(M, K, o, seed=3, dtype=torch.bfloat16)
    inv = torch.rand(K, generator=synth.gen(4)) + 0.5
    c, s, cs = _table(n, 0, kind)
    xq, xs = sq.sq_quant_act_rotated(x.to(DEV), inv.to(DEV), n, cs)
    xq_ref, xs_ref = oracle.quant_act_rotated(f32(x), inv.numpy(), n, c, s)
    np.testing.assert_array_equal(xq.cpu().numpy(), xq_ref)
    np.testing.assert_array_equal(xs.cpu().numpy(), xs_ref)
    if kind == "zero":  # the identity rotation is plain smoothing + quantization
        xq0, xs0 = sq.sq_quant_act(x.to(DEV), inv.to(DEV))
        assert torch.equal(xq, xq0) and torch.equal(xs, xs0)
    else:  # the Hadamard rotation spreads the outlier channels: smaller scales
        xq0, xs0 = sq.sq_quant_act(x.to(DEV), inv.to(DEV))
        assert float(xs.mean()) < float(xs0.mean())


@pytest.mark.parametrize("dt,K,N,n", [("bf16", 1024, 528, 256), ("f32", 272, 64, 16), ("f16", 4096, 256, 128),
                                      ("bf16", 4096, 64, 4096)])
def test_smooth_quant_weight_rotated(dt, K, N, n):
    w = synth.weights(K, N, K + N, TORCH_DT[dt], "nk")
    o = synth.outliers(K, count=max(1, K // 50), seed=K)
    amax = torch.from_numpy(oracle.calib_absmax(f32(synth.activations(64, K, o, K + 5))))
    c, s, cs = _table(n, K + n)
    wq, ws, sm, inv = sq.sq_smooth_quant_weight_rotated(w.to(DEV), amax.to(DEV), 0.5, n, cs)
    s_ref, inv_ref = oracle.smooth_factor(amax.numpy(), oracle.weight_absmax(f32(w), oracle.LAYOUT_NK), 0.5)
    np.testing.assert_array_equal(sm.cpu().numpy(), s_ref)
    np.testing.assert_array_equal(inv.cpu().numpy(), inv_ref)
    wq_ref, ws_ref = oracle.smooth_quant_weight_rotated(f32(w), oracle.LAYOUT_NK, s_ref, n, c, s)
    np.testing.assert_array_equal(ws.cpu().numpy(), ws_ref)
    np.testing.assert_array_equal(wq.cpu().numpy(), wq_ref)


def test_rotated_linear_matches_the_unrotated_product():
    # both operands rotated by the same R: the INT8 linear approximates X W
    M, K, N, n = 64, 2048, 512, 256
    o = synth.outliers(K, frac=0.01, mult=100.0, seed=8)
    x = synth.activations(M, K, o, seed=9, dtype=torch.bfloat16)
    w = synth.weights(K, N, 10, torch.bfloat16, "nk")
    amax = torch.zeros(K, device=DEV)
    sq.sq_calib_absmax(x.to(DEV), amax)
    c, s, cs = _table(n, 0, "hadamard")
    wq, ws, sm, inv = sq.sq_smooth_quant_weight_rotated(w.to(DEV), amax, 0.5, n, cs)
    xq, xs = sq.sq_quant_act_rotated(x.to(DEV), inv, n, cs)
    y = sq.sq_w8a8_linear(xq, xs, wq, ws, torch.float32).cpu().numpy().astype(np.float64)
    exact = f32(x).astype(np.float64) @ f32(w).astype(np.float64).T
    err = np.abs(y - exact).max() / np.abs(exact).max()
    assert err < 0.02, err


@pytest.mark.parametrize("n", [64, 1024])
def test_quant_act_rotated_strided_rows(n):
    # rows K wide inside a buffer with leading dimension K + 64
    M, K = 13, 2048
    base = synth.activations(M, K + 64, synth.outliers(K + 64, frac=0.01, mult=40.0, seed=8), seed=9,
                             dtype=torch.bfloat16)
    base[:, K:] = 1.0e4  # beyond the row: would dominate every maximum if read
    inv = torch.exp(torch.randn(K, generator=synth.gen(10)) * 0.5)
    c, s, cs = _table(n, n + 3)
    xq, xs = sq.sq_quant_act_rotated(base.to(DEV)[:, :K], inv.to(DEV), n, cs)
    xq_ref, xs_ref = oracle.quant_act_rotated(f32(base[:, :K]), inv.numpy(), n, c, s)
    np.testing.assert_array_equal(xs.cpu().numpy(), xs_ref)
    np.testing.assert_array_equal(xq.cpu().numpy(), xq_ref)

