"""Parity of every C-ABI call against the CPU oracle, element by element,
on the same seeded inputs (tests/../w8a8_post_quantization_channel_b200/synth.py).

Bar: INT8 codes, fp32 scales, s and 1/s, channel maxima and int32
accumulators bit-exact; outputs within max relative error 1e-2 (denominator
floored at 1e-6 * max|Y|) and, because both sides round the same fp32
products the same way, bit-exact as well.
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


def f32(t: torch.Tensor) -> np.ndarray:
    """Exact widening to fp32 numpy (f16/bf16 -> f32 is exact)."""
    return t.detach().to("cpu", torch.float32).numpy()


def out_bits(y: torch.Tensor) -> np.ndarray:
    y = y.detach().cpu()
    if y.dtype == torch.float32:
        return y.numpy()
    return y.view(torch.int16).numpy().view(np.uint16)


def oracle_y(y32: np.ndarray, dt: str) -> np.ndarray:
    return oracle.round_to(y32, dt)


def assert_y(gpu: torch.Tensor, ref_bits: np.ndarray, dt: str):
    g = out_bits(gpu)
    if dt == "f32":
        gv, rv = g.astype(np.float64), ref_bits.astype(np.float64)
    else:
        tdt = TORCH_DT[dt]
        gv = torch.from_numpy(g.view(np.int16)).view(tdt).to(torch.float64).numpy()
        rv = torch.from_numpy(ref_bits.view(np.int16)).view(tdt).to(torch.float64).numpy()
    floor = 1e-6 * max(np.abs(rv).max(), 1e-30)
    rel = np.abs(gv - rv) / np.maximum(np.abs(rv), floor)
    assert rel.max() <= 1e-2, f"max rel err {rel.max()}"
    np.testing.assert_array_equal(g, ref_bits)


def no_device_error():
    assert sq.sq_check_device_error() == sq.SQ_OK


# ---------------------------------------------------------------------------
# calibration
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("T,K", [(1, 16), (7, 48), (100, 272), (1000, 4096), (4099, 1040)])
def test_calib_absmax(dt, T, K):
    o = synth.outliers(K, count=max(1, K // 100), mult=100.0, seed=T + K)
    x = synth.activations(T, K, o, seed=T * 7 + K, dtype=TORCH_DT[dt])
    x[T // 2, K // 3] = -1234.5  # a negative extreme must count by magnitude
    amax = torch.zeros(K, device=DEV)
    cut = [(0, T)] if T < 3 else [(0, T // 3), (T // 3, T)]
    for a, b in cut:  # running maximum across calls
        sq.sq_calib_absmax(x[a:b].to(DEV), amax)
    ref = oracle.calib_absmax(f32(x))
    np.testing.assert_array_equal(amax.cpu().numpy(), ref)
    no_device_error()


def test_calib_padded_rows_and_empty():
    T, K, ld = 300, 256, 320
    base = synth.activations(T, ld, synth.outliers(ld, count=3, seed=1), seed=2, dtype=torch.bfloat16)
    x = base[:, :K]  # leading dimension 320 > K
    amax = torch.zeros(K, device=DEV)
    sq.sq_calib_absmax(base.to(DEV)[:, :K], amax)
    np.testing.assert_array_equal(amax.cpu().numpy(), oracle.calib_absmax(f32(x)))
    before = amax.clone()
    sq.sq_calib_absmax(torch.zeros(0, K, dtype=torch.bfloat16, device=DEV), amax)  # T == 0: no-op
    assert torch.equal(before, amax)
    no_device_error()


# ---------------------------------------------------------------------------
# smoothing factor + weight quantization
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("layout", ["kn", "nk"])
@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("alpha", [0.0, 0.25, 0.5, 0.75, 1.0, 0.3])
@pytest.mark.parametrize("K,N", [(48, 80), (272, 256), (1040, 528)])
def test_smooth_quant_weight(layout, dt, alpha, K, N):
    seed = K * 3 + N
    w = synth.weights(K, N, seed, TORCH_DT[dt], layout)
    # an all-zero output channel and an all-zero input channel
    if layout == "kn":
        w[:, N // 2] = 0
        w[K // 2, :] = 0
    else:
        w[N // 2, :] = 0
        w[:, K // 2] = 0
    o = synth.outliers(K, count=max(1, K // 50), seed=seed + 1)
    amax_t = torch.from_numpy(oracle.calib_absmax(f32(synth.activations(64, K, o, seed + 2))))
    amax_t[K // 4] = 0.0  # an input channel that never fired
    wq, ws, s, inv = sq.sq_smooth_quant_weight(w.to(DEV), LAYOUT[layout], amax_t.to(DEV), alpha)
    wmax = oracle.weight_absmax(f32(w), LAYOUT[layout])
    s_ref, inv_ref = oracle.smooth_factor(amax_t.numpy(), wmax, alpha)
    wq_ref, ws_ref = oracle.smooth_quant_weight(f32(w), LAYOUT[layout], s_ref)
    np.testing.assert_array_equal(s.cpu().numpy(), s_ref)
    np.testing.assert_array_equal(inv.cpu().numpy(), inv_ref)
    np.testing.assert_array_equal(wq.cpu().numpy(), wq_ref)
    np.testing.assert_array_equal(ws.cpu().numpy(), ws_ref)
    no_device_error()


# ---------------------------------------------------------------------------
# activation quantization: every register-tiling variant, the shared-memory
# staged kernel for long rows (K > 16384 at 16 bits, > 8192 at 32 bits) and
# the two-pass kernel beyond it
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dt,K", [("bf16", 16), ("bf16", 2048), ("bf16", 4096), ("f16", 11008), ("bf16", 16384),
                                  ("bf16", 28672), ("f16", 20480), ("bf16", 40960), ("f32", 256), ("f32", 4096),
                                  ("f32", 12288), ("f32", 20000), ("f16", 1040)])
@pytest.mark.parametrize("M", [1, 5, 33])
def test_quant_act(dt, K, M):
    o = synth.outliers(K, frac=0.01, mult=100.0, seed=K)
    x = synth.activations(M, K, o, seed=K + M, dtype=TORCH_DT[dt])
    if M > 2:
        x[2] = 0  # all-zero token
    inv = torch.exp(torch.randn(K, generator=synth.gen(K + 5)))
    xq, xs = sq.sq_quant_act(x.to(DEV), inv.to(DEV))
    xq_ref, xs_ref = oracle.quant_act(f32(x), inv.numpy())
    np.testing.assert_array_equal(xq.cpu().numpy(), xq_ref)
    np.testing.assert_array_equal(xs.cpu().numpy(), xs_ref)
    no_device_error()


# Heavy-tailed batches of a few hundred to ten thousand tokens: rows per CTA
# from one to dozens, a zero row among them.  Batches of 8192 rows or more
# run on the row kernel whose next rows are staged by cp.async, shorter ones
# on the one that holds the next row in registers.  The staged kernel takes
# eight vectors per thread at 16-bit K = 4096, 5120, 7168 and 11008 (two or
# more CTAs per SM) and four at K = 16384 and for fp32 rows.
@pytest.mark.parametrize("dt,K", [("bf16", 4096), ("bf16", 7168), ("f16", 16384), ("f32", 8192), ("f16", 1040),
                                  ("bf16", 11008), ("f16", 5120)])
@pytest.mark.parametrize("M", [300, 5000, 9000])
def test_quant_act_batch_kernels(dt, K, M):
    o = synth.outliers(K, frac=0.01, mult=100.0, seed=K + 1)
    x = synth.activations(M, K, o, seed=K + M + 1, dtype=TORCH_DT[dt], kind="student_t3")
    x[7] = 0  # all-zero token
    inv = torch.exp(torch.randn(K, generator=synth.gen(K + 6)))
    xq, xs = sq.sq_quant_act(x.to(DEV), inv.to(DEV))
    xq_ref, xs_ref = oracle.quant_act(f32(x), inv.numpy())
    np.testing.assert_array_equal(xs.cpu().numpy(), xs_ref)
    np.testing.assert_array_equal(xq.cpu().numpy(), xq_ref)
    no_device_error()


# Both sides of the row quantizers' routing: 2047 / 2048 rows of 7168 values
# (register / staged kernel), 7152 / 7168 values at 2048 rows, and the
# staged kernel's eight / four vectors per thread at 12288 / 13824 values.
@pytest.mark.parametrize("M,K,dt", [(2047, 7168, "bf16"), (2048, 7168, "bf16"), (2048, 7152, "f16"),
                                    (8192, 12288, "f16"), (8192, 13824, "bf16")])
def test_quant_act_routing_boundaries(M, K, dt):
    o = synth.outliers(K, frac=0.01, mult=100.0, seed=K + 3)
    x = synth.activations(M, K, o, seed=K + M + 3, dtype=TORCH_DT[dt], kind="student_t3")
    x[M - 1] = 0  # all-zero last token
    inv = torch.exp(torch.randn(K, generator=synth.gen(K + 7)))
    xq, xs = sq.sq_quant_act(x.to(DEV), inv.to(DEV))
    xq_ref, xs_ref = oracle.quant_act(f32(x), inv.numpy())
    np.testing.assert_array_equal(xs.cpu().numpy(), xs_ref)
    np.testing.assert_array_equal(xq.cpu().numpy(), xq_ref)
    no_device_error()


def _near_boundary_rows(n_rows, K, seed):
    """fp32 rows whose first value is the row's absmax m and whose other
    values sit within a few ulps of (k + 1/2) * delta, delta = fl(m / 127):
    v / delta lands next to a rounding boundary, where a reciprocal multiply
    alone could round to the other integer."""
    rng = np.random.default_rng(seed)
    x = np.zeros((n_rows, K), np.float32)
    for t in range(n_rows):
        m = np.float32(rng.uniform(0.5, 100.0))
        d = np.float32(m / np.float32(127.0))
        x[t, 0] = m
        k = rng.integers(-127, 127, K - 1)
        base = ((k + 0.5) * np.float64(d)).astype(np.float32)
        steps = rng.integers(-3, 4, K - 1)
        v = base.copy()
        for i in range(K - 1):
            for _ in range(abs(int(steps[i]))):
                v[i] = np.nextafter(v[i], np.float32(np.inf) if steps[i] > 0 else np.float32(-np.inf))
        x[t, 1:] = np.clip(v, -m, m)
    return x


@pytest.mark.parametrize("K", [16, 272, 4096, 20480])
def test_quant_act_near_rounding_boundaries(K):
    x = _near_boundary_rows(24, K, seed=K)
    ones = np.ones(K, np.float32)
    xq, xs = sq.sq_quant_act(torch.from_numpy(x).to(DEV), torch.from_numpy(ones).to(DEV))
    xq_ref, xs_ref = oracle.quant_act(x, ones)
    np.testing.assert_array_equal(xs.cpu().numpy(), xs_ref)
    np.testing.assert_array_equal(xq.cpu().numpy(), xq_ref)
    # the same values through the static path, with each row's own scale
    for t in (0, 5):
        delta = torch.tensor([xs_ref[t]], device=DEV)
        q, _ = sq.sq_quant_act_static(torch.from_numpy(x[t:t + 1]).to(DEV), torch.from_numpy(ones).to(DEV), delta)
        q_ref, _ = oracle.quant_act_static(x[t:t + 1], ones, float(xs_ref[t]))
        np.testing.assert_array_equal(q.cpu().numpy(), q_ref)
    no_device_error()


def test_weight_cols_near_rounding_boundaries():
    # W[K][N] columns with the same construction go through the column
    # quantizer (smoothing factor forced to 1: amax = w_j, alpha = 0.5)
    K, N = 64, 48
    w = np.ascontiguousarray(_near_boundary_rows(N, K, seed=7).T)  # [K][N]: column n = row n above
    amax = np.abs(w).max(axis=1).astype(np.float32)
    wq, ws, s, inv = sq.sq_smooth_quant_weight(torch.from_numpy(w).to(DEV), sq.SQ_W_KN, torch.from_numpy(amax).to(DEV),
                                               0.5)
    s_ref, _ = oracle.smooth_factor(amax, oracle.weight_absmax(w, oracle.LAYOUT_KN), 0.5)
    wq_ref, ws_ref = oracle.smooth_quant_weight(w, oracle.LAYOUT_KN, s_ref)
    np.testing.assert_array_equal(ws.cpu().numpy(), ws_ref)
    np.testing.assert_array_equal(wq.cpu().numpy(), wq_ref)


def test_quant_act_padded_rows_and_empty():
    M, K, ld = 9, 512, 640
    base = synth.activations(M, ld, synth.outliers(ld, count=5, seed=3), seed=4, dtype=torch.float16)
    inv = torch.exp(torch.randn(K, generator=synth.gen(6)))
    xq, xs = sq.sq_quant_act(base.to(DEV)[:, :K], inv.to(DEV))
    xq_ref, xs_ref = oracle.quant_act(f32(base[:, :K]), inv.numpy())
    np.testing.assert_array_equal(xq.cpu().numpy(), xq_ref)
    np.testing.assert_array_equal(xs.cpu().numpy(), xs_ref)
    xq0, xs0 = sq.sq_quant_act(torch.zeros(0, K, dtype=torch.float16, device=DEV), inv.to(DEV))
    assert xq0.shape == (0, K)
    no_device_error()


# ---------------------------------------------------------------------------
# tensor-core product and epilogue
# ---------------------------------------------------------------------------

GEMM_SHAPES = [(1, 16, 16), (3, 48, 160), (17, 272, 272), (129, 1040, 1040), (300, 4096, 48),
               (128, 256, 4096), (256, 512, 256), (200, 528, 1040), (64, 12288, 128), (513, 2064, 336)]


def _rand_codes(shape, seed):
    g = synth.gen(seed)
    return torch.randint(-127, 128, shape, generator=g, dtype=torch.int8)


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_accumulate_exact(M, N, K):
    xq = _rand_codes((M, K), M * 31 + K)
    wq = _rand_codes((N, K), N * 17 + K)
    acc = sq.sq_w8a8_accumulate(xq.to(DEV), wq.to(DEV))
    np.testing.assert_array_equal(acc.cpu().numpy(), oracle.gemm_i8(xq.numpy(), wq.numpy()))
    no_device_error()


# Shapes with at least one round of 256 x 256 tiles for every CTA pair, which
# the library runs on CTA pairs (tcgen05 cta_group::2): tails in M, N and K,
# including tiles whose second CTA's half of Xq or Wq lies entirely past the
# matrix edge.
PAIR_SHAPES = [(1000, 8464, 272), (2304, 4160, 144), (300, 16384, 256), (256, 18944, 256),
               (300, 10000, 1040), (512, 19200, 512)]


@pytest.mark.parametrize("M,N,K", PAIR_SHAPES)
def test_accumulate_exact_cta_pairs(M, N, K):
    xq = _rand_codes((M, K), M * 13 + K)
    wq = _rand_codes((N, K), N * 7 + K)
    acc = sq.sq_w8a8_accumulate(xq.to(DEV), wq.to(DEV))
    np.testing.assert_array_equal(acc.cpu().numpy(), oracle.gemm_i8(xq.numpy(), wq.numpy()))
    no_device_error()


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_linear_epilogue_cta_pairs(dt):
    M, N, K = 300, 16384, 256
    xq = _rand_codes((M, K), 21)
    wq = _rand_codes((N, K), 22)
    xs = torch.rand(M, generator=synth.gen(23)) * 1e-2
    ws = torch.rand(N, generator=synth.gen(24)) * 1e-2
    y = sq.sq_w8a8_linear(xq.to(DEV), xs.to(DEV), wq.to(DEV), ws.to(DEV), TORCH_DT[dt])
    y_ref = oracle_y(oracle.dequant(oracle.gemm_i8(xq.numpy(), wq.numpy()), xs.numpy(), ws.numpy()), dt)
    assert_y(y, y_ref, dt)
    no_device_error()


# Decode-shaped products (M <= 64 tokens): the weight-streaming kernels.
# Clusters of CTAs split several tiles' k-blocks and add partials through
# distributed shared memory (segments of one, two or more tiles per CTA,
# whole tiles stored directly); where no such split balances the SMs, the
# stream-K kernel adds them in the caller's workspace.  Tails in N (a
# partial 128-row tile) and in K, and every padded token count (16/32/48/64).
DECODE_SHAPES = [(1, 4096, 4096), (2, 272, 1040), (16, 1024, 8192), (17, 4096, 272), (33, 528, 4096),
                 (48, 16, 16), (64, 12288, 1040), (64, 1040, 11008), (8, 28672, 8192), (1, 8192, 8192),
                 (8, 11008, 4096), (1, 11008, 4096), (32, 4096, 11008), (64, 4096, 4096), (40, 1024, 8192),
                 (12, 12288, 4096), (3, 32768, 4096), (24, 4112, 1552)]


@pytest.mark.parametrize("M,N,K", DECODE_SHAPES)
def test_decode_shapes_exact_and_workspace_clean(M, N, K):
    xq = _rand_codes((M, K), M * 3 + K)
    wq = _rand_codes((N, K), N * 5 + K)
    xs = torch.rand(M, generator=synth.gen(M + 1)) * 1e-2
    ws = torch.rand(N, generator=synth.gen(N + 1)) * 1e-2
    need = sq.sq_w8a8_linear_workspace_size(M, N, K)
    # the stream-K kernel (and its workspace) exactly where tokens are few
    # and Wq tiles outnumber the SMs
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert (need > 0) == (M <= 32 and (N + 127) // 128 > sms)
    if need > 0:
        assert need >= M * N * 4
    work = torch.zeros(need, dtype=torch.uint8, device=DEV) if need > 0 else None
    acc_ref = oracle.gemm_i8(xq.numpy(), wq.numpy())
    xq_d, wq_d = xq.to(DEV), wq.to(DEV)
    for _ in range(2):  # two calls in a row on one workspace
        acc = sq.sq_w8a8_accumulate(xq_d, wq_d, workspace=work)
        np.testing.assert_array_equal(acc.cpu().numpy(), acc_ref)
        if work is not None:
            assert int(work.count_nonzero()) == 0  # left zero for the next call
    y_ref = oracle_y(oracle.dequant(acc_ref, xs.numpy(), ws.numpy()), "bf16")
    y = sq.sq_w8a8_linear(xq_d, xs.to(DEV), wq_d, ws.to(DEV), torch.bfloat16, workspace=work)
    assert_y(y, y_ref, "bf16")
    if work is not None:
        assert int(work.count_nonzero()) == 0
    no_device_error()


def test_binding_workspace_is_kept_per_stream_and_left_zero():
    # without a caller workspace the binding keeps one zeroed buffer per
    # (device, stream); the stream-K decode kernel leaves it zero, so calls
    # of different shapes reuse it
    shapes = [(8, 19968, 1040), (3, 32768, 512), (8, 19968, 1040)]
    for i, (M, N, K) in enumerate(shapes):
        assert sq.sq_w8a8_linear_workspace_size(M, N, K) > 0
        xq, wq = _rand_codes((M, K), 40 + i), _rand_codes((N, K), 50 + i)
        acc = sq.sq_w8a8_accumulate(xq.to(DEV), wq.to(DEV))
        np.testing.assert_array_equal(acc.cpu().numpy(), oracle.gemm_i8(xq.numpy(), wq.numpy()))
    key = (torch.device(DEV).index or 0, torch.cuda.current_stream().cuda_stream)
    cached = [w for k, w in sq._WORKSPACES.items() if k[1] == key[1]]
    assert len(cached) == 1 and int(cached[0].count_nonzero()) == 0
    no_device_error()


def test_accumulate_int32_extremes():
    M, N, K = 130, 272, 28672  # 127*127*28672 is the largest sum these layers reach
    xq = torch.full((M, K), 127, dtype=torch.int8)
    xq[1::2] = -127
    wq = torch.full((N, K), 127, dtype=torch.int8)
    wq[::3] = -127
    acc = sq.sq_w8a8_accumulate(xq.to(DEV), wq.to(DEV)).cpu().numpy()
    ref = oracle.gemm_i8(xq.numpy(), wq.numpy())
    np.testing.assert_array_equal(acc, ref)
    assert abs(int(ref.max())) == 127 * 127 * K
    no_device_error()


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("M,N,K", [(1, 256, 256), (37, 528, 1040), (129, 4096, 512), (300, 272, 2048)])
def test_linear_epilogue(dt, M, N, K):
    o = synth.outliers(K, frac=0.01, seed=K)
    x = synth.activations(M, K, o, seed=M + K)
    w = synth.weights(K, N, seed=N + K)
    s, inv = oracle.smooth_factor(oracle.calib_absmax(f32(x)), oracle.weight_absmax(f32(w), oracle.LAYOUT_NK), 0.5)
    wq_ref, ws_ref = oracle.smooth_quant_weight(f32(w), oracle.LAYOUT_NK, s)
    xq_ref, xs_ref = oracle.quant_act(f32(x), inv)
    y = sq.sq_w8a8_linear(torch.from_numpy(xq_ref).to(DEV), torch.from_numpy(xs_ref).to(DEV),
                          torch.from_numpy(wq_ref).to(DEV), torch.from_numpy(ws_ref).to(DEV), TORCH_DT[dt])
    y_ref = oracle_y(oracle.dequant(oracle.gemm_i8(xq_ref, wq_ref), xs_ref, ws_ref), dt)
    assert_y(y, y_ref, dt)
    no_device_error()


def test_linear_padded_output_and_empty():
    M, N, K, ldy = 40, 256, 512, 384
    xq = _rand_codes((M, K), 1)
    wq = _rand_codes((N, K), 2)
    xs = torch.rand(M, generator=synth.gen(3)) * 0.01
    ws = torch.rand(N, generator=synth.gen(4)) * 0.01
    ybuf = torch.full((M, ldy), 7.0, dtype=torch.bfloat16, device=DEV)
    sq.sq_w8a8_linear(xq.to(DEV), xs.to(DEV), wq.to(DEV), ws.to(DEV), torch.bfloat16, y=ybuf[:, :N])
    y_ref = oracle_y(oracle.dequant(oracle.gemm_i8(xq.numpy(), wq.numpy()), xs.numpy(), ws.numpy()), "bf16")
    assert_y(ybuf[:, :N], y_ref, "bf16")
    assert torch.all(ybuf[:, N:] == 7.0)  # nothing written past N
    y0 = sq.sq_w8a8_linear(torch.zeros(0, K, dtype=torch.int8, device=DEV), xs.to(DEV)[:0], wq.to(DEV),
                           ws.to(DEV), torch.bfloat16)
    assert y0.shape == (0, N)
    no_device_error()


# ---------------------------------------------------------------------------
# whole path
# ---------------------------------------------------------------------------

def _gpu_pipeline(calib_chunks, w, layout, alpha, x, out_dtype):
    K = x.shape[1]
    amax = torch.zeros(K, device=DEV)
    for c in calib_chunks:
        sq.sq_calib_absmax(c.to(DEV), amax)
    wq, ws, s, inv = sq.sq_smooth_quant_weight(w.to(DEV), LAYOUT[layout], amax, alpha)
    xq, xs = sq.sq_quant_act(x.to(DEV), inv)
    acc = sq.sq_w8a8_accumulate(xq, wq)
    y = sq.sq_w8a8_linear(xq, xs, wq, ws, out_dtype)
    no_device_error()
    return dict(amax=amax, s=s, inv_s=inv, wq=wq, dw=ws, xq=xq, dx=xs, acc=acc, y=y)


def test_single_linear_small_pipeline():
    d = synth.single_linear_small()
    g = _gpu_pipeline([d["calib"][:40], d["calib"][40:]], d["w"], d["layout"], d["alpha"], d["x"], torch.float32)
    r = oracle.pipeline([f32(d["calib"])], f32(d["w"]), oracle.LAYOUT_KN, d["alpha"], f32(d["x"]), "f32")
    for k in ("amax", "s", "inv_s", "wq", "dw", "xq", "dx", "acc"):
        np.testing.assert_array_equal(g[k].cpu().numpy(), r[k], err_msg=k)
    assert_y(g["y"], r["y"], "f32")


@pytest.mark.parametrize("layer", [0, 3])
def test_opt67b_layer_full_size_sampled(layer):
    """OPT-6.7B QKV (4096->12288) and FC2 (16384->4096) at the benchmark's
    sizes: M = 2048, calibration 128 x 512 tokens, fp16.  Channel maxima,
    s, Wq and the scales are compared in full; Xq, the accumulators and Y on
    a sample of token rows (the oracle computes those rows one by one)."""
    d = synth.opt67b_layer(layer)
    K, N, M = d["K"], d["N"], d["M"]
    calib = d["calib"]
    g = _gpu_pipeline([calib[a:b] for a, b in synth.chunks(calib.shape[0], 512)], d["w"], "nk", 0.5, d["x"],
                      torch.float16)
    amax = np.zeros(K, np.float32)
    for a, b in synth.chunks(calib.shape[0], 4096):
        amax = oracle.calib_absmax(f32(calib[a:b]), amax)
    np.testing.assert_array_equal(g["amax"].cpu().numpy(), amax)
    w = f32(d["w"])
    s, inv = oracle.smooth_factor(amax, oracle.weight_absmax(w, oracle.LAYOUT_NK), 0.5)
    np.testing.assert_array_equal(g["s"].cpu().numpy(), s)
    wq, dw = oracle.smooth_quant_weight(w, oracle.LAYOUT_NK, s)
    np.testing.assert_array_equal(g["wq"].cpu().numpy(), wq)
    np.testing.assert_array_equal(g["dw"].cpu().numpy(), dw)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, M - 1], np.random.default_rng(layer).integers(0, M, 11)]))
    xq, dx = oracle.quant_act(f32(d["x"][rows]), inv)
    np.testing.assert_array_equal(g["xq"].cpu().numpy()[rows], xq)
    np.testing.assert_array_equal(g["dx"].cpu().numpy()[rows], dx)
    acc = oracle.gemm_i8(xq, wq)
    np.testing.assert_array_equal(g["acc"].cpu().numpy()[rows], acc)
    y_ref = oracle_y(oracle.dequant(acc, dx, dw), "f16")
    assert_y(g["y"][torch.from_numpy(rows).to(DEV)], y_ref, "f16")
    # properties on every row: each token reaches the code 127
    assert torch.all(g["xq"].abs().amax(dim=1) == 127)
    assert torch.isfinite(g["y"]).all()


# ---------------------------------------------------------------------------
# the remaining configurations' sizes and distributions
# ---------------------------------------------------------------------------

def test_calib_widest_rows_student_t():
    """Calibration on the sweep's widest rows (K = 28672, bf16) with its
    heavy-tailed draws (Student-t, 3 degrees of freedom, 1% outlier channels
    x100), streamed in three calls."""
    T, K = 3000, 28672
    o = synth.outliers(K, frac=0.01, mult=100.0, seed=41)
    x = synth.activations(T, K, o, seed=42, dtype=torch.bfloat16, kind="student_t3")
    amax = torch.zeros(K, device=DEV)
    for a, b in ((0, 1000), (1000, 2001), (2001, T)):
        sq.sq_calib_absmax(x[a:b].to(DEV), amax)
    np.testing.assert_array_equal(amax.cpu().numpy(), oracle.calib_absmax(f32(x)))
    no_device_error()


@pytest.mark.parametrize("layout", ["kn", "nk"])
@pytest.mark.parametrize("K,N", [(8192, 8192), (28672, 1024)])
def test_smooth_quant_weight_sweep_sizes(layout, K, N):
    """The weight path on the sweep's [K, K] weights at K = 8192 and on a
    1024-channel slab of the 28672-wide ones, in both layouts, bf16."""
    w = synth.weights(K, N, K + N, torch.bfloat16, layout)
    o = synth.outliers(K, frac=0.01, mult=100.0, seed=K)
    amax = torch.from_numpy(oracle.calib_absmax(f32(synth.activations(256, K, o, K + 1, torch.bfloat16,
                                                                          "student_t3"))))
    wq, ws, s, inv = sq.sq_smooth_quant_weight(w.to(DEV), LAYOUT[layout], amax.to(DEV), 0.5)
    s_ref, inv_ref = oracle.smooth_factor(amax.numpy(), oracle.weight_absmax(f32(w), LAYOUT[layout]), 0.5)
    np.testing.assert_array_equal(s.cpu().numpy(), s_ref)
    np.testing.assert_array_equal(inv.cpu().numpy(), inv_ref)
    wq_ref, ws_ref = oracle.smooth_quant_weight(f32(w), LAYOUT[layout], s_ref)
    np.testing.assert_array_equal(ws.cpu().numpy(), ws_ref)
    np.testing.assert_array_equal(wq.cpu().numpy(), wq_ref)
    no_device_error()


@pytest.mark.parametrize("alpha", [0.25, 0.75])
@pytest.mark.parametrize("layer", [4, 6])
def test_llama2_7b_layer_other_alphas(alpha, layer):
    """A Llama-2-7B linear (gate 4096->11008, or down 11008->4096 whose input
    is SiLU(a)*b) at the migration strengths 0.25 and 0.75, bf16, M = 128
    tokens, 4096 calibration tokens: the whole path against the oracle."""
    d = synth.llama_layer(synth.LLAMA2_7B, layer, M=128, alpha=alpha)
    g = _gpu_pipeline([d["calib"][:2048], d["calib"][2048:]], d["w"], "nk", alpha, d["x"], torch.bfloat16)
    r = oracle.pipeline([f32(d["calib"])], f32(d["w"]), oracle.LAYOUT_NK, alpha, f32(d["x"]), "bf16")
    for k in ("amax", "s", "inv_s", "wq", "dw", "xq", "dx", "acc"):
        np.testing.assert_array_equal(g[k].cpu().numpy(), r[k], err_msg=k)
    assert_y(g["y"], r["y"], "bf16")
